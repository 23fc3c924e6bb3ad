"""The seeded input generator: determinism, chunk independence, rounding, recipe."""
import numpy as np

from awq_inputs import WORKLOADS, make_inputs, make_weight_rows, gen


def test_splitmix64_reference_values():
    # splitmix64 seeded with 0: the first outputs of the published generator
    key = np.uint64(0)
    w = gen.words(key, 0, 3)
    assert [int(x) for x in w] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_normal_is_chunk_independent_and_standard():
    key = gen.stream_key(123, gen.STREAM_X)
    z = gen.normal(key, 0, 200001)
    assert np.array_equal(gen.normal(key, 77, 1000), z[77:1077])
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01


def test_bf16_rounding_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20, -2.5])
    bits = gen.f64_to_bf16_bits(vals)
    assert list(bits) == [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xC020]


def test_workload_recipe_c1():
    wl = WORKLOADS["C1"]
    W, X = make_inputs(wl)
    W2, X2 = make_inputs(wl)
    assert np.array_equal(W, W2) and np.array_equal(X, X2)
    assert W.shape == (256, 512) and X.shape == (256, 512) and W.dtype == np.uint16
    assert np.array_equal(make_weight_rows(wl, [3, 200]), W[[3, 200]])
    outl = gen.pick_channels(wl.seed, wl.d_in, wl.outlier_count)
    assert len(set(outl.tolist())) == 5
    x = (X.astype(np.uint32) << 16).view(np.float32)
    a = np.abs(x).mean(axis=0)
    assert np.all(a[outl] > 8.0) and np.median(a) < 1.0
