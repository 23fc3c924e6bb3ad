"""The inference side on the GPU: awq_fold_inv_scales against the oracle's
fold (bit-exact: both sides round the same fp32 quotient to bf16), and
awq_w4a16_gemm against the oracle's W4A16 product on packed weights.

Tolerance of the product, with u the unit roundoff of the activation type
(fp16 2^-11, bf16 2^-8): the kernel rounds each dequantised weight once in
fp16 ((code - z) Delta) and twice in bf16 (Delta, then the product), so the
weight carries a relative error e_w <= u (fp16) or 2u (bf16); it accumulates
in fp32 and rounds Y once more. So |Y_gpu - Y| <= u |Y| + (e_w + d_in 2^-23)
sum_i |X'_ti| |W_hat_oi| to first order (the last term also covers fp32
accumulation of d_in products); the test allows 1.1 times that."""
import zlib

import numpy as np
import pytest

from awq_inputs import custom, gen, make_inputs
from oracle import awq_oracle as O

from gpu_util import to_device


def to_device_f16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.float16).cuda()

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import weight_only_int4_act_b200 as awq  # noqa: E402

UNIT = {"bf16": 2.0 ** -8, "f16": 2.0 ** -11}
W_ERR = {"bf16": 2, "f16": 1}   # roundings of the dequantised weight, in units of u
DTYPES = ["bf16", "f16"]

CASES = [
    # name, N, d_out, d_in, bits, group, symmetric
    ("decode_1", 1, 256, 512, 4, 128, False),            # K split across CTAs
    ("decode_16_4096", 16, 4096, 4096, 4, 128, False),   # K split, 32 output tiles
    ("ragged", 37, 200, 352, 4, 32, False),              # ragged N, d_out and last K step
    ("prefill_sym3", 300, 130, 256, 3, 64, True),        # two token tiles of 256
    ("g256", 5, 96, 768, 4, 256, False),
    ("g8", 64, 128, 512, 4, 8, False),
    ("g16_2bit_sym", 130, 256, 1024, 2, 16, True),
    ("prefill_4096", 4096, 4096, 4096, 4, 128, False),   # no split, 512 tiles
    ("prefill_ragged", 777, 640, 1152, 4, 128, False),   # ragged rows and tokens, an odd number of K steps
    ("decode_17_odd_steps", 17, 384, 1216, 4, 64, False),  # last unit of 3 K steps: a half pair
    ("decode_33", 33, 256, 2048, 4, 128, False),         # 64-row token boxes
    ("decode_long_k", 8, 128, 16384, 4, 128, False),     # one tile split over many CTAs
    ("decode_whole_tiles", 64, 1024, 2048, 4, 128, False),
    ("decode_g16", 24, 256, 1024, 4, 16, False),
]


def _scaled_layer(N, d_out, d_in, bits, group, symmetric, seed, dtype="bf16"):
    """W, X (bf16 bits), X' = X S^-1 in `dtype` (bits), s (fp32)."""
    wl = custom(d_out, d_in, N, bits=bits, symmetric=symmetric, group=group, seed=seed)
    Wb, Xb = make_inputs(wl)
    s32 = O.candidate_scales(O.act_stats(Xb), 0.5).astype(np.float32)
    X16 = Xb if dtype == "bf16" else O.to_f16_bits(O.widen_bf16(Xb).astype(np.float32))
    Xp = np.ascontiguousarray(O.fold_inv_scales(np.ascontiguousarray(X16.T), s32, dtype).T)
    return Wb, Xb, Xp, s32


def _dev(bits, dtype):
    return to_device(bits) if dtype == "bf16" else to_device_f16(bits)


def _check_product(Y, Xp, qw, sc, zr, group, dtype="bf16"):
    ref = O.w4a16_matmul(Xp, qw, sc, zr, group, dtype)
    What = O.dequant_packed(qw, sc, zr, group, Xp.shape[1])
    form = np.abs(O.widen(Xp, dtype)) @ np.abs(What).T
    u = UNIT[dtype]
    tol = 1.1 * (u * np.abs(ref) + (W_ERR[dtype] * u + Xp.shape[1] * 2.0 ** -23) * form) + 1e-30
    got = Y.float().cpu().numpy().astype(np.float64)
    bad = np.abs(got - ref) > tol
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], ref[bad][:5])
    return np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("name,N,d_out,d_in,bits,group,symmetric", CASES)
def test_w4a16_against_oracle(name, N, d_out, d_in, bits, group, symmetric, dtype):
    Wb, _, Xp, s32 = _scaled_layer(N, d_out, d_in, bits, group, symmetric, seed=zlib.crc32(name.encode()) % 1000,
                                   dtype=dtype)
    qw, sc, zr, _, _, _ = O.pack(Wb, s32.astype(np.float64), bits, group, symmetric)
    cfg = awq.make_cfg(bits, group, symmetric, 1)
    Y = awq.w4a16_gemm(_dev(Xp, dtype), torch.from_numpy(qw.view(np.int32)).cuda(),
                       torch.from_numpy(sc).cuda(), torch.from_numpy(zr).cuda(), cfg)
    torch.cuda.synchronize()
    assert Y.dtype == (torch.bfloat16 if dtype == "bf16" else torch.float16)
    rel = _check_product(Y, Xp, qw, sc, zr, group, dtype)
    print(name, dtype, "max |err| / max |Y| =", rel)


def test_w4a16_deterministic_and_workspace_error_clear():
    # 2 tiles of 32 K steps on 16 CTAs: every tile summed from 8 partial slabs
    N, d_out, d_in = 16, 256, 8192
    Wb, _, Xp, s32 = _scaled_layer(N, d_out, d_in, 4, 128, False, seed=11)
    qw, sc, zr, _, _, _ = O.pack(Wb, s32.astype(np.float64), 4, 128, False)
    cfg = awq.make_cfg(4, 128, False, 1)
    args = (to_device(Xp), torch.from_numpy(qw.view(np.int32)).cuda(), torch.from_numpy(sc).cuda(),
            torch.from_numpy(zr).cuda(), cfg)
    ws = awq.workspace(awq.w4a16_workspace_size(N, d_out, d_in, cfg))
    a = awq.w4a16_gemm(*args, ws=ws)
    b = awq.w4a16_gemm(*args, ws=ws)
    torch.cuda.synchronize()
    awq.workspace_error(ws)
    assert torch.equal(a, b)
    _check_product(a, Xp, qw, sc, zr, 128)


def test_pack_then_product_on_the_gpu():
    """The chain a user runs: GPU pack at s, fold S^-1 into the activations'
    producer, GPU product; checked against the oracle product on the GPU's
    own packed output, and the oracle pack decides the same codes off the
    rounding boundary."""
    N, d_out, d_in, g = 64, 384, 1024, 128
    Wb, Xb, Xp, s32 = _scaled_layer(N, d_out, d_in, 4, g, False, seed=12)
    cfg = awq.make_cfg(4, g, False, 1)
    W = to_device(Wb)
    s_dev = torch.from_numpy(s32).cuda()
    qw, sc, zr = awq.quantize_pack(W, s_dev, cfg)
    X_dev = to_device(Xb)
    # the activations' producer carries S^-1: here the activation rows themselves, channel on axis 1
    Xt = X_dev.t().contiguous()
    awq.fold_inv_scales(s_dev, Xt)
    Xp_dev = Xt.t().contiguous()
    assert np.array_equal(Xp_dev.view(torch.int16).cpu().numpy().view(np.uint16), Xp)
    Y = awq.w4a16_gemm(Xp_dev, qw, sc, zr, cfg)
    torch.cuda.synchronize()
    qw_h, sc_h, zr_h = qw.cpu().numpy().view(np.uint32), sc.cpu().numpy(), zr.cpu().numpy()
    _check_product(Y, Xp, qw_h, sc_h, zr_h, g)
    _, sc_ref, zr_ref, codes_ref, _, _ = O.pack(Wb, s32.astype(np.float64), 4, g, False)
    near = O.boundary_mask(Wb, s32.astype(np.float64), 4, g, False)
    assert not ((O.unpack_codes(qw_h, d_in) != codes_ref) & ~near).any()


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", [(512,), (512, 24), (384, 5), (256, 1)])
def test_fold_bit_exact(shape, dtype):
    rng = np.random.default_rng(40 + len(shape))
    x = (rng.standard_normal(shape) * 3).astype(np.float32)
    p = gen.f64_to_bf16_bits(x.astype(np.float64)) if dtype == "bf16" else O.to_f16_bits(x)
    s = np.exp(rng.standard_normal(shape[0]) * 1.5).astype(np.float32)
    dev = _dev(p, dtype)
    awq.fold_inv_scales(torch.from_numpy(s).cuda(), dev)
    torch.cuda.synchronize()
    got = dev.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, O.fold_inv_scales(p, s, dtype))
