"""Pins of the CPU oracle to facts fixed outside itself.

Each test ties one oracle function to something the pages print (fixtures in
tests/golden/ with their citation), a closed form, brute-force enumeration, a
statistical law, or an invariant of the mathematics, chosen so that a dropped
term, a wrong sign or index or a transposed operand in the oracle fails one of
them. No GPU is used.
"""
import json
import math
import pathlib

import numpy as np
import pytest

from oracle import awq_oracle as O
from awq_inputs import WORKLOADS, make_inputs, custom, gen

GOLD = json.loads((pathlib.Path(__file__).parent / "golden" / "p5_worked_examples.json").read_text())


def _bits(x):
    """float64 values that are exact in bf16 -> bf16 bit patterns."""
    b = gen.f64_to_bf16_bits(np.asarray(x, dtype=np.float64))
    assert np.array_equal(O.widen_bf16(b), np.asarray(x, dtype=np.float64))
    return b


# ---------------------------------------------------------------------------
# the pages' worked examples
# ---------------------------------------------------------------------------
def test_quantiser_nonlinearity_step_one():
    """Q(0.4)=0 but Q(0.8)/2=0.5 (AWQ, scholia-log §2.2). A symmetric INT4 group
    whose largest magnitude is 7 has step exactly 1."""
    f = GOLD["nonlinearity_step_one"]
    for w, expect in ((f["w"], f["Q_w"]), (f["w"] * f["s"], f["Q_sw"])):
        V = np.array([[7.0, w, 0, 0, 0, 0, 0, 0]])
        Vh, codes, delta, zero = O.quantize_groups(V, 4, 8, True)
        assert delta[0, 0] == f["step"]
        assert Vh[0, 1] == expect
    W = np.array([[7.0, f["w"], 0, 0, 0, 0, 0, 0]])
    s = np.ones(8)
    s[1] = f["s"]
    assert O.fake_quant(W, s, 4, 8, True)[0][0, 1] == f["Q_sw_over_s"]
    assert O.fake_quant(W, np.ones(8), 4, 8, True)[0][0, 1] == f["Q_w"]


def test_int4_group_worked_example():
    """w_max=1, Delta=1/7, w=0.05, x=10: output error -0.5 unscaled and
    (1/28 - 0.05)*10 = -1/7 ~ -0.143 with s=4 (AWQ, scholia-log §3.1)."""
    f = GOLD["int4_group_example"]
    g, i = 128, 37
    W = np.zeros((1, g))
    W[0, 0] = f["w_max"]
    W[0, i] = f["w_i"]
    X = np.zeros((1, g))
    X[0, i] = f["x_i"]
    _, codes, delta, _ = O.quantize_groups(W, f["bits"], g, True)
    assert delta[0, 0] == pytest.approx(f["delta"], rel=1e-15)
    assert abs(delta[0, 0] - f["delta_printed"]) < 5e-4
    assert codes[0, i] - 8 == f["unscaled_code"]
    dy = O.output_error(O.delta_weight(W, np.ones(g), 4, g, True), X)[0, 0]
    assert dy == pytest.approx(f["unscaled_dy"], abs=1e-15)

    s = np.ones(g)
    s[i] = f["s_i"]
    V = W * s
    assert V[0, i] == pytest.approx(f["scaled_w"])
    assert f["x_i"] / f["s_i"] == f["scaled_x"]
    Vh, codes, delta, _ = O.quantize_groups(V, 4, g, True)
    assert delta[0, 0] == pytest.approx(f["delta"], rel=1e-15)   # group max unchanged
    assert abs(V[0, i] / delta[0, 0] - f["scaled_ratio_printed"]) < 5e-3
    assert codes[0, i] - 8 == f["scaled_code"]
    assert abs((Vh[0, i] - V[0, i]) - f["scaled_weight_error_printed"]) < 5e-4
    dy4 = O.output_error(O.delta_weight(W, s, 4, g, True), X)[0, 0]
    assert dy4 == pytest.approx((1.0 / 28.0 - 0.05) * 10.0, rel=1e-12)
    assert abs(dy4 - f["scaled_dy_printed"]) < 5e-4
    assert abs(delta[0, 0] / s[i] - f["delta_eff_printed"]) < 5e-4


def test_range_expansion_example():
    """s=40 makes 0.05 -> 2 the group maximum; step 2/7 (AWQ, scholia-log §3.3)."""
    f = GOLD["range_expansion"]
    g, i = 128, 3
    W = np.zeros((1, g))
    W[0, 0] = f["w_max"]
    W[0, i] = f["w_i"]
    s = np.ones(g)
    s[i] = f["s_i"]
    _, _, delta, _ = O.quantize_groups(W * s, f["bits"], g, True)
    assert (W * s)[0, i] == pytest.approx(f["scaled_w"])
    assert delta[0, 0] == pytest.approx(f["delta"], rel=1e-15)
    assert abs(delta[0, 0] - f["delta_printed"]) < 5e-4


def test_output_error_products():
    """Delta Y = Delta W X for single products (AWQ, scholia-log §1.1)."""
    for dw, x, dy in GOLD["output_error_products"]["cases"]:
        assert O.output_error(np.array([[dw]]), np.array([[x]]))[0, 0] == pytest.approx(dy, rel=1e-12)


def test_output_error_orientation():
    """Delta W [rows, d_in] times X [N, d_in] gives [rows, N], entry (r, t) =
    sum_i dW[r,i] X[t,i]: checked on index-coded matrices (a transposed operand
    or swapped index fails)."""
    dW = np.arange(6, dtype=np.float64).reshape(2, 3)          # 2 rows, 3 channels
    X = 10.0 ** np.arange(12, dtype=np.float64).reshape(4, 3)  # 4 tokens
    D = O.output_error(dW, X)
    assert D.shape == (2, 4)
    for r in range(2):
        for t in range(4):
            assert D[r, t] == sum(dW[r, i] * X[t, i] for i in range(3))


# ---------------------------------------------------------------------------
# the quantiser: bounds, brute force, statistics
# ---------------------------------------------------------------------------
def _random_groups(rng, rows, g, mixed=True):
    V = rng.standard_normal((rows, g))
    if mixed:
        V[:, 0] = -np.abs(V[:, 0]) - 0.01
        V[:, 1] = np.abs(V[:, 1]) + 0.01
    return V


@pytest.mark.parametrize("bits,sym", [(4, False), (4, True), (3, True), (3, False), (2, False)])
def test_rounding_error_bound(bits, sym):
    """|v_hat - v| <= Delta/2 wherever no clipping applies ([P5] §2.3):
    symmetric grids always cover [-max|v|, max|v|]; asymmetric grids cover the
    group's range when it contains 0."""
    rng = np.random.default_rng(1)
    V = _random_groups(rng, 4000, 64)
    Vh, codes, delta, zero = O.quantize_groups(V, bits, 64, sym)
    err = np.abs(Vh - V)
    assert np.all(err <= delta.repeat(64, axis=1) * (0.5 + 1e-12))


def test_asymmetric_clips_one_signed_groups():
    """A group with all values positive has zero point 0; values beyond 15*Delta
    clip to code 15 (the range is not forced to include 0)."""
    V = np.linspace(1.0, 2.0, 16)[None, :]
    Vh, codes, delta, zero = O.quantize_groups(V, 4, 16, False)
    assert zero[0, 0] == 0
    assert delta[0, 0] == pytest.approx(1.0 / 15.0)
    assert codes.max() == 15 and codes.min() == 15
    assert Vh[0, -1] == pytest.approx(1.0)


@pytest.mark.parametrize("bits,sym", [(4, False), (3, True), (4, True), (3, False)])
def test_brute_force_codes(bits, sym):
    """For each element, the code is the one of all 2^b codes whose
    dequantised value is nearest to v (exact ties excluded), and the zero point
    is the integer in range nearest to -min/Delta."""
    rng = np.random.default_rng(2)
    g = 16
    V = _random_groups(rng, 300, g, mixed=False) * rng.uniform(0.1, 3.0, (300, 1))
    Vh, codes, delta, zero = O.quantize_groups(V, bits, g, sym)
    n = 2 ** bits
    for r in range(V.shape[0]):
        d, z = delta[r, 0], zero[r, 0]
        offs = 2 ** (bits - 1) if sym else z
        if not sym:
            cand_z = np.arange(n)
            dist = np.abs(-cand_z * d - V[r].min())
            assert z == cand_z[np.argmin(dist)]
        for i in range(g):
            cands = (np.arange(n) - offs) * d
            dist = np.abs(cands - V[r, i])
            order = np.argsort(dist)
            if dist[order[1]] - dist[order[0]] < 1e-12:
                continue
            assert codes[r, i] == order[0]
            assert Vh[r, i] == pytest.approx(cands[order[0]], abs=1e-15)


def test_symmetric_step_closed_form():
    """Symmetric step = max|v| / (2^(b-1) - 1) ([P1] 量化基础); 1/7 for a group
    maximum of 1 at INT4 and 1/3 at INT3; the -2^(b-1) code is never used."""
    V = np.array([[1.0, -0.5, 0.25, 0.0, 0.3, -0.9, 0.1, 0.2]])
    assert O.quantize_groups(V, 4, 8, True)[2][0, 0] == pytest.approx(1 / 7, rel=1e-15)
    assert O.quantize_groups(-V, 3, 8, True)[2][0, 0] == pytest.approx(1 / 3, rel=1e-15)
    rng = np.random.default_rng(3)
    for bits in (3, 4):
        codes = O.quantize_groups(rng.standard_normal((2000, 64)), bits, 64, True)[1]
        assert codes.min() >= 1


def test_asymmetric_zero_point_cases():
    """A range symmetric about 0 at INT4 (min=-7.5, max=7.5): Delta=1, z=rne(7.5)=8;
    a range starting at 0: z=0 and code = v/Delta."""
    V = np.array([[-7.5, 7.5, 0.0, 1.0]])
    _, codes, delta, zero = O.quantize_groups(V, 4, 4, False)
    assert delta[0, 0] == 1.0 and zero[0, 0] == 8
    assert list(codes[0]) == [0, 15, 8, 9]
    V = np.array([[0.0, 1.5, 3.0, 0.2]])
    _, codes, delta, zero = O.quantize_groups(V, 4, 4, False)
    assert zero[0, 0] == 0 and delta[0, 0] == pytest.approx(0.2)
    assert list(codes[0]) == [0, 8, 15, 1]


def test_degenerate_groups():
    """An all-zero group dequantises to exact zeros; an all-equal group too
    (the range floor keeps Delta > 0)."""
    V = np.zeros((2, 8))
    V[1] = 0.0
    for sym in (True, False):
        Vh, codes, delta, zero = O.quantize_groups(V, 4, 8, sym)
        assert np.all(Vh == 0.0) and np.all(delta > 0)


def test_uniform_error_variance():
    """Mean squared rounding error ~ Delta^2/12 ([P1] 误差分析) on 10^6 weights.
    Each group's extremes fix its grid, so the law is checked on the other
    elements, which fall uniformly within their cells."""
    rng = np.random.default_rng(4)
    V = rng.uniform(-1, 1, (8192, 128)) + rng.uniform(-0.5, 0.5, (8192, 1))
    for sym in (False, True):
        Vh, _, delta, _ = O.quantize_groups(V, 4, 128, sym)
        e2 = (Vh - V) ** 2 / (delta.repeat(128, axis=1) ** 2 / 12.0)
        order = np.argsort(V, axis=1)
        inner = np.take_along_axis(e2, order[:, 1:-1], axis=1)
        assert abs(inner.mean() - 1.0) < 0.01


def test_protected_channel_error_shrinks_by_s_squared():
    """Scaling one channel by s (without changing its group's range) divides
    that channel's restored error variance by s^2 ([P1] 误差分析,
    E_protected ~ (s_q/s_i)^2/12; [P5] §2.3 Delta_eff = Delta'/s)."""
    rng = np.random.default_rng(5)
    W = rng.uniform(-1, 1, (100000, 32))
    W[:, 0] = 1.0
    W[:, 1] = -1.0
    W[:, 2] = rng.uniform(-0.2, 0.2, 100000)
    base = O.fake_quant(W, np.ones(32), 4, 32, False)
    s = np.ones(32)
    s[2] = 3.0
    prot = O.fake_quant(W, s, 4, 32, False)
    d = base[2][:, 0]
    e0 = np.mean((base[0][:, 2] - W[:, 2]) ** 2 / (d ** 2 / 12))
    e1 = np.mean((prot[0][:, 2] - W[:, 2]) ** 2 / (d ** 2 / 12))
    assert abs(e0 - 1.0) < 0.02
    assert abs(e1 * 9.0 - 1.0) < 0.02


# ---------------------------------------------------------------------------
# statistics and scales
# ---------------------------------------------------------------------------
def test_act_stats_closed_form():
    """a_i = mean_t |X[t,i]| ([P1] 激活感知, [P5] §1.2): alternating signs of a
    per-channel magnitude give exactly that magnitude."""
    c = np.array([0.5, 1.0, 3.0, 0.0, 40.0, 0.125, 2.0, 7.0])
    X = np.array([(-1.0) ** t * c for t in range(6)])
    a = O.act_stats(_bits(X))
    assert np.array_equal(a, c)
    X2 = np.array([[1.0, 2.0], [3.0, -6.0], [0.0, 1.0]])
    assert np.allclose(O.act_stats(_bits(X2)), [4.0 / 3.0, 3.0], rtol=1e-15)


def test_act_stats_half_normal_mean():
    """For N(0,1) activations, E|x| = sqrt(2/pi)."""
    W, X = make_inputs(WORKLOADS["C1"])
    a = O.act_stats(X)
    outl = gen.pick_channels(WORKLOADS["C1"].seed, 512, 5)
    mask = np.ones(512, bool)
    mask[outl] = False
    assert abs(a[mask].mean() - math.sqrt(2 / math.pi)) < 0.01
    assert abs(a[outl].mean() / math.sqrt(2 / math.pi) - 20.0) < 1.0


def test_candidate_scales_closed_forms():
    a = np.array([1.0, 4.0, 2.0])
    assert np.array_equal(O.candidate_scales(a, 0.0), np.ones(3))   # alpha=0: no scaling ([P5] §4.1)
    for al in (0.25, 0.5, 0.95):
        s = O.candidate_scales(a, al)
        # normalisation: max(s) * min(s) = 1, so s = a^alpha / sqrt(4^alpha)
        assert s.max() * s.min() == pytest.approx(1.0, rel=1e-14)
        assert np.allclose(s, a ** al / 2.0 ** al, rtol=1e-14)
        assert np.allclose(O.candidate_scales(a, al, normalise=False), a ** al, rtol=1e-15)
    # the floor keeps dead channels positive
    s = O.candidate_scales(np.array([0.0, 1.0]), 0.5, normalise=False)
    assert s[0] == pytest.approx(1e-2) and s[1] == 1.0
    assert np.allclose(O.alpha_grid(20), [k / 20 for k in range(20)])


def test_normalisation_extremes_are_powers_of_the_extreme_statistics():
    """For alpha >= 0, t = max(a, eps)^alpha does not decrease as a grows, so
    max_j t_j and min_j t_j are the powers of the largest and smallest floored
    a_j (the GPU kernel takes the normalisation from those two values alone);
    the oracle's scales, built from every t_j, agree to float64 rounding."""
    rng = np.random.default_rng(17)
    for trial in range(20):
        a = np.exp(rng.standard_normal(rng.integers(8, 600)) * 2.0)
        a[rng.integers(0, a.size, 3)] = 0.0  # dead channels hit the floor
        for al in O.alpha_grid(20):
            t = np.maximum(a, O.EPS_A) ** al
            fl = np.maximum(a, O.EPS_A)
            assert t.max() == pytest.approx(fl.max() ** al, rel=1e-15)
            assert t.min() == pytest.approx(fl.min() ** al, rel=1e-15)
            shortcut = t / np.sqrt(fl.max() ** al * fl.min() ** al)
            assert np.allclose(O.candidate_scales(a, al), shortcut, rtol=1e-14, atol=0)


def test_scale_equivariance_of_normalisation():
    """Q(cV) = c Q(V) for c a power of two, so multiplying every s_i by c leaves
    Q(WS)S^-1 bit-identical; the sqrt(max*min) normalisation therefore only
    changes the loss by float64 rounding."""
    W, X = make_inputs(WORKLOADS["C1"])
    Wf = O.widen_bf16(W)
    a = O.act_stats(X)
    for sym, bits, g in ((False, 4, 128), (True, 3, 64)):
        s = O.candidate_scales(a, 0.6)
        ref = O.fake_quant(Wf, s, bits, g, sym)
        for c in (0.25, 8.0):
            got = O.fake_quant(Wf, c * s, bits, g, sym)
            assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])
        l_norm = O.loss_direct(ref[0] - Wf, X)
        su = O.candidate_scales(a, 0.6, normalise=False)
        l_raw = O.loss_direct(O.fake_quant(Wf, su, bits, g, sym)[0] - Wf, X)
        assert l_norm == pytest.approx(l_raw, rel=1e-9)


def test_identity_without_quantisation():
    """(W S)(S^-1 X^T) = W X^T for positive s, to float64 rounding ([P5] §2.1)."""
    rng = np.random.default_rng(6)
    W = rng.standard_normal((16, 64))
    X = rng.standard_normal((32, 64))
    s = O.candidate_scales(rng.uniform(0.01, 50, 64), 0.7)
    lhs = O.output_error(W * s, X / s)
    rhs = O.output_error(W, X)
    assert np.allclose(lhs, rhs, rtol=1e-13, atol=1e-12)


# ---------------------------------------------------------------------------
# the search: special cases, brute force, reassociation
# ---------------------------------------------------------------------------
def _rtn_reference(W, bits, g):
    """Plain asymmetric round-to-nearest per group, written with scalar loops."""
    rows, d_in = W.shape
    out = np.zeros_like(W)
    levels = 2 ** bits - 1
    for r in range(rows):
        for g0 in range(0, d_in, g):
            grp = [float(v) for v in W[r, g0:g0 + g]]
            lo, hi = min(grp), max(grp)
            step = max(hi - lo, 1e-8) / levels
            zp = min(max(round(-lo / step), 0), levels)
            for j, v in enumerate(grp):
                q = min(max(round(v / step) + zp, 0), levels)
                out[r, g0 + j] = (q - zp) * step
    return out


def test_alpha_zero_is_plain_rtn():
    """alpha = 0 gives s = 1, so the candidate is plain group RTN of W
    ([P5] §4.1)."""
    wl = custom(8, 256, 16, seed=11)
    W, X = make_inputs(wl)
    a = O.act_stats(X)
    Wf = O.widen_bf16(W)
    s0 = O.candidate_scales(a, 0.0)
    assert np.array_equal(s0, np.ones(256))
    What = O.fake_quant(Wf, s0, 4, 128, False)[0]
    assert np.array_equal(What, _rtn_reference(Wf, 4, 128))
    res = O.search(W, X, a, 4, 128, False, 20)
    dW = What - Wf
    brute = sum(sum(sum(dW[r, i] * float(xv) for i, xv in enumerate(O.widen_bf16(X)[t])) ** 2
                    for t in range(16)) for r in range(8))
    assert res["losses"][0] == pytest.approx(brute, rel=1e-12)


@pytest.mark.parametrize("sym,bits", [(False, 4), (True, 3)])
def test_brute_force_loss_tiny(sym, bits):
    """d_out=2, d_in=g=8, N=3: the loss for each alpha equals a triple loop over
    (row, token, channel) with the dequantised weights found by enumerating
    every code."""
    rng = np.random.default_rng(7)
    W = _bits(O.widen_bf16(gen.f64_to_bf16_bits(rng.standard_normal((2, 8)) * 0.05)))
    X = _bits(O.widen_bf16(gen.f64_to_bf16_bits(rng.standard_normal((3, 8)) * np.array([1, 1, 9, 1, 1, 1, 2, 1]))))
    Wf, Xf = O.widen_bf16(W), O.widen_bf16(X)
    a = np.abs(Xf).mean(axis=0)
    res = O.search(W, X, O.act_stats(X), bits, 8, sym, 5)
    for k, al in enumerate(O.alpha_grid(5)):
        s = O.candidate_scales(a, al)
        total = 0.0
        for r in range(2):
            v = Wf[r] * s
            if sym:
                d = np.abs(v).max() / (2 ** (bits - 1) - 1)
                grid = np.arange(-(2 ** (bits - 1)), 2 ** (bits - 1)) * d
            else:
                d = (v.max() - v.min()) / (2 ** bits - 1)
                z = min(range(2 ** bits), key=lambda c: abs(c * d + v.min()))
                grid = (np.arange(2 ** bits) - z) * d
            vh = np.array([grid[np.argmin(np.abs(grid - x))] for x in v])
            dw = vh / s - Wf[r]
            for t in range(3):
                total += sum(dw[i] * Xf[t, i] for i in range(8)) ** 2
        assert res["losses"][k] == pytest.approx(total, rel=1e-12)


def test_direct_and_gram_forms_agree():
    """||dW X^T||_F^2 = sum_r dW_r (X^T X) dW_r^T, to float64 rounding."""
    W, X = make_inputs(WORKLOADS["C1"])
    a = O.act_stats(X)
    d = O.search(W, X, a, 4, 128, False, 20, form="direct")
    g = O.search(W, X, a, 4, 128, False, 20, form="gram")
    assert np.allclose(d["losses"], g["losses"], rtol=1e-12)
    assert d["best"] == g["best"]
    rows = [0, 5, 255]
    sub = O.search(W, X, a, 4, 128, False, 20, rows=rows)
    full_rows = O.search(W[rows], X, a, 4, 128, False, 20)
    assert np.allclose(sub["row_losses"].sum(axis=1), full_rows["losses"], rtol=1e-13)


def test_choice_rules():
    assert O.choose(np.array([3.0, 1.0, 1.0, 2.0])) == 1
    assert O.acceptable_choices(np.array([3.0, 1.0, 1.004, 1.006])) == [1, 2]


def test_search_prefers_scaling_on_outlier_layer():
    """Expected direction (not a fixed value): with outlier channels the best
    alpha beats plain RTN (alpha = 0) on C1."""
    W, X = make_inputs(WORKLOADS["C1"])
    res = O.search(W, X, O.act_stats(X), 4, 128, False, 20)
    assert res["best"] > 0
    assert res["losses"][res["best"]] < res["losses"][0]


# ---------------------------------------------------------------------------
# pack
# ---------------------------------------------------------------------------
def test_pack_nibble_order():
    codes = np.array([[0, 1, 2, 3, 4, 5, 6, 7, 15, 15, 15, 15, 15, 15, 15, 15]])
    words = O.pack_codes(codes)
    assert words.dtype == np.uint32
    assert list(words[0]) == [0x76543210, 0xFFFFFFFF]
    for j in range(8):
        c = np.zeros((1, 8), dtype=np.int64)
        c[0, j] = 1
        assert O.pack_codes(c)[0, 0] == 1 << (4 * j)


def test_fp16_rounding_is_nearest_even():
    assert O.to_fp16(1.0 + 2.0 ** -11) == 1.0
    assert O.to_fp16(1.0 + 3 * 2.0 ** -11) == 1.0 + 2.0 ** -9
    assert O.to_fp16(1.0 + 2.0 ** -11 + 2.0 ** -30) == 1.0 + 2.0 ** -10


def test_pack_layer_consistency():
    """Unpacking the words, and dequantising with the float64 step and zero,
    reproduces Q(WS) for every element."""
    W, X = make_inputs(WORKLOADS["C1"])
    a = O.act_stats(X)
    s = O.candidate_scales(a, 0.45)
    qw, sc, zr, codes, delta, zero = O.pack(W, s, 4, 128, False)
    assert qw.shape == (256, 64) and sc.shape == (256, 4) and sc.dtype == np.float16
    unpacked = np.stack([(qw >> np.uint32(4 * j)) & np.uint32(0xF) for j in range(8)], axis=-1).reshape(256, 512)
    assert np.array_equal(unpacked, codes)
    Vh = (codes - zero.repeat(128, axis=1)) * delta.repeat(128, axis=1)
    ref = O.fake_quant(O.widen_bf16(W), s, 4, 128, False)[0] * s
    assert np.allclose(Vh, ref, rtol=1e-14, atol=1e-18)
    assert np.array_equal(zr.astype(np.float64), zero)


# ---------------------------------------------------------------------------
# clipping and arbitrary candidates
# ---------------------------------------------------------------------------
def test_clip_one_is_plain_quantiser():
    rng = np.random.default_rng(20)
    V = rng.standard_normal((50, 128))
    for sym in (False, True):
        a = O.quantize_groups(V, 4, 128, sym)
        b = O.quantize_groups(V, 4, 128, sym, clip=1.0)
        assert all(np.array_equal(x, y) for x, y in zip(a, b))


def test_clip_closed_forms():
    """With ratio c the step is c*range/(2^b-1) (asymmetric) or
    c*max|v|/(2^(b-1)-1) (symmetric), and values beyond the shrunk range take
    the extreme codes."""
    V = np.array([[-1.0, -0.2, 0.1, 0.4, 2.0, 0.0, 0.3, -0.5]])
    _, codes, delta, zero = O.quantize_groups(V, 4, 8, False, clip=0.5)
    assert delta[0, 0] == pytest.approx(0.5 * 3.0 / 15.0)
    assert zero[0, 0] == np.rint(0.5 / delta[0, 0])       # -min' / Delta = 0.5 / 0.1 = 5
    assert codes[0, 4] == 15 and codes[0, 0] == 0           # 2.0 > 1.0 = max', -1.0 < -0.5 = min'
    _, codes, delta, _ = O.quantize_groups(V, 4, 8, True, clip=0.25)
    assert delta[0, 0] == pytest.approx(0.25 * 2.0 / 7.0)
    assert codes[0, 4] == 15 and codes[0, 0] == 0           # 2.0 and -1.0 clip to q = 7 and q = -8


def test_clip_brute_force_codes():
    """Clipped codes are the nearest dequantised grid points (exact ties excluded)."""
    rng = np.random.default_rng(21)
    V = rng.standard_normal((200, 16))
    for sym, bits in ((False, 4), (True, 3)):
        Vh, codes, delta, zero = O.quantize_groups(V, bits, 16, sym, clip=0.7)
        n = 2 ** bits
        for r in range(V.shape[0]):
            offs = 2 ** (bits - 1) if sym else zero[r, 0]
            cands = (np.arange(n) - offs) * delta[r, 0]
            for i in range(16):
                dist = np.abs(cands - V[r, i])
                o = np.argsort(dist)
                if dist[o[1]] - dist[o[0]] < 1e-12:
                    continue
                assert codes[r, i] == o[0]


def test_search_candidates_matches_search():
    """The alpha grid given as explicit candidates reproduces search()."""
    W, X = make_inputs(WORKLOADS["C1"])
    a = O.act_stats(X)
    ref = O.search(W, X, a, 4, 128, False, 5)
    s_cand = np.stack([O.candidate_scales(a, al) for al in O.alpha_grid(5)])
    got = O.search_candidates(W, X, s_cand, 4, 128, False)
    assert np.allclose(got["losses"], ref["losses"], rtol=1e-14) and got["best"] == ref["best"]
    # clip ratio 1 changes nothing; clipping a lot increases the loss
    clipped = O.search_candidates(W, X, np.stack([s_cand[2]] * 3), 4, 128, False, clips=[1.0, 0.9, 0.3])
    assert clipped["losses"][0] == pytest.approx(ref["losses"][2], rel=1e-14)
    assert clipped["losses"][2] > clipped["losses"][0]


def test_per_group_clip_clamp_matches_scalar():
    """A per-group clip array applies each group's own ratio."""
    rng = np.random.default_rng(22)
    V = rng.standard_normal((6, 32))
    clip = np.array([[1.0, 0.5]] * 6)
    full = O.quantize_groups(V, 4, 16, False, clip=clip)
    for j, c in enumerate((1.0, 0.5)):
        part = O.quantize_groups(V[:, 16 * j:16 * (j + 1)], 4, 16, False, clip=c)
        assert np.array_equal(full[0][:, 16 * j:16 * (j + 1)], part[0])


def test_group_clip_errors_brute_force():
    """err[c, r, j] equals the direct per-group output error with a triple loop
    over tokens and the group's channels."""
    rng = np.random.default_rng(23)
    Wb = gen.f64_to_bf16_bits(rng.standard_normal((3, 32)) * 0.05)
    Xb = gen.f64_to_bf16_bits(rng.standard_normal((5, 32)) * np.linspace(0.5, 3, 32))
    s = O.candidate_scales(O.act_stats(Xb), 0.4)
    clips = [1.0, 0.8, 0.6]
    err = O.group_clip_errors(Wb, Xb, s, 4, 16, False, clips)
    W, X = O.widen_bf16(Wb), O.widen_bf16(Xb)
    for ci, c in enumerate(clips):
        dW = O.delta_weight(W, s, 4, 16, False, c)
        for r in range(3):
            for j in range(2):
                tot = 0.0
                for t in range(5):
                    tot += sum(dW[r, i] * X[t, i] for i in range(16 * j, 16 * j + 16)) ** 2
                assert err[ci, r, j] == pytest.approx(tot, rel=1e-12, abs=1e-300)
    best = O.group_clip_choice(err)
    assert best.shape == (3, 2)
    assert np.all(err[best, np.arange(3)[:, None], np.arange(2)[None, :]] <= err[0] + 0.0)


# ---------------------------------------------------------------------------
# inference side: fold, unpack, dequantise, W4A16 product
# ---------------------------------------------------------------------------
def test_bf16_rounding_matches_torch():
    """to_bf16_bits is round-to-nearest-even; torch's CPU float32 -> bfloat16
    conversion is the library routine it must equal (ties included)."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(30)
    x = (rng.standard_normal(20000) * np.exp(rng.standard_normal(20000) * 4)).astype(np.float32)
    ties = (np.arange(1, 2001, dtype=np.uint32) << np.uint32(16)) | np.uint32(0x8000)  # exact midpoints
    x = np.concatenate([x, ties.view(np.float32), np.array([0.0, -0.0, np.inf, -np.inf], dtype=np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.to_bf16_bits(x), ref)


def test_fold_matches_library_and_special_cases():
    """p / s_i per channel (first axis), fp32 quotient rounded to bf16: equals
    torch's float32 division + bfloat16 rounding; s = 1 leaves p unchanged and a
    power-of-two s only moves the exponent."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(31)
    p = gen.f64_to_bf16_bits(rng.standard_normal((64, 24)))
    s = np.exp(rng.standard_normal(64)).astype(np.float32)
    ref = (torch.from_numpy(O.widen_bf16(p).astype(np.float32)) / torch.from_numpy(s)[:, None]).to(torch.bfloat16)
    assert np.array_equal(O.fold_inv_scales(p, s), ref.view(torch.int16).numpy().view(np.uint16))
    vec = p[:, 0]
    assert np.array_equal(O.fold_inv_scales(vec, np.ones(64, dtype=np.float32)), vec)
    folded = O.widen_bf16(O.fold_inv_scales(vec, np.full(64, 4.0, dtype=np.float32)))
    assert np.array_equal(folded, O.widen_bf16(vec) / 4.0)


def test_unpack_inverts_pack_codes():
    rng = np.random.default_rng(32)
    codes = rng.integers(0, 16, size=(5, 64))
    assert np.array_equal(O.unpack_codes(O.pack_codes(codes), 64), codes)


@pytest.mark.parametrize("symmetric,bits", [(False, 4), (True, 4), (False, 3), (True, 2)])
def test_dequant_of_pack_is_fake_quant_up_to_fp16_step(symmetric, bits):
    """dequant_packed(pack(W, s)) reproduces Q(W S) from quantize_groups, and
    the difference is exactly (code - z)(fp16(Delta) - Delta): the zero point
    is an integer <= 15, exact in fp16, so the fp16 step is the only rounding."""
    rng = np.random.default_rng(33 + bits)
    Wb = gen.f64_to_bf16_bits(rng.standard_normal((6, 256)) * 0.02)
    s = np.exp(rng.standard_normal(256) * 0.5)
    qw, sc, zr, codes, delta, zero = O.pack(Wb, s, bits, 64, symmetric)
    Vh = O.quantize_groups(O.widen_bf16(Wb) * s[None, :], bits, 64, symmetric)[0]
    deq = O.dequant_packed(qw, sc, zr, 64, 256)
    assert np.array_equal(zr.astype(np.float64), zero)
    expected = (codes - np.repeat(zero, 64, axis=1)) * np.repeat(sc.astype(np.float64) - delta, 64, axis=1)
    assert np.allclose(deq - Vh, expected, rtol=0, atol=1e-12 * np.abs(Vh).max())
    assert np.all(np.abs(deq - Vh) <= (2 ** bits - 1) * 2.0 ** -11 * np.repeat(delta, 64, axis=1) + 1e-15)


def test_w4a16_exact_on_the_grid():
    """Weights already on the asymmetric grid with a power-of-two step (every
    group holds codes 0 and 15) and s = 1: the pack is lossless, so the
    quantised layer equals the plain product."""
    rng = np.random.default_rng(34)
    rows, d_in, g = 8, 128, 32
    codes = rng.integers(0, 16, size=(rows, d_in))
    codes[:, ::g] = 0
    codes[:, 1::g] = 15
    z = rng.integers(1, 15, size=(rows, d_in // g))
    W = (codes - np.repeat(z, g, axis=1)) * 2.0 ** -6
    Wb = gen.f64_to_bf16_bits(W)
    assert np.array_equal(O.widen_bf16(Wb), W)
    qw, sc, zr, c2, _, _ = O.pack(Wb, np.ones(d_in), 4, g, False)
    assert np.array_equal(c2, codes)
    Xb = gen.f64_to_bf16_bits(rng.standard_normal((5, d_in)))
    Y = O.w4a16_matmul(Xb, qw, sc, zr, g)
    assert np.allclose(Y, O.widen_bf16(Xb) @ W.T, rtol=1e-13, atol=0)


def test_w4a16_brute_force():
    """Triple loop with the nibbles taken out of the words one by one."""
    rng = np.random.default_rng(35)
    rows, d_in, g, N = 3, 32, 16, 2
    Wb = gen.f64_to_bf16_bits(rng.standard_normal((rows, d_in)) * 0.1)
    qw, sc, zr, _, _, _ = O.pack(Wb, np.ones(d_in), 4, g, False)
    Xb = gen.f64_to_bf16_bits(rng.standard_normal((N, d_in)))
    X = O.widen_bf16(Xb)
    Y = O.w4a16_matmul(Xb, qw, sc, zr, g)
    words = qw.view(np.uint32)
    for t in range(N):
        for o in range(rows):
            acc = 0.0
            for i in range(d_in):
                code = (int(words[o, i // 8]) >> (4 * (i % 8))) & 0xF
                acc += X[t, i] * (code - float(zr[o, i // g])) * float(sc[o, i // g])
            assert Y[t, o] == pytest.approx(acc, rel=1e-12, abs=1e-14)


def test_p5_worked_example_through_the_inference_path():
    """AWQ (scholia-log) §3.1 数值例子, run the way a deployed layer runs it:
    symmetric INT4 group with w_max = 1 and w_i = 0.05 (x_i = 10). Unscaled, the
    code of w_i is 0 and the output error is -0.5; with s_i = 4 folded into the
    activation (x' = 2.5) and the stored fp16 step, the output error is the
    printed -0.143."""
    ex = GOLD["int4_group_example"]
    d_in = 8
    W = np.zeros((1, d_in))
    W[0, 0], W[0, 1] = ex["w_max"], ex["w_i"]
    Wb = gen.f64_to_bf16_bits(W)
    x = np.zeros((1, d_in))
    x[0, 1] = ex["x_i"]
    xb = gen.f64_to_bf16_bits(x)
    y_true = float((O.widen_bf16(xb) @ O.widen_bf16(Wb).T)[0, 0])
    for s_i, code, dy, tol in ((1.0, ex["unscaled_code"], ex["unscaled_dy"], 1e-3),
                               (ex["s_i"], ex["scaled_code"], ex["scaled_dy_printed"], 5e-4)):
        s = np.ones(d_in, dtype=np.float32)
        s[1] = s_i
        qw, sc, zr, codes, _, _ = O.pack(Wb, s.astype(np.float64), ex["bits"], d_in, True)
        assert codes[0, 1] - zr[0, 0] == code
        assert float(sc[0, 0]) == pytest.approx(ex["delta_printed"], abs=5e-4)
        xp = O.fold_inv_scales(xb.T, s).T  # the producer of x carries 1/s
        assert O.widen_bf16(xp)[0, 1] == pytest.approx(ex["x_i"] / s_i)
        y = float(O.w4a16_matmul(xp, qw, sc, zr, d_in)[0, 0])
        assert y - y_true == pytest.approx(dy, abs=tol)


def test_f16_rounding_and_fold_match_torch():
    """float32 -> fp16 round to nearest even equals torch's conversion, and the
    fp16 fold equals torch's float32 division rounded to fp16."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(36)
    x = (rng.standard_normal(20000) * np.exp(rng.standard_normal(20000) * 3)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.to_f16_bits(x), ref)
    p = O.to_f16_bits(rng.standard_normal((48, 16)).astype(np.float32))
    s = np.exp(rng.standard_normal(48)).astype(np.float32)
    want = (torch.from_numpy(O.widen_f16(p).astype(np.float32)) / torch.from_numpy(s)[:, None]).to(torch.float16)
    assert np.array_equal(O.fold_inv_scales(p, s, "f16"), want.view(torch.int16).numpy().view(np.uint16))


def test_w4a16_f16_activations_brute_force():
    """The fp16-activation product (the pages' FP16 inference) equals a
    triple loop over fp16 inputs and the stored codes."""
    rng = np.random.default_rng(37)
    rows, d_in, g, N = 3, 32, 16, 2
    Wb = gen.f64_to_bf16_bits(rng.standard_normal((rows, d_in)) * 0.1)
    qw, sc, zr, _, _, _ = O.pack(Wb, np.ones(d_in), 4, g, True)
    Xh = O.to_f16_bits(rng.standard_normal((N, d_in)).astype(np.float32))
    Y = O.w4a16_matmul(Xh, qw, sc, zr, g, "f16")
    X = Xh.view(np.float16).astype(np.float64)
    words = qw.view(np.uint32)
    for t in range(N):
        for o in range(rows):
            acc = sum(X[t, i] * (((int(words[o, i // 8]) >> (4 * (i % 8))) & 0xF) - float(zr[o, i // g]))
                      * float(sc[o, i // g]) for i in range(d_in))
            assert Y[t, o] == pytest.approx(acc, rel=1e-12, abs=1e-14)


# ---------------------------------------------------------------------------
# per-tensor quantisation (group = 0)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("symmetric,bits", [(True, 4), (False, 4), (True, 3), (False, 2)])
def test_per_tensor_quantiser_brute_force(symmetric, bits):
    """group = 0: one step for the whole matrix ([P1] 量化基础 for the
    symmetric case), checked element by element against the textbook formula
    written with Python scalars."""
    rng = np.random.default_rng(50 + bits)
    V = rng.standard_normal((3, 16)) * np.linspace(0.2, 2.0, 16)
    Vh, codes, delta, zero = O.quantize_groups(V, bits, 0, symmetric)
    assert delta.shape == (1, 1) and zero.shape == (1, 1)
    flat = [float(x) for x in V.ravel()]
    if symmetric:
        qmax = 2 ** (bits - 1) - 1
        d = max(abs(x) for x in flat) / qmax
        for x, vh, c in zip(flat, Vh.ravel(), codes.ravel()):
            q = min(max(round(x / d), -qmax - 1), qmax)   # Python round: half to even
            assert vh == pytest.approx(q * d, rel=1e-15, abs=1e-15)
            assert c == q + qmax + 1
    else:
        levels = 2 ** bits - 1
        d = (max(flat) - min(flat)) / levels
        z = min(max(round(-min(flat) / d), 0), levels)
        for x, vh, c in zip(flat, Vh.ravel(), codes.ravel()):
            q = min(max(round(x / d) + z, 0), levels)
            assert vh == pytest.approx((q - z) * d, rel=1e-15, abs=1e-15)
            assert c == q


def test_per_tensor_worked_example():
    """AWQ (scholia-log) §3.1: w_max = 1 anywhere in the tensor gives the INT4
    step 1/7, and w_i = 0.05 rounds to 0 (output error -0.5 with x_i = 10)."""
    ex = GOLD["int4_group_example"]
    W = np.zeros((2, 8))
    W[1, 3] = ex["w_max"]
    W[0, 1] = ex["w_i"]
    Vh, codes, delta, _ = O.quantize_groups(W, 4, 0, True)
    assert delta[0, 0] == pytest.approx(ex["delta"], rel=1e-15)
    assert Vh[0, 1] == 0.0
    assert (Vh[0, 1] - W[0, 1]) * ex["x_i"] == pytest.approx(ex["unscaled_dy"])


def test_per_tensor_pack_and_search_shapes():
    """The search and the pack take group = 0: one fp16 step / zero for the
    layer; alpha = 0 of the search is plain per-tensor RTN."""
    rng = np.random.default_rng(53)
    Wb = gen.f64_to_bf16_bits(rng.standard_normal((4, 32)) * 0.05)
    Xb = gen.f64_to_bf16_bits(rng.standard_normal((6, 32)))
    a = O.act_stats(Xb)
    res = O.search(Wb, Xb, a, 4, 0, True, 4)
    W = O.widen_bf16(Wb)
    rtn = O.quantize_groups(W, 4, 0, True)[0]
    assert res["losses"][0] == pytest.approx(float(((rtn - W) @ O.widen_bf16(Xb).T) ** 2 @ np.ones(6) @ np.ones(4)),
                                             rel=1e-12)
    qw, sc, zr, codes, delta, zero = O.pack(Wb, res["s_best"], 4, 0, True)
    assert sc.shape == (1, 1) and zr.shape == (1, 1) and qw.shape == (4, 4)
    assert O.boundary_mask(Wb, res["s_best"], 4, 0, True).shape == (4, 32)


# ---------------------------------------------------------------------------
# the rounding-boundary band: which codes a float32 computation may decide
# either way (AWQ (scholia-log) §2.3: Q(w) = Delta round(w / Delta) changes its
# answer only where w / Delta crosses a half-integer)
# ---------------------------------------------------------------------------
BAND = 1e-4
_IN, _OUT = 5e-5, 2e-4   # offsets inside and outside the band


def test_boundary_band_asymmetric_elements():
    """One asymmetric INT4 group of 8 with min 0 and max 1 (Delta = 1/15,
    z = 0, -min/Delta = 0 far from any boundary); the other six elements are
    0.5 * s_i with s_i placing v/Delta at chosen distances from a half-integer
    or an integer. Only those within the band are flagged, and no zero point."""
    targets = [2.5 + _IN, 4.5 - _IN, 6.5 + _OUT, 8.5 - _OUT, 10.5, 12.0 + _IN]
    expect = [False, False, True, True, False, False, True, False]
    W = _bits([[0.0, 1.0] + [0.5] * 6])
    s = np.array([1.0, 1.0] + [2.0 * t / 15.0 for t in targets])
    el, zn = O.boundary_mask(W, s, 4, 8, False, parts=True)
    assert el[0].tolist() == expect
    assert not zn.any()
    assert O.boundary_mask(W, s, 4, 8, False)[0].tolist() == expect
    # the band's width is the argument: widened past 2e-4, the outer pair joins
    wide = O.boundary_mask(W, s, 4, 8, False, band=3e-4)[0]
    assert wide.tolist() == [False, False, True, True, True, True, True, False]


def test_boundary_band_symmetric_negative_side():
    """Symmetric INT4, max |v| = 1 so Delta = 1/7 (AWQ (scholia-log) §3.1):
    negative values at v/Delta = -(k + 1/2 +- e) are flagged inside the band
    only (the fractional part is taken from below, floor, not by rounding);
    the symmetric zero point is fixed and never flags a group."""
    targets = [1.5 + _IN, 2.5 - _IN, 3.5 + _OUT, 4.5 - _OUT, 5.5, 3.0 - _IN, 0.5 + _IN]
    expect = [False, True, True, False, False, True, False, True]
    W = _bits([[1.0] + [-0.5] * 7])
    s = np.array([1.0] + [2.0 * t / 7.0 for t in targets])
    el, zn = O.boundary_mask(W, s, 4, 8, True, parts=True)
    assert el[0].tolist() == expect
    assert not zn.any()


def test_boundary_band_zero_point_flags_the_whole_group():
    """Asymmetric INT4, two groups of 8 in one row. Group A: v = (-m, 1, 0 ...)
    with m chosen so that -min/Delta = 15 m / (1 + m) = 3.5 + e, so z sits at a
    rounding boundary; group B is an ordinary group. Inside the band the whole
    of group A is flagged (every code depends on z) and nothing of group B;
    outside the band nothing is flagged at all."""
    for e, flagged in ((_IN, True), (-_IN, True), (_OUT, False), (-_OUT, False)):
        c = 3.5 + e
        m = c / (15.0 - c)
        W = _bits([[-0.5, 1.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0,
                    0.25, -0.75, 0.5, 0.125, 1.0, -1.0, 0.0, 0.375]])
        s = np.ones(16)
        s[0] = 2.0 * m
        s[8:] = [1.0, 1.0, 1.1, 0.9, 1.0, 0.8, 1.0, 1.3]   # group B: -min/Delta = 15*0.8/1.8 = 6.67
        el, zn = O.boundary_mask(W, s, 4, 8, False, parts=True)
        assert zn[0].tolist() == [flagged, False]
        mask = O.boundary_mask(W, s, 4, 8, False)[0]
        assert mask[:8].all() == flagged and mask[:8].any() == flagged
        assert not mask[8:].any()
        # the group's extremes sit at c and 15 - c on the grid: flagged with z
        assert el[0, 0] == flagged and el[0, 1] == flagged and not el[0, 2:8].any()


def test_boundary_band_per_tensor():
    """group = 0: the layer is one group. Symmetric: Delta = 1/7 from the
    layer's max wherever it sits; elements flagged as in a group. Asymmetric:
    a zero point at a boundary flags every element of the layer."""
    targets = [1.5 + _IN, 2.5 + _OUT, 3.5 - _IN]
    W = _bits([[1.0, -0.5, -0.5, -0.5], [0.0, 0.0, 0.0, 0.0]])
    s = np.array([1.0] + [2.0 * t / 7.0 for t in targets])
    el, zn = O.boundary_mask(W, s, 4, 0, True, parts=True)
    assert el.tolist() == [[False, True, False, True], [False] * 4]
    assert zn.shape == (1, 1) and not zn.any()
    for e, flagged in ((_IN, True), (_OUT, False)):
        c = 3.5 + e
        m = c / (15.0 - c)
        Wa = _bits([[-0.5, 1.0, 0.0, 0.0], [0.0, 0.0, 0.0, 0.0]])
        sa = np.array([2.0 * m, 1.0, 1.0, 1.0])
        mask = O.boundary_mask(Wa, sa, 4, 0, False)
        assert mask.all() == flagged and mask.any() == flagged


def test_boundary_band_clip_uses_the_clipped_step():
    """With clip ratio c the step comes from the shrunk range (max|v| -> c
    max|v|): at c = 1/2, Delta = 1/14, so v = (2.5 + e)/14 is flagged and the
    same v is not flagged at c = 1 (v/Delta = 1.25)."""
    W = _bits([[1.0, 0.5, 0.0, 0.0]])
    s = np.array([1.0, 2.0 * (2.5 + _IN) / 14.0, 1.0, 1.0])
    assert O.boundary_mask(W, s, 4, 4, True, clip=0.5)[0].tolist() == [False, True, False, False]
    assert not O.boundary_mask(W, s, 4, 4, True)[0].any()


@pytest.mark.parametrize("bits,sym", [(4, False), (4, True), (3, True), (2, False)])
def test_boundary_band_covers_every_float32_disagreement(bits, sym):
    """Outside the band a float32 evaluation of the same quantiser (products,
    step and 1/Delta in float32, round to nearest even) takes every code and
    zero point the float64 oracle takes: the band is wide enough. Inside the
    band the excluded fraction stays near its expectation 2 * band per
    element (and per group for the zero point)."""
    rng = np.random.default_rng(100 + bits + 10 * sym)
    rows, d_in, g = 512, 1024, 64
    Wb = gen.f64_to_bf16_bits(rng.standard_normal((rows, d_in)) * 0.02)
    s = np.exp(rng.standard_normal(d_in))
    codes64 = O.pack(Wb, s, bits, g, sym)[3]
    el, zn = O.boundary_mask(Wb, s, bits, g, sym, parts=True)
    # float32 restatement of the quantiser, written here for this check only
    v = (O.widen_bf16(Wb).astype(np.float32) * s.astype(np.float32)).reshape(rows, -1, g)
    if sym:
        qmax = np.float32(2 ** (bits - 1) - 1)
        d = np.abs(v).max(-1) / qmax
        q = np.clip(np.rint(v * (np.float32(1) / d)[..., None]), -qmax - 1, qmax) + qmax + 1
    else:
        lv = np.float32(2 ** bits - 1)
        mx, mn = v.max(-1), v.min(-1)
        d = (mx - mn) / lv
        inv = np.float32(1) / d
        z = np.clip(np.rint(-mn * inv), 0, lv)
        q = np.clip(np.rint(v * inv[..., None]) + z[..., None], 0, lv)
    q = q.reshape(rows, d_in).astype(np.int64)
    mask = el | np.repeat(zn, g, axis=1)
    assert np.array_equal(q[~mask], codes64[~mask])
    assert el.mean() <= 2 * BAND * 2
    assert zn.mean() <= 2 * BAND * 5 + 1.0 / zn.size
