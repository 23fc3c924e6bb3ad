"""Parity of the CUDA path with the CPU oracle, element by element on seeded
inputs, through the C ABI (Python binding).

Tolerances (stated by the benchmark spec for this path):
  * a_i within 1e-5 relative;
  * every candidate loss within 1e-2 relative;
  * the chosen alpha equal, unless the oracle's best losses are within 0.5%
    (then any of those is accepted);
  * packed codes bit-exact except where the oracle's v/Delta (or -min/Delta
    for the zero point) lies within 1e-4 of a rounding boundary; those
    exceptions are counted and reported.
"""
import numpy as np
import pytest

from awq_inputs import WORKLOADS, custom, make_inputs
from oracle import awq_oracle as O

from gpu_util import to_device, unpack_words, bf16_to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU machines, skipped there
    pytest.skip("needs a CUDA device", allow_module_level=True)

import weight_only_int4_act_b200 as awq  # noqa: E402

A_RTOL = 1e-5
LOSS_RTOL = 1e-2
TIE_REL = 0.005


def check_stats(Xb, a_gpu):
    a_ref = O.act_stats(Xb)
    a = a_gpu.cpu().numpy().astype(np.float64)
    rel = np.abs(a - a_ref) / np.maximum(np.abs(a_ref), 1e-30)
    assert rel.max() <= A_RTOL, f"a_i max rel err {rel.max():.3g}"
    return a_ref


EXCLUDE_FRAC = 1e-3  # bound on the fraction of codes (and of groups) left out near a rounding boundary


def check_exclusions(el, zn):
    """The band of rounding boundaries excludes about 2e-4 of the elements (and
    of the groups, for their zero point) at random; bound each part by 1e-3,
    plus a count of 3 elements / 1 group so that tiny layers, where a single
    flagged group is already more than 1e-3 of them, do not fail by chance."""
    n_el, n_g = int(el.sum()), int(zn.sum())
    assert n_el <= EXCLUDE_FRAC * el.size + 3, f"{n_el} of {el.size} codes excluded"
    assert n_g <= EXCLUDE_FRAC * zn.size + 1, f"{n_g} of {zn.size} zero points excluded"
    return n_el, n_g


def check_pack(Wb, s_ref, q, sc, zr, bits, g, sym):
    d_out, d_in = Wb.shape
    qw, sc_ref, zr_ref, codes_ref, delta_ref, zero_ref = O.pack(Wb, s_ref, bits, g, sym)
    codes = unpack_words(q, d_in)
    el, zn = O.boundary_mask(Wb, s_ref, bits, g, sym, parts=True)
    near = el | np.repeat(zn, g, axis=1)
    bad = (codes != codes_ref) & ~near
    assert not bad.any(), f"{bad.sum()} codes differ away from rounding boundaries"
    check_exclusions(el, zn)
    sc_g = sc.cpu().numpy().astype(np.float64)
    zr_g = zr.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(sc_g - sc_ref.astype(np.float64)) <= 2.0 ** -10 * np.abs(sc_ref.astype(np.float64)) + 1e-12)
    zbad = (zr_g != zr_ref.astype(np.float64)) & ~zn
    assert not zbad.any(), f"{zbad.sum()} zero points differ"
    return int((codes != codes_ref).sum()), int(near.sum())


def check_row_losses(Wb, Xb, a_ref, wl, rows, rl_gpu):
    """Per-row losses of the given rows against the oracle. A row holding an
    element whose code the oracle decides within 1e-4 of a rounding boundary
    may legitimately differ by more (one flipped code moves its row's loss by
    up to a few percent); such rows are counted and left to the total-loss
    check."""
    sub = O.search(Wb, Xb, a_ref, wl.bits, wl.group, wl.symmetric, wl.n_alpha, rows=rows)
    ref = sub["row_losses"]
    got = rl_gpu[:, rows]
    tol = LOSS_RTOL * ref + 1e-3 * ref.mean()
    ok = np.abs(got - ref) <= tol
    near = np.stack([O.boundary_mask(Wb[rows], O.candidate_scales(a_ref, al), wl.bits, wl.group,
                                     wl.symmetric).any(axis=1) for al in O.alpha_grid(wl.n_alpha)])
    bad = ~ok & ~near
    assert not bad.any(), f"{bad.sum()} (alpha, row) losses differ away from rounding boundaries"
    return int((~ok).sum()), int(near.sum())


def run_case(wl, form="auto", check_rows=True):
    Wb, Xb = make_inputs(wl)
    W, X = to_device(Wb), to_device(Xb)
    cfg = awq.make_cfg(wl.bits, wl.group, wl.symmetric, wl.n_alpha, form=form)
    a = awq.act_stats(X)
    res = awq.search_scales(W, X, a, cfg, row_losses=True)
    q, sc, zr = awq.quantize_pack(W, res["s_best"], cfg)
    torch.cuda.synchronize()
    awq.workspace_error(res["ws"])

    a_ref = check_stats(Xb, a)
    ref = O.search(Wb, Xb, a_ref, wl.bits, wl.group, wl.symmetric, wl.n_alpha,
                   form="gram" if wl.d_in < wl.N else "direct")
    losses = res["losses"].cpu().numpy().astype(np.float64)
    rel = np.abs(losses - ref["losses"]) / ref["losses"]
    assert rel.max() <= LOSS_RTOL, f"loss max rel err {rel.max():.3g}"
    rl = res["row_losses"].cpu().numpy().astype(np.float64)
    assert np.allclose(rl.sum(axis=1), losses, rtol=1e-5)
    if check_rows:
        check_row_losses(Wb, Xb, a_ref, wl, np.arange(wl.d_out), rl)
    best = int(res["best"].item())
    assert best in O.acceptable_choices(ref["losses"], TIE_REL), (best, ref["best"], ref["losses"])
    s_ref = O.candidate_scales(a_ref, O.alpha_grid(wl.n_alpha)[best])
    s_gpu = res["s_best"].cpu().numpy().astype(np.float64)
    assert np.allclose(s_gpu, s_ref, rtol=1e-5)
    flips, near = check_pack(Wb, s_ref, q, sc, zr, wl.bits, wl.group, wl.symmetric)
    return dict(rel=rel.max(), flips=flips, near=near, best=best)


SMALL = {
    "C1": WORKLOADS["C1"],
    "ragged_200x384_N300": custom(200, 384, 300, seed=3),
    "sym3_g64_130x512_N77": custom(130, 512, 77, bits=3, symmetric=True, group=64, seed=4),
    "asym2_g32_64x256_N1000_silu": custom(64, 256, 1000, bits=2, group=32, x_kind="absnormal",
                                          x_lognormal_sigma=None, seed=5),
    "g16_33x128_N9": custom(33, 128, 9, group=16, seed=6),
    "g256_300x1024_N520": custom(300, 1024, 520, group=256, seed=8),
    "g8_sym4_40x64_N1": custom(40, 64, 1, bits=4, symmetric=True, group=8, seed=9),
    "tokens_gt_din_129x256_N2000": custom(129, 256, 2000, seed=10),
    # G' of 91 tiles on 74 CTA pairs: the last wave's 17 tiles run as 4 K pieces each
    "gram_tail_64x3328_N512": custom(64, 3328, 512, seed=14),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_search_small_auto(name):
    out = run_case(SMALL[name])
    print(name, out)


@pytest.mark.parametrize("name", ["C1", "ragged_200x384_N300", "sym3_g64_130x512_N77", "g256_300x1024_N520",
                                  "gram_tail_64x3328_N512"])
@pytest.mark.parametrize("form", ["direct", "gram"])
def test_search_small_forced_form(name, form):
    run_case(SMALL[name], form=form, check_rows=False)


def test_gram_tail_pieces_match_direct_form():
    """The Gram form with its last wave split in K (the pieces' fp32 partials
    summed by the fix-up) gives the direct form's losses, row by row, to the
    bf16 rounding of G'."""
    wl = SMALL["gram_tail_64x3328_N512"]
    Wb, Xb = make_inputs(wl)
    W, X = to_device(Wb), to_device(Xb)
    a = awq.act_stats(X)
    rows = {}
    for form in ("direct", "gram"):
        cfg = awq.make_cfg(wl.bits, wl.group, wl.symmetric, wl.n_alpha, form=form)
        res = awq.search_scales(W, X, a, cfg, row_losses=True)
        torch.cuda.synchronize()
        awq.workspace_error(res["ws"])
        rows[form] = res["row_losses"].cpu().numpy().astype(np.float64)
    rel = np.abs(rows["gram"] - rows["direct"]) / np.abs(rows["direct"])
    assert rel.max() < LOSS_RTOL, rel.max()


def test_delta_weight_stack_elementwise():
    """The bf16 dW stack the contraction reads equals the oracle's
    Q(WS)S^-1 - W to bf16 rounding, except at rounding boundaries."""
    wl = custom(200, 384, 300, seed=3)
    Wb, Xb = make_inputs(wl)
    W, X = to_device(Wb), to_device(Xb)
    cfg = awq.make_cfg(4, 128, False, 20)
    a = awq.act_stats(X)
    res = awq.search_scales(W, X, a, cfg)
    a_ref = O.act_stats(Xb)
    Wf = O.widen_bf16(Wb)
    for k in (0, 7, 19):
        s = O.candidate_scales(a_ref, O.alpha_grid(20)[k])
        ref = O.delta_weight(Wf, s, 4, 128, False)
        got = bf16_to_f64(awq.debug_dw(res["ws"], 200, 384, 300, cfg, k))
        near = O.boundary_mask(Wb, s, 4, 128, False)
        tol = 2.0 ** -8 * np.abs(ref) + 4e-6 * np.abs(Wf) + 1e-30
        bad = (np.abs(got - ref) > tol) & ~near
        assert not bad.any(), f"alpha {k}: {bad.sum()} dW elements differ"


def test_determinism_bitwise():
    wl = SMALL["ragged_200x384_N300"]
    Wb, Xb = make_inputs(wl)
    W, X = to_device(Wb), to_device(Xb)
    cfg = awq.make_cfg(4, 128, False, 20)
    outs = []
    for _ in range(2):
        a = awq.act_stats(X)
        r = awq.search_scales(W, X, a, cfg, row_losses=True)
        outs.append((a.cpu().numpy(), r["losses"].cpu().numpy(), r["row_losses"].cpu().numpy()))
    for x, y in zip(outs[0], outs[1]):
        assert np.array_equal(x, y)


def test_nonfinite_activation_reported():
    wl = custom(64, 256, 32, seed=12)
    Wb, Xb = make_inputs(wl)
    Xb = Xb.copy()
    Xb[3, 17] = 0x7FC0  # NaN planted on the host
    W, X = to_device(Wb), to_device(Xb)
    cfg = awq.make_cfg(4, 128, False, 20)
    a = awq.act_stats(X)
    res = awq.search_scales(W, X, a, cfg)
    torch.cuda.synchronize()
    assert int(res["best"].item()) == -1
    with pytest.raises(awq.AwqError, match="NONFINITE"):
        awq.workspace_error(res["ws"])
    awq.workspace_error(res["ws"])  # cleared by the read-back


def test_dead_channel_and_zero_rows():
    """A channel with no activation (a_i = 0) and all-zero weight rows."""
    wl = custom(128, 256, 64, seed=13)
    Wb, Xb = make_inputs(wl)
    Wb = Wb.copy()
    Xb = Xb.copy()
    Xb[:, 5] = 0
    Wb[7] = 0
    out = run_case_arrays(Wb, Xb, wl)
    assert out["zero_row_loss"] == 0.0


def run_case_arrays(Wb, Xb, wl):
    W, X = to_device(Wb), to_device(Xb)
    cfg = awq.make_cfg(wl.bits, wl.group, wl.symmetric, wl.n_alpha)
    a = awq.act_stats(X)
    res = awq.search_scales(W, X, a, cfg, row_losses=True)
    q, sc, zr = awq.quantize_pack(W, res["s_best"], cfg)
    torch.cuda.synchronize()
    awq.workspace_error(res["ws"])
    a_ref = check_stats(Xb, a)
    ref = O.search(Wb, Xb, a_ref, wl.bits, wl.group, wl.symmetric, wl.n_alpha)
    losses = res["losses"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(losses - ref["losses"]) <= LOSS_RTOL * ref["losses"])
    best = int(res["best"].item())
    assert best in O.acceptable_choices(ref["losses"], TIE_REL)
    s_ref = O.candidate_scales(a_ref, O.alpha_grid(wl.n_alpha)[best])
    check_pack(Wb, s_ref, q, sc, zr, wl.bits, wl.group, wl.symmetric)
    return dict(zero_row_loss=float(res["row_losses"][:, 7].abs().max().item()))


def test_gpu_rejects_bad_arguments():
    X = torch.zeros((16, 500), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(awq.AwqError, match="SHAPE"):
        awq.act_stats(X)
    W = torch.zeros((64, 256), dtype=torch.bfloat16, device="cuda")
    X = torch.zeros((16, 256), dtype=torch.bfloat16, device="cuda")
    a = torch.ones(256, dtype=torch.float32, device="cuda")
    small_ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(awq.AwqError, match="WORKSPACE"):
        awq.search_scales(W, X, a, awq.make_cfg(4, 128, False, 20), ws=small_ws)
    with pytest.raises(awq.AwqError, match="INVALID_ARG"):
        awq.search_scales(W, X, a, awq.make_cfg(5, 128, False, 20))


def test_bounded_wait_gives_up_and_context_survives():
    """A wait that nothing satisfies ends after the wall-clock limit with an
    error in the workspace (no trap, no hang), and the context keeps working."""
    import time
    ws = awq.workspace(256)
    t0 = time.perf_counter()
    awq.selftest_bounded_wait(ws)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert 1.0 < waited < 30.0, waited
    with pytest.raises(awq.AwqError, match="DEVICE"):
        awq.workspace_error(ws)
    awq.workspace_error(ws)  # the read cleared the word
    run_case(SMALL["C1"], check_rows=False)
