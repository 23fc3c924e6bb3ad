"""Per-group clipping search (awq_search_group_clip) and the pack with a clip
ratio per group, against the oracle's group_clip_errors / group_clip_choice.

Both sides get the same fp32 scales (the oracle's a^0.5 candidate, rounded to
fp32). Tolerance of a group error: the GPU rounds dW and the diagonal blocks
of G to bf16 (8-bit significand, unit roundoff u = 2^-8 each) and accumulates
in fp32, so to first order |err_gpu - err| <= (2 + 1) u sum_ik |dW_i| |G_ik|
|dW_k| (the same form with absolute values); the test allows 1.1 times that
(second-order and fp32 accumulation terms are far below the 10%). Groups holding an
element within the oracle's boundary band for a clip ratio are left out for
that ratio (a rounding flip changes their dW by a whole step), and the chosen
ratio is accepted when its oracle error is within both tolerances of the
oracle's minimum."""
import numpy as np
import pytest

from awq_inputs import WORKLOADS, custom, make_inputs
from oracle import awq_oracle as O

from gpu_util import to_device, unpack_words

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import weight_only_int4_act_b200 as awq  # noqa: E402

CLIPS = [1.0, 0.95, 0.9, 0.85, 0.8, 0.75, 0.7, 0.6, 0.5]
FORM_TOL = 1.1 * 3 * 2.0 ** -8

CASES = [
    ("C1", WORKLOADS["C1"]),
    ("ragged_d_in_384", custom(200, 384, 300, seed=3)),          # last 256-block half full
    ("sym3_g64", custom(130, 512, 300, bits=3, symmetric=True, group=64, seed=4)),
    ("g32_d_in_320", custom(128, 320, 200, group=32, seed=5)),   # 32-wide groups, ragged block
    ("g256", custom(96, 768, 256, group=256, seed=6)),
]


def _oracle_tables(Wb, Xb, s64, wl):
    """Oracle errors, the absolute-value form per (clip, row, group), and the
    near-boundary mask per (clip, row, group)."""
    err = O.group_clip_errors(Wb, Xb, s64, wl.bits, wl.group, wl.symmetric, CLIPS)
    W = O.widen_bf16(Wb)
    G = O.gram(Xb)
    ng = wl.d_in // wl.group
    form = np.zeros_like(err)
    near = np.zeros(err.shape, dtype=bool)
    for ci, c in enumerate(CLIPS):
        dW = np.abs(O.delta_weight(W, s64, wl.bits, wl.group, wl.symmetric, c))
        for j in range(ng):
            sl = slice(j * wl.group, (j + 1) * wl.group)
            form[ci, :, j] = np.einsum("ri,ri->r", dW[:, sl] @ np.abs(G[sl, sl]), dW[:, sl])
        m = O.boundary_mask(Wb, s64, wl.bits, wl.group, wl.symmetric, clip=c)
        near[ci] = m.reshape(wl.d_out, ng, wl.group).any(axis=-1)
    return err, form, near


@pytest.mark.parametrize("name,wl", CASES)
def test_group_clip_search_and_pack(name, wl):
    Wb, Xb = make_inputs(wl)
    W, X = to_device(Wb), to_device(Xb)
    s32 = O.candidate_scales(O.act_stats(Xb), 0.5).astype(np.float32)
    s64 = s32.astype(np.float64)
    cfg = awq.make_cfg(wl.bits, wl.group, wl.symmetric, len(CLIPS))
    s_dev = torch.from_numpy(s32).cuda()
    res = awq.search_group_clip(W, X, s_dev, CLIPS, cfg, group_err=True)
    torch.cuda.synchronize()
    awq.workspace_error(res["ws"])
    err_gpu = res["group_err"].cpu().numpy().astype(np.float64)
    best_gpu = res["best_clip"].cpu().numpy().astype(np.int64)

    err, form, near = _oracle_tables(Wb, Xb, s64, wl)
    tol = FORM_TOL * form + 1e-30
    ok = ~near
    assert ok.mean() > 0.8, f"too few groups away from a rounding boundary: {ok.mean()}"
    bad = (np.abs(err_gpu - err) > tol) & ok
    assert not bad.any(), (name, np.argwhere(bad)[:5], err_gpu[bad][:5], err[bad][:5])

    # the chosen ratio: exact argmin where the candidates are far apart, else
    # within the two tolerances of the oracle's minimum
    ng = wl.d_in // wl.group
    rows, cols = np.meshgrid(np.arange(wl.d_out), np.arange(ng), indexing="ij")
    clean = ok.all(axis=0)
    best_ref = O.group_clip_choice(err)
    e_gpu_choice = err[best_gpu, rows, cols]
    e_min = err[best_ref, rows, cols]
    slack = tol[best_gpu, rows, cols] + tol[best_ref, rows, cols]
    wrong = clean & (e_gpu_choice > e_min + slack)
    assert not wrong.any(), (name, np.argwhere(wrong)[:5])
    assert (best_gpu < len(CLIPS)).all()
    agree = (best_gpu == best_ref)[clean].mean()
    assert agree > 0.9, agree

    # pack with the GPU's per-group choice; the oracle packs with the same ratios
    q, sc, zr = awq.quantize_pack_group_clip(W, s_dev, CLIPS, res["best_clip"], cfg)
    torch.cuda.synchronize()
    clip_arr = np.asarray(CLIPS)[best_gpu]
    _, sc_ref, zr_ref, codes_ref, _, _ = O.pack(Wb, s64, wl.bits, wl.group, wl.symmetric, clip=clip_arr)
    nearp = O.boundary_mask(Wb, s64, wl.bits, wl.group, wl.symmetric, clip=clip_arr)
    codes = unpack_words(q, wl.d_in)
    assert not ((codes != codes_ref) & ~nearp).any()
    sc_g = sc.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(sc_g - sc_ref.astype(np.float64)) <= 2.0 ** -10 * np.abs(sc_ref.astype(np.float64)))
    gnear = nearp.reshape(wl.d_out, ng, wl.group).any(axis=-1)
    assert not ((zr.cpu().numpy() != zr_ref) & ~gnear).any()
    print(name, "groups checked", ok.mean(), "choice agreement", agree,
          "ratio histogram", np.bincount(best_gpu.ravel(), minlength=len(CLIPS)))


def test_group_clip_single_ratio_is_plain_pack():
    """One candidate ratio 1.0: every group takes index 0, and the pack equals
    the unclipped pack bit for bit."""
    wl = custom(128, 512, 128, seed=7)
    Wb, Xb = make_inputs(wl)
    W, X = to_device(Wb), to_device(Xb)
    s = torch.from_numpy(O.candidate_scales(O.act_stats(Xb), 0.3).astype(np.float32)).cuda()
    cfg = awq.make_cfg(4, 128, False, 1)
    res = awq.search_group_clip(W, X, s, [1.0], cfg)
    torch.cuda.synchronize()
    awq.workspace_error(res["ws"])
    assert (res["best_clip"] == 0).all()
    a = awq.quantize_pack_group_clip(W, s, [1.0], res["best_clip"], cfg)
    b = awq.quantize_pack(W, s, cfg)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_group_clip_nonpositive_scale_flagged():
    wl = custom(64, 256, 64, seed=8)
    Wb, Xb = make_inputs(wl)
    W, X = to_device(Wb), to_device(Xb)
    s = torch.ones(256, dtype=torch.float32, device="cuda")
    s[3] = 0.0
    res = awq.search_group_clip(W, X, s, [1.0, 0.8], awq.make_cfg(4, 128, False, 2))
    torch.cuda.synchronize()
    with pytest.raises(awq.AwqError, match="NONFINITE"):
        awq.workspace_error(res["ws"])
