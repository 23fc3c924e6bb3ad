"""The debug build with index checks (-DAWQ_BOUNDS_CHECK) on the GPU.

- Its failure path: a store the check refuses is recorded with its site,
  read back and cleared by awq_bounds_error, and the context stays usable.
- The whole path through it (statistics, both forms of the search, the
  segmented, per-tensor and per-group-clip searches, the packs, the fold and
  the W4A16 product with and without split-K) gives results identical to the
  release build, and no check fires.

The rest of the GPU suite runs on whichever build AWQ_B200_LIB selects;
conftest.py fails any GPU test during which a check of that build fired."""
import numpy as np
import pytest

from awq_inputs import custom, make_inputs
from oracle import awq_oracle as O

from gpu_util import to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import weight_only_int4_act_b200 as awq  # noqa: E402

CLIPS = [1.0, 0.95, 0.9, 0.85]


class _using:
    """Route the binding's calls to one build for the duration of a block."""

    def __init__(self, variant):
        self.variant = variant

    def __enter__(self):
        self.prev = awq.select_library(self.variant)

    def __exit__(self, *exc):
        awq.select_library(self.prev)


def test_release_build_has_no_checks_and_no_selftest():
    with _using("release"):
        assert not awq.bounds_checks_enabled()
        with pytest.raises(awq.AwqError, match="UNSUPPORTED"):
            awq.selftest_bounds(awq.workspace(256))
        assert awq.bounds_error() == (0, 0)


def test_refused_store_is_recorded_and_cleared():
    with _using("check"):
        assert awq.bounds_checks_enabled()
        assert awq.bounds_error() == (0, 0)
        ws = awq.workspace(256)
        ws.zero_()
        awq.selftest_bounds(ws)
        assert awq.bounds_error() == (awq.AWQ_ERR_BOUNDS, 0x7F)
        assert awq.bounds_error() == (0, 0)  # reading cleared it
        assert int(ws.view(torch.int32)[63]) == 0  # the refused store did not happen
        # the context is still usable
        wl = custom(64, 256, 100, seed=5)
        _, Xb = make_inputs(wl)
        a = awq.act_stats(to_device(Xb))
        torch.cuda.synchronize()
        assert np.allclose(a.cpu().numpy(), O.act_stats(Xb), rtol=1e-5, atol=0)
        assert awq.bounds_error() == (0, 0)


def _chain():
    """Every kernel of the library once, on small ragged shapes; the outputs
    as host arrays."""
    out = {}
    wl = custom(200, 384, 300, seed=3)
    Wb, Xb = make_inputs(wl)
    W, X = to_device(Wb), to_device(Xb)
    a = awq.act_stats(X)
    out["a"] = a
    for form in ("gram", "direct"):
        cfg = awq.make_cfg(4, 128, False, 20, form=form)
        r = awq.search_scales(W, X, a, cfg, row_losses=True)
        awq.workspace_error(r["ws"])
        for k in ("losses", "best", "s_best", "row_losses"):
            out[f"{form}_{k}"] = r[k]
    cfg = awq.make_cfg(4, 128, False, 20)
    seg = awq.search_scales_segmented(W, X, a, cfg, [72, 128], row_losses=True)
    awq.workspace_error(seg["ws"])
    for k in ("losses", "best", "s_best", "row_losses"):
        out[f"seg_{k}"] = seg[k]
    s = out["gram_s_best"]
    out["q"], out["sc"], out["zr"] = awq.quantize_pack(W, s, cfg)
    # per tensor
    cfg0 = awq.make_cfg(4, 0, False, 8)
    r0 = awq.search_scales(W, X, a, cfg0)
    awq.workspace_error(r0["ws"])
    out["pt_losses"], out["pt_best"] = r0["losses"], r0["best"]
    out["pt_q"], out["pt_sc"], out["pt_zr"] = awq.quantize_pack(W, r0["s_best"], cfg0)
    # per-group clipping
    cfgc = awq.make_cfg(3, 64, False, len(CLIPS))
    gc = awq.search_group_clip(W, X, s, CLIPS, cfgc, group_err=True)
    awq.workspace_error(gc["ws"])
    out["gc_best"], out["gc_err"] = gc["best_clip"], gc["group_err"]
    out["gc_q"], out["gc_sc"], out["gc_zr"] = awq.quantize_pack_group_clip(W, s, CLIPS, gc["best_clip"], cfgc)
    # fold (8 per thread, and one per thread) and the W4A16 product without split-K
    Xt = X.t().contiguous()
    awq.fold_inv_scales(s, Xt)
    Xp = Xt.t().contiguous()
    out["Xp"] = Xp
    v = X[0].clone()
    awq.fold_inv_scales(s, v)
    out["fold_vec"] = v
    out["Y"] = awq.w4a16_gemm(Xp, out["q"], out["sc"], out["zr"], cfg)
    # decode width on a deeper layer: the product splits K across CTAs
    wl2 = custom(256, 4096, 16, seed=9)
    W2b, X2b = make_inputs(wl2)
    W2, X2 = to_device(W2b), to_device(X2b)
    s2 = torch.ones(4096, dtype=torch.float32, device="cuda")
    q2, sc2, zr2 = awq.quantize_pack(W2, s2, cfg)
    ws2 = awq.workspace(awq.w4a16_workspace_size(16, 256, 4096, cfg))
    out["Y_split"] = awq.w4a16_gemm(X2, q2, sc2, zr2, cfg, ws=ws2)
    awq.workspace_error(ws2)
    torch.cuda.synchronize()
    return {k: v.cpu() for k, v in out.items() if v is not None}


def test_check_build_matches_release_and_no_check_fires():
    with _using("release"):
        ref = _chain()
    with _using("check"):
        assert awq.bounds_error() == (0, 0)
        got = _chain()
        st, site = awq.bounds_error()
        assert st == 0, f"an index check failed at site {site:#x}"
    assert ref.keys() == got.keys()
    for k in ref:
        # same arithmetic in both builds: compare bit patterns
        a, b = ref[k].contiguous(), got[k].contiguous()
        assert a.shape == b.shape and a.dtype == b.dtype, k
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), f"{k} differs between the builds"
