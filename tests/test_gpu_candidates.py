"""Search over explicit candidates (awq_search_candidates) and the clipped
pack, against the oracle: the clipping search (one scale vector, a grid of
clip ratios) and a salience-mask candidate set. The candidate scales are
built from the oracle's statistics, rounded to fp32, and the same fp32
values are given to both sides."""
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
from test_gpu_parity import LOSS_RTOL, TIE_REL  # noqa: E402

CLIPS = [1.0, 0.95, 0.9, 0.85, 0.8, 0.7, 0.6, 0.5]


def _run(wl, s_cand32, clips):
    Wb, Xb = make_inputs(wl)
    W, X = to_device(Wb), to_device(Xb)
    n = s_cand32.shape[0]
    cfg = awq.make_cfg(wl.bits, wl.group, wl.symmetric, n)
    res = awq.search_candidates(W, X, torch.from_numpy(s_cand32).cuda(), cfg, clips=clips)
    torch.cuda.synchronize()
    awq.workspace_error(res["ws"])
    ref = O.search_candidates(Wb, Xb, s_cand32.astype(np.float64), wl.bits, wl.group, wl.symmetric, clips=clips)
    losses = res["losses"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(losses - ref["losses"]) <= LOSS_RTOL * ref["losses"]), (losses, ref["losses"])
    best = int(res["best"].item())
    assert best in O.acceptable_choices(ref["losses"], TIE_REL)
    assert np.array_equal(res["s_best"].cpu().numpy(), s_cand32[best])
    return Wb, W, cfg, best, ref


@pytest.mark.parametrize("name,wl", [("C1", WORKLOADS["C1"]),
                                     ("sym3_g64", custom(130, 512, 300, bits=3, symmetric=True, group=64, seed=4)),
                                     ("ragged", custom(200, 384, 300, seed=3))])
def test_clip_search_and_clipped_pack(name, wl):
    _, Xb = make_inputs(wl)
    a = O.act_stats(Xb)
    s_star = O.candidate_scales(a, 0.5).astype(np.float32)
    s_cand = np.stack([s_star] * len(CLIPS))
    Wb, W, cfg, best, ref = _run(wl, s_cand, CLIPS)
    s64 = s_star.astype(np.float64)
    for c in sorted({CLIPS[best], 0.8, 0.55}):
        q, sc, zr = awq.quantize_pack(W, torch.from_numpy(s_star).cuda(), cfg, clip=c)
        torch.cuda.synchronize()
        _, sc_ref, zr_ref, codes_ref, _, _ = O.pack(Wb, s64, wl.bits, wl.group, wl.symmetric, clip=c)
        near = O.boundary_mask(Wb, s64, wl.bits, wl.group, wl.symmetric, clip=c)
        codes = unpack_words(q, wl.d_in)
        assert not ((codes != codes_ref) & ~near).any(), c
        sc_g = sc.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(sc_g - sc_ref.astype(np.float64)) <= 2.0 ** -10 * np.abs(sc_ref.astype(np.float64)))
        gnear = near.reshape(wl.d_out, -1, wl.group).any(axis=-1)
        assert not ((zr.cpu().numpy() != zr_ref) & ~gnear).any(), c
    print(name, "best clip", CLIPS[best], "losses", ref["losses"])


def test_salience_mask_candidates():
    """[P1] 显著识别 / Python demo: channels whose importance exceeds the 70th
    percentile get a fixed factor, the rest 1; factors 1..4 as candidates."""
    wl = custom(256, 512, 400, seed=17)
    _, Xb = make_inputs(wl)
    a = O.act_stats(Xb)
    mask = a > np.percentile(a, 70)
    factors = [1.0, 1.5, 2.0, 3.0, 4.0]
    s_cand = np.stack([np.where(mask, f, 1.0) for f in factors]).astype(np.float32)
    _run(wl, s_cand, None)


def test_candidate_validation():
    wl = custom(64, 256, 32, seed=18)
    Wb, Xb = make_inputs(wl)
    W, X = to_device(Wb), to_device(Xb)
    cfg = awq.make_cfg(4, 128, False, 2)
    s = torch.ones((2, 256), dtype=torch.float32, device="cuda")
    with pytest.raises(awq.AwqError, match="INVALID_ARG"):
        awq.search_candidates(W, X, s, cfg, clips=[1.0, 1.5])
    s[1, 7] = -1.0
    res = awq.search_candidates(W, X, s, cfg)
    torch.cuda.synchronize()
    with pytest.raises(awq.AwqError, match="NONFINITE"):
        awq.workspace_error(res["ws"])
    with pytest.raises(awq.AwqError, match="INVALID_ARG"):
        awq.quantize_pack(W, torch.ones(256, dtype=torch.float32, device="cuda"), cfg, clip=0.0)
