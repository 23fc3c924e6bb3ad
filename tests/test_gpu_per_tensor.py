"""Per-tensor quantisation (group = 0: one step for the whole layer, the
tutorial's 量化基础) through the search and the workspace pack, against the
oracle. Tolerances as in test_gpu_parity: losses within 1e-2, the chosen
alpha within the oracle's 0.5 % set, codes bit-exact away from rounding
boundaries, the fp16 step within its rounding. The boundary mask of the
per-tensor quantiser is taken over the whole layer (one step for all rows)."""
import numpy as np
import pytest

from awq_inputs import custom, make_inputs
from oracle import awq_oracle as O

from gpu_util import to_device, unpack_words, bf16_to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import weight_only_int4_act_b200 as awq  # noqa: E402
from test_gpu_parity import LOSS_RTOL, TIE_REL  # noqa: E402

CASES = {
    "sym4_256x512_N300": custom(256, 512, 300, bits=4, symmetric=True, group=0, seed=21),
    "asym3_200x384_N77": custom(200, 384, 77, bits=3, symmetric=False, group=0, seed=22),
    "sym4_130x256_N1024_gram": custom(130, 256, 1024, bits=4, symmetric=True, group=0, seed=23),
    "asym4_64x1024_N40_lognormal": custom(64, 1024, 40, bits=4, symmetric=False, group=0, x_lognormal_sigma=1.5,
                                          seed=24),
}


@pytest.mark.parametrize("name", list(CASES))
def test_per_tensor_search_and_pack(name):
    wl = CASES[name]
    Wb, Xb = make_inputs(wl)
    W, X = to_device(Wb), to_device(Xb)
    cfg = awq.make_cfg(wl.bits, 0, wl.symmetric, wl.n_alpha)
    a = awq.act_stats(X)
    res = awq.search_scales(W, X, a, cfg, row_losses=True)
    torch.cuda.synchronize()
    awq.workspace_error(res["ws"])
    a_ref = O.act_stats(Xb)
    ref = O.search(Wb, Xb, a_ref, wl.bits, 0, wl.symmetric, wl.n_alpha)
    losses = res["losses"].cpu().numpy().astype(np.float64)
    rel = np.abs(losses - ref["losses"]) / ref["losses"]
    assert rel.max() <= LOSS_RTOL, (rel.max(), losses, ref["losses"])
    best = int(res["best"].item())
    assert best in O.acceptable_choices(ref["losses"], TIE_REL), (best, ref["losses"])

    # per-row losses of every candidate, rows with a near-boundary element left out
    W64 = O.widen_bf16(Wb)
    rl = res["row_losses"].cpu().numpy().astype(np.float64)
    for k, al in enumerate(O.alpha_grid(wl.n_alpha)):
        s = O.candidate_scales(a_ref, al)
        ref_rows = O.row_losses_direct(O.delta_weight(W64, s, wl.bits, 0, wl.symmetric), Xb)
        near = O.boundary_mask(Wb, s, wl.bits, 0, wl.symmetric).any(axis=1)
        bad = (np.abs(rl[k] - ref_rows) > LOSS_RTOL * ref_rows + 1e-3 * ref_rows.mean()) & ~near
        assert not bad.any(), (k, np.flatnonzero(bad)[:5])

    # the pack at the chosen scales: one fp16 step and zero point for the layer
    s_ref = O.candidate_scales(a_ref, O.alpha_grid(wl.n_alpha)[best])
    q, sc, zr = awq.quantize_pack(W, res["s_best"], cfg)
    torch.cuda.synchronize()
    assert sc.shape == (1, 1) and zr.shape == (1, 1)
    _, sc_ref, zr_ref, codes_ref, _, _ = O.pack(Wb, s_ref, wl.bits, 0, wl.symmetric)
    near = O.boundary_mask(Wb, s_ref, wl.bits, 0, wl.symmetric)
    codes = unpack_words(q, wl.d_in)
    assert not ((codes != codes_ref) & ~near).any()
    assert abs(float(sc.item()) - float(sc_ref[0, 0])) <= 2.0 ** -10 * abs(float(sc_ref[0, 0]))
    if not near.any():
        assert float(zr.item()) == float(zr_ref[0, 0])
    print(name, "best", best, "max rel loss err", rel.max())


def test_per_tensor_dw_elementwise():
    """The bf16 dW stack of the per-tensor quantiser equals the oracle's
    Q(WS)S^-1 - W to bf16 rounding, away from rounding boundaries."""
    wl = CASES["sym4_256x512_N300"]
    Wb, Xb = make_inputs(wl)
    W, X = to_device(Wb), to_device(Xb)
    cfg = awq.make_cfg(4, 0, True, 20)
    res = awq.search_scales(W, X, awq.act_stats(X), cfg)
    a_ref = O.act_stats(Xb)
    Wf = O.widen_bf16(Wb)
    for k in (0, 9, 19):
        s = O.candidate_scales(a_ref, O.alpha_grid(20)[k])
        ref = O.delta_weight(Wf, s, 4, 0, True)
        got = bf16_to_f64(awq.debug_dw(res["ws"], wl.d_out, wl.d_in, wl.N, cfg, k))
        near = O.boundary_mask(Wb, s, 4, 0, True)
        tol = 2.0 ** -8 * np.abs(ref) + 4e-6 * np.abs(Wf) + 1e-30
        bad = (np.abs(got - ref) > tol) & ~near
        assert not bad.any(), (k, bad.sum())
