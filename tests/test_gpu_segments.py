"""Several layers that read the same activations, searched in one call
(awq_search_scales_segmented) against the oracle run on each layer alone;
and the shared-scale variant (awq_search_scales on the row concatenation)
against the oracle on the concatenation."""
import numpy as np
import pytest

from awq_inputs import custom, make_inputs, make_weight_rows
from oracle import awq_oracle as O

from gpu_util import to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import weight_only_int4_act_b200 as awq  # noqa: E402
from test_gpu_parity import LOSS_RTOL, TIE_REL  # noqa: E402


@pytest.mark.parametrize("seg_rows,bits,sym,g", [((96, 200, 150), 4, False, 128), ((128, 64), 3, True, 64),
                                                 ((300,), 4, False, 128)])
def test_segmented_matches_per_layer_oracle(seg_rows, bits, sym, g):
    d_in, N = 512, 700
    layers = [make_inputs(custom(r, d_in, N, bits=bits, symmetric=sym, group=g, seed=40 + i))[0]
              for i, r in enumerate(seg_rows)]
    _, Xb = make_inputs(custom(8, d_in, N, bits=bits, symmetric=sym, group=g, seed=40))
    Wcat = np.concatenate(layers, axis=0)
    W, X = to_device(Wcat), to_device(Xb)
    cfg = awq.make_cfg(bits, g, sym, 20)
    a = awq.act_stats(X)
    res = awq.search_scales_segmented(W, X, a, cfg, list(seg_rows), row_losses=True)
    torch.cuda.synchronize()
    awq.workspace_error(res["ws"])
    a_ref = O.act_stats(Xb)
    losses = res["losses"].cpu().numpy().astype(np.float64)
    best = res["best"].cpu().numpy()
    s_best = res["s_best"].cpu().numpy().astype(np.float64)
    for i, Wl in enumerate(layers):
        ref = O.search(Wl, Xb, a_ref, bits, g, sym, 20)
        assert np.all(np.abs(losses[i] - ref["losses"]) <= LOSS_RTOL * ref["losses"]), i
        assert int(best[i]) in O.acceptable_choices(ref["losses"], TIE_REL), (i, best[i], ref["best"])
        assert np.allclose(s_best[i], O.candidate_scales(a_ref, O.alpha_grid(20)[best[i]]), rtol=1e-5)
    # the per-layer losses add up to the shared (concatenated) search's losses
    shared = awq.search_scales(W, X, a, cfg)
    torch.cuda.synchronize()
    tot = shared["losses"].cpu().numpy().astype(np.float64)
    assert np.allclose(losses.sum(axis=0), tot, rtol=1e-5)
    ref_cat = O.search(Wcat, Xb, a_ref, bits, g, sym, 20)
    assert int(shared["best"].item()) in O.acceptable_choices(ref_cat["losses"], TIE_REL)
