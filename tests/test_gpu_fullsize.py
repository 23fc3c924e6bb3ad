"""Parity at the full workload sizes, in the launch configuration bench.py
times (automatic contraction form, one stream).

At these sizes the oracle cannot redo the whole search within a test, so:
  * a_i is compared for every channel (the oracle's statistics are cheap);
  * every candidate loss and the choice are compared with the oracle's full
    losses stored in tests/golden/search_<key>.json (written by
    tests/golden/make_search_golden.py, which calls only the oracle), after
    checking that the seeded inputs hash to the same bytes;
  * per-row losses of 8 seeded rows, at every alpha, are compared with the
    oracle's direct definition;
  * the codes, steps and zero points of those rows are compared with the
    oracle's pack at the chosen scales;
  * properties that hold at any size: row losses sum to the losses, the
    returned index is the argmin of the returned losses, s_best is that
    candidate's scale vector.
"""
import hashlib
import json
import pathlib

import numpy as np
import pytest

from awq_inputs import WORKLOADS, make_inputs
from oracle import awq_oracle as O

from gpu_util import to_device, unpack_words

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import weight_only_int4_act_b200 as awq  # noqa: E402
from test_gpu_parity import A_RTOL, LOSS_RTOL, TIE_REL, check_row_losses  # noqa: E402

GOLDEN = pathlib.Path(__file__).parent / "golden"


@pytest.mark.parametrize("key", ["C2", "C3", "C4", "C5"])
def test_full_size(key):
    wl = WORKLOADS[key]
    Wb, Xb = make_inputs(wl)
    W, X = to_device(Wb), to_device(Xb)
    cfg = awq.make_cfg(wl.bits, wl.group, wl.symmetric, wl.n_alpha)
    a = awq.act_stats(X)
    res = awq.search_scales(W, X, a, cfg, row_losses=True)
    q, sc, zr = awq.quantize_pack(W, res["s_best"], cfg)
    torch.cuda.synchronize()
    awq.workspace_error(res["ws"])
    losses = res["losses"].cpu().numpy().astype(np.float64)
    rl = res["row_losses"].cpu().numpy().astype(np.float64)
    best = int(res["best"].item())
    s_gpu = res["s_best"].cpu().numpy()
    codes_gpu = unpack_words(q, wl.d_in)
    sc_gpu = sc.cpu().numpy()
    zr_gpu = zr.cpu().numpy()
    del res, q, sc, zr, W, X
    torch.cuda.empty_cache()

    # statistics, every channel
    a_ref = O.act_stats(Xb)
    a_g = a.cpu().numpy().astype(np.float64)
    assert (np.abs(a_g - a_ref) / a_ref).max() <= A_RTOL

    # properties at any size
    assert np.allclose(rl.sum(axis=1), losses, rtol=1e-5)
    assert best == int(np.argmin(losses))
    print(key, "form", awq.search_form(wl.d_out, wl.d_in, wl.N, cfg), "best", best)

    # full losses against the stored oracle values
    gpath = GOLDEN / f"search_{key}.json"
    if gpath.exists():
        g = json.loads(gpath.read_text())
        h = hashlib.sha256()
        h.update(Wb.tobytes())
        h.update(Xb.tobytes())
        assert h.hexdigest() == g["input_sha256"], "seeded inputs differ from the stored oracle run"
        ref = np.array(g["losses"])
        rel = np.abs(losses - ref) / ref
        print(key, "max rel loss err vs oracle", rel.max())
        assert rel.max() <= LOSS_RTOL
        assert best in g["acceptable"], (best, g["best"], g["acceptable"])
    else:
        pytest.fail(f"missing {gpath.name}: run tests/golden/make_search_golden.py {key}")

    # 8 seeded rows: per-row losses at every alpha, and their packed codes
    rows = np.sort(np.random.default_rng(wl.seed).choice(wl.d_out, 8, replace=False))
    check_row_losses(Wb, Xb, a_ref, wl, rows, rl)
    s_ref = O.candidate_scales(a_ref, O.alpha_grid(wl.n_alpha)[best])
    assert np.allclose(s_gpu, s_ref, rtol=1e-5)
    _, sc_ref, zr_ref, codes_ref, _, _ = O.pack(Wb[rows], s_ref, wl.bits, wl.group, wl.symmetric)
    near = O.boundary_mask(Wb[rows], s_ref, wl.bits, wl.group, wl.symmetric)
    assert not ((codes_gpu[rows] != codes_ref) & ~near).any()
    assert np.all(np.abs(sc_gpu[rows].astype(np.float64) - sc_ref.astype(np.float64))
                  <= 2.0 ** -10 * np.abs(sc_ref.astype(np.float64)))
    gnear = near.reshape(len(rows), -1, wl.group).any(axis=-1)
    assert not ((zr_gpu[rows] != zr_ref) & ~gnear).any()
    print(key, "codes near boundary", int(near.sum()), "flipped", int((codes_gpu[rows] != codes_ref).sum()))
