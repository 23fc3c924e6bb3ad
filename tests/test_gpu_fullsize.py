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
  * every packed code, step and zero point of the layer is compared with the
    oracle's pack at the chosen scales (in row chunks), the codes bit-exact
    off the rounding-boundary band; the codes the band excludes and the ones
    that differ inside it are counted and printed, and the excluded fraction
    is bounded;
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

from gpu_util import to_device, unpack_words_np

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import weight_only_int4_act_b200 as awq  # noqa: E402
from test_gpu_parity import A_RTOL, EXCLUDE_FRAC, LOSS_RTOL, TIE_REL, check_row_losses  # noqa: E402

GOLDEN = pathlib.Path(__file__).parent / "golden"
CHUNK_ROWS = 2048


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
    words_gpu = q.cpu().numpy().view(np.uint32)
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

    # 8 seeded rows: per-row losses at every alpha
    rows = np.sort(np.random.default_rng(wl.seed).choice(wl.d_out, 8, replace=False))
    check_row_losses(Wb, Xb, a_ref, wl, rows, rl)
    s_ref = O.candidate_scales(a_ref, O.alpha_grid(wl.n_alpha)[best])
    assert np.allclose(s_gpu, s_ref, rtol=1e-5)

    # every code, step and zero point of the layer, in row chunks
    el_all = np.zeros(wl.d_out, dtype=np.int64)
    zn_n, flipped, zflip = 0, 0, 0
    ng = wl.d_in // wl.group
    for r0 in range(0, wl.d_out, CHUNK_ROWS):
        r1 = min(wl.d_out, r0 + CHUNK_ROWS)
        _, sc_ref, zr_ref, codes_ref, _, _ = O.pack(Wb[r0:r1], s_ref, wl.bits, wl.group, wl.symmetric)
        el, zn = O.boundary_mask(Wb[r0:r1], s_ref, wl.bits, wl.group, wl.symmetric, parts=True)
        near = el | np.repeat(zn, wl.group, axis=1)
        codes = unpack_words_np(words_gpu[r0:r1], wl.d_in)
        diff = codes != codes_ref
        assert not (diff & ~near).any(), f"rows {r0}..{r1}: {int((diff & ~near).sum())} codes differ off the band"
        assert np.all(np.abs(sc_gpu[r0:r1].astype(np.float64) - sc_ref.astype(np.float64))
                      <= 2.0 ** -10 * np.abs(sc_ref.astype(np.float64)))
        zd = zr_gpu[r0:r1] != zr_ref
        assert not (zd & ~zn).any(), f"rows {r0}..{r1}: zero points differ off the band"
        el_all[r0:r1] = el.sum(axis=1)
        zn_n += int(zn.sum())
        flipped += int(diff.sum())
        zflip += int(zd.sum())
    n_el = int(el_all.sum())
    assert n_el <= EXCLUDE_FRAC * wl.d_out * wl.d_in + 3
    assert zn_n <= EXCLUDE_FRAC * wl.d_out * ng + 1
    print(f"{key} codes compared {wl.d_out * wl.d_in}: near-boundary elements {n_el} "
          f"({n_el / (wl.d_out * wl.d_in):.2e}), near-boundary zero points {zn_n} of {wl.d_out * ng}, "
          f"codes differing inside the band {flipped}, zero points differing inside the band {zflip}")
