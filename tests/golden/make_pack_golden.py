"""Write the oracle's packed output of the full-size workloads, as digests.

    python tests/golden/make_pack_golden.py C1 C2 C3 C4 C5

For each workload and each choice of alpha the stored oracle run accepts
(tests/golden/search_<key>.json: the choices within 0.5% of the best), this
runs only the CPU oracle (statistics, the scales of that alpha, the pack in
row chunks and the rounding-boundary band) on the seeded inputs and stores:

  * pack_<key>.npz: the flat indices of the codes whose v/Delta lies within
    1e-4 of a half-integer, the oracle's codes there, and the flat indices of
    the groups whose -min/Delta does (their zero point and every code of the
    group may round either way in float32);
  * pack_<key>.json: SHA-256 of the codes (uint8, [d_out, d_in], row-major)
    and of the fp16 zero points (uint16 bits, [d_out, d_in/g]) with those
    positions overwritten by 0xFF / 0xFFFF, the sum of the fp16 steps, and the
    counts.

bench.py reads these to check every code of the timed run's pack without
running the oracle.
"""
import hashlib
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from awq_inputs import WORKLOADS, make_inputs  # noqa: E402
from oracle import awq_oracle as O  # noqa: E402

CHUNK_ROWS = 2048


def masked_digests(codes, zeros_bits, el_idx, zn_idx, group):
    """SHA-256 of codes and zero points with the band's positions blanked."""
    c = np.array(codes, dtype=np.uint8, copy=True)
    z = np.array(zeros_bits, dtype=np.uint16, copy=True)
    c.reshape(-1)[el_idx] = 0xFF
    ng = z.shape[1]
    cg = c.reshape(c.shape[0], ng, group)
    r, j = np.divmod(zn_idx.astype(np.int64), ng)
    cg[r, j, :] = 0xFF
    z.reshape(-1)[zn_idx] = 0xFFFF
    return hashlib.sha256(c.tobytes()).hexdigest(), hashlib.sha256(z.tobytes()).hexdigest()


def main(keys):
    for key in keys:
        wl = WORKLOADS[key]
        with open(os.path.join(HERE, f"search_{key}.json")) as f:
            srch = json.load(f)
        assert srch["workload"] == wl.as_dict()
        t0 = time.time()
        Wb, Xb = make_inputs(wl)
        a = O.act_stats(Xb)
        del Xb
        ng = wl.d_in // wl.group
        meta = {"workload": wl.as_dict(),
                "written_by": "tests/golden/make_pack_golden.py (CPU oracle only, float64)",
                "band": 1e-4, "choices": {}}
        arrays = {}
        for k in srch["acceptable"]:
            s = O.candidate_scales(a, O.alpha_grid(wl.n_alpha)[k])
            codes = np.empty((wl.d_out, wl.d_in), dtype=np.uint8)
            zeros = np.empty((wl.d_out, ng), dtype=np.uint16)
            scale_sum = 0.0
            el_idx, zn_idx = [], []
            for r0 in range(0, wl.d_out, CHUNK_ROWS):
                r1 = min(wl.d_out, r0 + CHUNK_ROWS)
                _, sc, zr, cd, _, _ = O.pack(Wb[r0:r1], s, wl.bits, wl.group, wl.symmetric)
                el, zn = O.boundary_mask(Wb[r0:r1], s, wl.bits, wl.group, wl.symmetric, parts=True)
                codes[r0:r1] = cd
                zeros[r0:r1] = zr.view(np.uint16)
                scale_sum += float(sc.astype(np.float64).sum())
                el_idx.append(np.flatnonzero(el) + r0 * wl.d_in)
                zn_idx.append(np.flatnonzero(zn) + r0 * ng)
            el_idx = np.concatenate(el_idx).astype(np.uint32)
            zn_idx = np.concatenate(zn_idx).astype(np.uint32)
            cdig, zdig = masked_digests(codes, zeros, el_idx, zn_idx, wl.group)
            arrays[f"k{k}_near_idx"] = el_idx
            arrays[f"k{k}_near_codes"] = codes.reshape(-1)[el_idx]
            arrays[f"k{k}_zero_near_groups"] = zn_idx
            meta["choices"][str(k)] = {"codes_sha256": cdig, "zeros_sha256": zdig, "scale_sum": scale_sum,
                                       "near_codes": int(el_idx.size), "near_zero_points": int(zn_idx.size),
                                       "codes": wl.d_out * wl.d_in, "groups": wl.d_out * ng}
            print(key, k, meta["choices"][str(k)], flush=True)
        meta["seconds"] = round(time.time() - t0, 1)
        np.savez_compressed(os.path.join(HERE, f"pack_{key}.npz"), **arrays)
        with open(os.path.join(HERE, f"pack_{key}.json"), "w") as f:
            json.dump(meta, f, indent=1)


if __name__ == "__main__":
    main(sys.argv[1:] or ["C1", "C2", "C3", "C4", "C5"])
