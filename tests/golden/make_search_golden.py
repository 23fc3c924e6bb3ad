"""Write the oracle's full candidate losses for the full-size workloads.

    python tests/golden/make_search_golden.py C2 C3 C4 C5

For each workload this runs only the CPU oracle (float64; the Gram form
G = X^T X, which equals the direct sum up to float64 rounding) on the seeded
inputs and stores the losses of every alpha, the oracle's choice, the set of
choices within 0.5% of the best, and a hash of the bf16 inputs (so that a test
can confirm it sees the same bytes). The GPU tests compare against these files.
"""
import hashlib
import json
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from awq_inputs import WORKLOADS, make_inputs  # noqa: E402
from oracle import awq_oracle as O  # noqa: E402


def input_hash(Wb, Xb):
    h = hashlib.sha256()
    h.update(Wb.tobytes())
    h.update(Xb.tobytes())
    return h.hexdigest()


def main(keys):
    for key in keys:
        wl = WORKLOADS[key]
        t0 = time.time()
        Wb, Xb = make_inputs(wl)
        a = O.act_stats(Xb)
        res = O.search(Wb, Xb, a, wl.bits, wl.group, wl.symmetric, wl.n_alpha, form="gram")
        out = {
            "workload": wl.as_dict(),
            "written_by": "tests/golden/make_search_golden.py (CPU oracle only, float64, Gram form)",
            "input_sha256": input_hash(Wb, Xb),
            "losses": [float(x) for x in res["losses"]],
            "best": int(res["best"]),
            "acceptable": O.acceptable_choices(res["losses"], 0.005),
            "a_checksum": float(a.sum()),
            "seconds": round(time.time() - t0, 1),
        }
        with open(os.path.join(HERE, f"search_{key}.json"), "w") as f:
            json.dump(out, f, indent=1)
        print(key, out["best"], out["acceptable"], out["seconds"], flush=True)


if __name__ == "__main__":
    main(sys.argv[1:] or ["C2", "C3", "C4", "C5"])
