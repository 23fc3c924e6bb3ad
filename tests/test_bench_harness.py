"""Host-side logic of bench.py: the max-over-ranks timing used when one
process per GPU runs under torchrun (checked here with 2 gloo ranks on the
CPU), the triangular multiply-add count, launch counting, the ncu-summary
reader, and the reference (CPU oracle) arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [float(rank + 1), 10.0 - rank, 3.0]
        res = bench.max_over_ranks(mine, "cpu")
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        assert json.loads((tmp_path / f"r{r}.json").read_text()) == [2.0, 10.0, 3.0]


def test_tri_macs_matches_block_count():
    for d_in in (64, 256, 384, 4096, 11008):
        brute = 0
        for i in range(d_in):
            brute += min(d_in, (i // 256 + 1) * 256)  # row i of G' holds columns of blocks <= its block
        assert bench.tri_macs_per_row(d_in) == brute


def test_launch_count():
    assert bench.launches_per_step("direct", 20) == 8
    assert bench.launches_per_step("gram", 20) == 9
    assert bench.launches_per_step("gram", 20, 4096, 4096) == 9      # C2: a last wave of 62 of 74 pairs
    assert bench.launches_per_step("gram", 20, 8192, 65536) == 10    # C5: 528 = 7 x 74 + 10 tiles, split in K


def test_profiled_traffic_requires_matching_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "contract_pair_gram_CX.md").write_text(
        f"- source_sha256: `{bench.kernel_source_hash()}`\n- traffic_bytes_per_launch: `123`\n")
    (prof / "contract_pair_gram_CY.md").write_text("- source_sha256: `0000`\n- traffic_bytes_per_launch: `456`\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "weight_only_int4_act_b200" / "csrc").mkdir(parents=True)
    for f in ("gemm_pair_sm100.cuh", "gemm_sm100.cuh", "ptx.cuh", "awq_api.cu"):
        src = os.path.join(ROOT, "weight_only_int4_act_b200", "csrc", f)
        (tmp_path / "weight_only_int4_act_b200" / "csrc" / f).write_bytes(open(src, "rb").read())
    assert bench.profiled_traffic("CX", "gram") == 123.0
    assert bench.profiled_traffic("CY", "gram") is None
    assert bench.profiled_traffic("CZ", "gram") is None


def test_reference_arm_json_line(tmp_path):
    dest = tmp_path / "ref.json"
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "C1",
                          "--steps", "1", "--warmup", "3", "--ref-rows", "64", "--json-out", str(dest)],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert json.loads(dest.read_text()) == line
    assert line["impl"] == "reference" and line["unit"] == bench.UNIT and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["higher_is_better"] is True
    assert line["extrapolated"] is True and line["sample_s_per_step"] > 0 and line["cpu_baseline"]["cores"] == 1
    from awq_inputs import configs
    assert line["config"] == bench.workload_config(configs.WORKLOADS["C1"], 1)


def test_sample_rows_bounded():
    from awq_inputs import configs
    for key, wl in configs.WORKLOADS.items():
        for secs in (3.0, 15.0):
            r = bench.sample_rows(wl, secs)
            assert 8 <= r <= wl.d_out and (r % 8 == 0 or r == wl.d_out), key
            # per-row oracle cost ~ d_in * N: the sample stays within its time unless at its floor
            assert r == 8 or r * wl.d_in * wl.N * bench.ORACLE_ROW_COST_S <= secs, key
    assert bench.sample_rows(configs.WORKLOADS["C1"], 15.0) == 256  # the whole small layer


def test_reference_step_sample_bounded():
    """The oracle arm's step: rows as sample_rows gives them, and a token
    slice (a multiple of 1024) only where 8 rows over every token would
    overrun the step's budget; the estimated work then stays within it."""
    from awq_inputs import configs
    for key, wl in configs.WORKLOADS.items():
        rows, tokens = bench.ref_sample(wl, bench.REF_STEP_S)
        assert rows == bench.sample_rows(wl, bench.REF_STEP_S), key
        assert tokens == wl.N or (tokens % 1024 == 0 and 1024 <= tokens < wl.N), key
        if tokens < wl.N:
            assert rows == 8, key
        est = rows * wl.d_in * tokens * bench.ORACLE_ROW_COST_S
        assert est <= bench.REF_STEP_S or tokens == 1024 or (rows == 8 and tokens == wl.N), key
    assert bench.ref_sample(configs.WORKLOADS["C5"], bench.REF_STEP_S)[1] < 65536  # C5 runs on a token slice


def test_pack_parity_against_stored_digests():
    """bench's code check: the oracle's own pack of C1 passes; a code changed
    away from the rounding-boundary band fails it; a code changed inside the
    band is counted and passes."""
    import numpy as np
    import torch
    from awq_inputs import configs
    from oracle import awq_oracle as O
    wl = configs.WORKLOADS["C1"]
    with open(os.path.join(ROOT, "tests", "golden", "search_C1.json")) as f:
        k = json.load(f)["best"]
    Wb, Xb = configs.make_inputs(wl)
    s = O.candidate_scales(O.act_stats(Xb), O.alpha_grid(wl.n_alpha)[k])
    qw, sc, zr, codes, _, _ = O.pack(Wb, s, wl.bits, wl.group, wl.symmetric)
    el = O.boundary_mask(Wb, s, wl.bits, wl.group, wl.symmetric)

    def as_torch(q, c=None):
        if c is not None:
            q = O.pack_codes(c)
        return (torch.from_numpy(q.view(np.int32)), torch.from_numpy(sc), torch.from_numpy(zr))

    res = bench.pack_parity(wl, k, *as_torch(qw))
    assert res["ok"] and res["codes_differing_inside_band"] == 0 and res["compared"] == Wb.size
    far = codes.copy()
    r, c = np.argwhere(~el)[5]
    far[r, c] ^= 1
    assert not bench.pack_parity(wl, k, *as_torch(None, far))["ok"]
    inside = codes.copy()
    r, c = np.argwhere(el)[0]
    inside[r, c] ^= 1
    res = bench.pack_parity(wl, k, *as_torch(None, inside))
    assert res["ok"] and res["codes_differing_inside_band"] == 1
    assert not bench.pack_parity(wl, (k + 5) % wl.n_alpha, *as_torch(qw))["ok"]  # no digest for that choice


def test_golden_parity_reads_stored_oracle_runs():
    import json as _json
    from awq_inputs import configs, custom
    for key in ("C1", "C2", "C3", "C4", "C5"):
        wl = configs.WORKLOADS[key]
        with open(os.path.join(ROOT, "tests", "golden", f"search_{key}.json")) as f:
            g = _json.load(f)
        a_const = [g["a_checksum"] / wl.d_in] * wl.d_in
        near = bench.golden_parity(wl, [v * (1 + 1e-4) for v in g["losses"]], g["best"], a_const)
        assert near["ok"] and abs(near["loss_max_rel"] - 1e-4) < 1e-9 and near["a_sum_rel"] < 1e-9, key
        far = bench.golden_parity(wl, [v * 1.05 for v in g["losses"]], g["best"], a_const)
        assert not far["ok"], key
        wrong = [k for k in range(wl.n_alpha) if k not in g["acceptable"]][0]
        assert not bench.golden_parity(wl, g["losses"], wrong, a_const)["ok"], key
    assert bench.golden_parity(custom(64, 256, 32), [1.0] * 20, 0, [1.0] * 256) is None


def test_seed_flag_changes_the_inputs(tmp_path):
    """--seed reseeds the workload (here through the oracle arm, which needs no GPU)."""
    lines = []
    for seed in ("", "123"):
        cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "C1",
               "--steps", "1", "--warmup", "3", "--ref-rows", "32"] + (["--seed", seed] if seed else [])
        out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
        assert out.returncode == 0, out.stderr
        lines.append(json.loads(out.stdout.strip().splitlines()[-1]))
    assert all(ln["impl"] == "reference" and ln["value"] > 0 for ln in lines)
    from awq_inputs import configs
    wl = configs.WORKLOADS["C1"]
    import dataclasses
    a0 = configs.make_inputs(wl)[1]
    a1 = configs.make_inputs(dataclasses.replace(wl, seed=123))[1]
    assert not (a0 == a1).all()
    # a reseeded workload has no stored oracle run to compare with
    g = bench.golden_parity(dataclasses.replace(wl, seed=123), [1.0] * 20, 0, [1.0] * 512)
    assert g is not None and "error" in g
