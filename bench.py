"""Benchmark of the AWQ calibration / scale-search path on B200.

One step = the whole hot path for one linear layer: activation statistics,
candidate scales, the fake-quantised dW stack, (Gram product,) the tensor-core
error contraction with its fused squared-sum epilogue, the fixed-order
reduction with argmin, and the pack at the chosen scales.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C2] [--impl ours|reference]

Prints one JSON line (rank 0). The metric is alpha-candidate layer
evaluations per second (n_alpha / step time, summed over ranks); under
torchrun every rank runs its own replica of the layer ("replicas only": the
path has no exchange step). `--impl reference` times the CPU oracle on a
bounded row sample of the same layer instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from awq_inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "AWQ search: alpha-candidate layer evals/s, TFLOP/s vs bf16 peak; stats GB/s"
UNIT = "alpha-candidate layer evals/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
L2_FLUSH_BYTES = 256 << 20
LONG_STEP_MS = 10.0  # steps at least this long are timed against the sustained (power-capped) peak
GROUP_CLIPS = [1.0, 0.95, 0.9, 0.85, 0.8, 0.75, 0.7, 0.6, 0.5]  # ratios of the per-group clipping pass


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


LOSS_RTOL = 1e-2  # candidate losses against the oracle's (relative)
STATS_RTOL = 1e-5  # activation statistics against the oracle's (relative)


def golden_parity(wl, losses, best, a, packed=None):
    """The timed run's outputs against the stored oracle run of the same seeded
    workload (tests/golden/search_<key>.json and pack_<key>.{json,npz},
    written by tests/golden/make_search_golden.py and make_pack_golden.py,
    which call only the oracle): every candidate loss, the choice (inside the
    oracle's set of choices within 0.5 % of its best), the sum of the
    activation statistics, and, when ``packed`` = (qweight, scales, zeros) is
    given, every packed code and zero point (a SHA-256 of the layer's codes
    with the oracle's rounding-boundary positions blanked must equal the
    stored one; the codes inside the band are counted) and the sum of the fp16
    steps. Reads stored numbers only; None if the workload has no stored run."""
    path = os.path.join(ROOT, "tests", "golden", f"search_{wl.key}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        g = json.load(f)
    out = {"against": f"tests/golden/search_{wl.key}.json (stored oracle run, float64)"}
    if g.get("workload") != wl.as_dict():
        out["error"] = "the stored run was made for other inputs"
        return out
    ref = np.asarray(g["losses"], dtype=np.float64)
    got = np.asarray(losses, dtype=np.float64)
    rel = float(np.max(np.abs(got - ref) / ref))
    a_rel = abs(float(np.sum(np.asarray(a, dtype=np.float64))) - g["a_checksum"]) / g["a_checksum"]
    ok = bool(rel <= LOSS_RTOL and int(best) in g["acceptable"] and a_rel <= STATS_RTOL)
    out.update({"loss_max_rel": rel, "loss_rtol": LOSS_RTOL,
                "alpha_index": int(best), "oracle_alpha_set": g["acceptable"], "a_sum_rel": a_rel})
    if packed is not None:
        codes = pack_parity(wl, int(best), *packed)
        out["codes"] = codes
        ok = ok and bool(codes.get("ok"))
    out["ok"] = ok
    return out


def unpack_codes_host(words, d_in):
    """uint32 words [rows, d_in/8] -> codes uint8 [rows, d_in] (nibble j of
    word w is channel 8w + j)."""
    rows = words.shape[0]
    out = np.empty((rows, d_in // 8, 8), dtype=np.uint8)
    for j in range(8):
        out[:, :, j] = (words >> np.uint32(4 * j)) & np.uint32(0xF)
    return out.reshape(rows, d_in)


def pack_parity(wl, best, qweight, scales, zeros):
    """Every code and zero point of the timed run's pack against the stored
    oracle digests of the same choice of alpha (see golden_parity)."""
    jpath = os.path.join(ROOT, "tests", "golden", f"pack_{wl.key}.json")
    npath = os.path.join(ROOT, "tests", "golden", f"pack_{wl.key}.npz")
    if not (os.path.exists(jpath) and os.path.exists(npath)):
        return {"ok": False, "error": f"no stored pack digest for {wl.key}"}
    with open(jpath) as f:
        meta = json.load(f)
    if meta.get("workload") != wl.as_dict() or str(best) not in meta["choices"]:
        return {"ok": False, "error": "no stored pack digest for this workload and choice"}
    ch = meta["choices"][str(best)]
    arr = np.load(npath)
    el_idx = arr[f"k{best}_near_idx"].astype(np.int64)
    near_ref = arr[f"k{best}_near_codes"]
    zn_idx = arr[f"k{best}_zero_near_groups"].astype(np.int64)
    codes = unpack_codes_host(qweight.cpu().numpy().view(np.uint32), wl.d_in)
    zbits = zeros.cpu().numpy().view(np.uint16).copy()
    ng = wl.d_in // wl.group
    flipped = int((codes.reshape(-1)[el_idx] != near_ref).sum())
    codes.reshape(-1)[el_idx] = 0xFF
    r, j = np.divmod(zn_idx, ng)
    codes.reshape(codes.shape[0], ng, wl.group)[r, j, :] = 0xFF
    zbits.reshape(-1)[zn_idx] = 0xFFFF
    codes_ok = hashlib.sha256(codes.tobytes()).hexdigest() == ch["codes_sha256"]
    zeros_ok = hashlib.sha256(zbits.tobytes()).hexdigest() == ch["zeros_sha256"]
    sc_sum = float(scales.cpu().numpy().astype(np.float64).sum())
    sc_rel = abs(sc_sum - ch["scale_sum"]) / ch["scale_sum"]
    return {"against": f"tests/golden/pack_{wl.key}.json (stored oracle pack digests)",
            "compared": ch["codes"], "zero_points_compared": ch["groups"],
            "codes_equal_off_band": bool(codes_ok), "zero_points_equal_off_band": bool(zeros_ok),
            "near_boundary_codes": ch["near_codes"], "near_boundary_zero_points": ch["near_zero_points"],
            "excluded_fraction": round((ch["near_codes"] + ch["near_zero_points"] * wl.group) / ch["codes"], 7),
            "codes_differing_inside_band": flipped, "scale_sum_rel": sc_rel,
            "ok": bool(codes_ok and zeros_ok and sc_rel <= 1e-3)}


L2_NOTE = ("flushed: 256 MiB write between timed GPU steps, outside the step events "
           "(the CPU oracle arm has no device cache to flush)")


def workload_config(wl, world):
    """The workload as both arms name it (same keys and values)."""
    return {"workload": f"{wl.key}: {wl.title}", "d_out": wl.d_out, "d_in": wl.d_in, "N": wl.N,
            "bits": wl.bits, "group": wl.group, "symmetric": wl.symmetric, "n_alpha": wl.n_alpha,
            "l2": L2_NOTE, "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("gemm_pair_sm100.cuh", "gemm_sm100.cuh", "ptx.cuh", "awq_api.cu"):  # kernels and their launch
        with open(os.path.join(ROOT, "weight_only_int4_act_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(config_key, form):
    """Per-launch DRAM bytes of the contraction from the committed ncu summary,
    if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", f"contract_pair_{form}_{config_key}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_sha256") != kernel_source_hash():
        return None
    try:
        return float(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm = [float(r[1]) for r in self.rows if len(r) >= 9 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if len(r) >= 9 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows if len(r) >= 9 for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(sm)}


def max_over_ranks(values, device):
    """Element-wise maximum of a list of floats over all ranks of the default
    process group (every rank must call it, in the same order)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu().tolist()]


def tri_macs_per_row(d_in, block=256):
    """Multiply-adds per row of the block-triangular Gram contraction:
    sum over 256-wide column blocks J of width(J) * min(d_in, 256 (J + 1))."""
    return float(sum(min(block, d_in - j0) * min(d_in, j0 + block) for j0 in range(0, d_in, block)))


def gram_tail_split(d_in, N, pairs=74):
    """Whether the Gram product's last wave runs as K pieces (and so ends with
    the fix-up launch): the library's rule for a last wave of R <= pairs / 2
    tiles of 256 x 256, S = pairs // R pieces of at least two 64-token steps."""
    nbm = -(-d_in // 256)
    tiles = nbm * (nbm + 1) // 2
    pairs = min(tiles, pairs)
    if tiles <= pairs:
        return False
    R = tiles % pairs
    if R == 0:
        return False
    S = min(pairs // R, -(-N // 64) // 2)
    return S >= 2 and R * S <= 74


def launches_per_step(form, n_alpha, d_in=0, N=0):
    # stats 2 + scales 1 + fake quant 1 + (Gram 1, + its last-wave fix-up) + contraction 1 + reduce 2 + pack 1
    return 8 + ((2 if gram_tail_split(d_in, N) else 1) if form == "gram" else 0)


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import weight_only_int4_act_b200 as awq
    from weight_only_int4_act_b200 import binding as B

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[args.config]
    Wb, Xb = make_inputs(wl)
    d_out, d_in, N = wl.d_out, wl.d_in, wl.N
    W = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).to(dev)
    X = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).to(dev)
    cfg = awq.make_cfg(wl.bits, wl.group, wl.symmetric, wl.n_alpha, form=args.form)
    form = awq.search_form(d_out, d_in, N, cfg)
    ws = awq.workspace(awq.search_workspace_size(d_out, d_in, N, cfg))
    ws_stats = awq.workspace(awq.stats_workspace_size(N, d_in))
    a = torch.empty(d_in, dtype=torch.float32, device=dev)
    outs = dict(losses=torch.empty(wl.n_alpha, dtype=torch.float32, device=dev),
                best=torch.empty(1, dtype=torch.int32, device=dev),
                s_best=torch.empty(d_in, dtype=torch.float32, device=dev), row_losses=None)
    ng = d_in // wl.group
    packed = (torch.empty((d_out, d_in // 8), dtype=torch.int32, device=dev),
              torch.empty((d_out, ng), dtype=torch.float16, device=dev),
              torch.empty((d_out, ng), dtype=torch.float16, device=dev))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    L = B.lib()
    import ctypes
    cptr = ctypes.byref(cfg)
    wsp, wsn = ctypes.c_void_p(ws.data_ptr()), ws.numel()

    def step_api(ev):
        # the public calls, as a user makes them
        if ev is not None:
            ev[0].record()
        awq.act_stats(X, ws_stats, out=a)
        if ev is not None:
            ev[1].record()
        awq.search_scales(W, X, a, cfg, ws=ws, outputs=outs)
        if ev is not None:
            ev[2].record()
        awq.quantize_pack(W, outs["s_best"], cfg, outputs=packed)
        if ev is not None:
            ev[3].record()

    def step(ev=None):
        # the same path one step entry point at a time (no overlap), for the per-kernel breakdown
        st = B._stream()
        if ev is not None:
            ev[0].record()
        awq.act_stats(X, ws_stats, out=a)
        if ev is not None:
            ev[1].record()
        B._check(L.awq_step_scales(ctypes.c_void_p(a.data_ptr()), d_out, d_in, N, cptr, wsp, wsn, st), "scales")
        B._check(L.awq_step_fake_quant(ctypes.c_void_p(W.data_ptr()), d_out, d_in, N, cptr, wsp, wsn, st), "fq")
        if ev is not None:
            ev[2].record()
        B._check(L.awq_step_gram(ctypes.c_void_p(X.data_ptr()), d_out, d_in, N, cptr, wsp, wsn, st), "gram")
        if ev is not None:
            ev[3].record()
        B._check(L.awq_step_contract(ctypes.c_void_p(X.data_ptr()), d_out, d_in, N, cptr, wsp, wsn, st), "contract")
        if ev is not None:
            ev[4].record()
        B._check(L.awq_step_reduce(d_out, d_in, N, cptr, wsp, wsn, ctypes.c_void_p(outs["losses"].data_ptr()),
                                   ctypes.c_void_p(outs["best"].data_ptr()),
                                   ctypes.c_void_p(outs["s_best"].data_ptr()), None, st), "reduce")
        if ev is not None:
            ev[5].record()
        awq.quantize_pack(W, outs["s_best"], cfg, outputs=packed)
        if ev is not None:
            ev[6].record()

    warm_ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for _ in range(args.warmup):
        step()
        step_api(warm_ev)
    torch.cuda.synchronize()
    awq.workspace_error(ws)

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    t_wall0 = time.perf_counter()
    for k in range(K):
        flush.fill_(k & 0xFF)  # evict L2 between timed steps (outside the step's events)
        step_api(evs[k])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_wall = time.perf_counter() - t_wall0
    awq.workspace_error(ws)

    api = np.array([[evs[k][i].elapsed_time(evs[k][i + 1]) for i in range(3)] for k in range(K)])  # ms
    step_ms = api.sum(axis=1)
    total_ms = float(step_ms.sum())
    eager_losses, eager_best = outs["losses"].clone(), outs["best"].clone()

    # ---- the same public calls captured once in a CUDA graph and replayed: the
    # calls are stream-ordered with no host synchronisation, so they capture, and
    # the replay removes the host's launch time between the step's kernels
    graph, graph_note = None, "eager public calls"
    if not args.no_graph:
        try:
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                step_api(None)
            torch.cuda.current_stream().wait_stream(side)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                step_api(None)
            torch.cuda.synchronize()
            graph = g
        except Exception as e:  # report it; the eager timing stands
            graph_note = f"eager public calls (graph capture failed: {type(e).__name__})"
    if graph is not None:
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        awq.workspace_error(ws)
        gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_wall0 = time.perf_counter()
        for k in range(K):
            flush.fill_(k & 0xFF)  # outside the replay's events
            gev[k][0].record()
            graph.replay()
            gev[k][1].record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        t_wall = time.perf_counter() - t_wall0
        awq.workspace_error(ws)
        if not (torch.equal(outs["losses"], eager_losses) and torch.equal(outs["best"], eager_best)):
            raise RuntimeError("graph replay results differ from the eager calls")
        eager_total_ms = total_ms
        total_ms = float(sum(e0.elapsed_time(e1) for e0, e1 in gev))
        graph_note = "CUDA graph replay of the public calls (act_stats, search_scales, quantize_pack)"
    else:
        eager_total_ms = total_ms
    clk = clocks.stop()
    # the last timed step's outputs against the stored oracle run (stored numbers only)
    try:
        parity = golden_parity(wl, outs["losses"].cpu().numpy(), int(outs["best"].item()), a.cpu().numpy(),
                               packed=packed)
    except Exception as e:  # report it; the timing stands
        parity = {"error": f"{type(e).__name__}: {e}"}

    # per-kernel breakdown: the same work one entry point at a time
    KB = min(K, 20)
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(KB)]
    for k in range(KB):
        flush.fill_(k & 0xFF)
        step(kev[k])
    torch.cuda.synchronize()
    awq.workspace_error(ws)
    seg = np.array([[kev[k][i].elapsed_time(kev[k][i + 1]) for i in range(6)] for k in range(KB)])
    if world > 1:
        seg = np.array(max_over_ranks(seg.ravel().tolist(), dev)).reshape(seg.shape)
    if world > 1:
        total_ms = max_over_ranks([total_ms], dev)[0]
        eager_total_ms = max_over_ranks([eager_total_ms], dev)[0]
    ms_per_step = total_ms / K
    mean = seg.mean(axis=0)
    names = ["stats", "scales+fake_quant", "gram", "contraction", "reduce_argmin", "pack"]
    breakdown = {n: round(float(v), 4) for n, v in zip(names, mean)}
    api_mean = api.mean(axis=0)
    step_split = {"stats": round(float(api_mean[0]), 4), "search": round(float(api_mean[1]), 4),
                  "pack": round(float(api_mean[2]), 4)}

    # ---- end to end through the public API with host buffers. Every step copies
    # its inputs (W, X) from pinned host memory and all its results back; the
    # inputs of step k+1 are copied on a second stream while step k computes
    # (two device slots for inputs and results, ordered by events).
    Wh = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).pin_memory()
    Xh = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).pin_memory()
    dev_in = [(torch.empty_like(W), torch.empty_like(X)) for _ in range(2)]
    dev_out = [dict(losses=torch.empty_like(outs["losses"]), best=torch.empty_like(outs["best"]),
                    s_best=torch.empty_like(outs["s_best"]), row_losses=None) for _ in range(2)]
    dev_pack = [tuple(torch.empty_like(t) for t in packed) for _ in range(2)]
    host_out = [[torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in
                 (outs["losses"], outs["best"], outs["s_best"], *packed)] for _ in range(2)]
    comp = torch.cuda.current_stream()
    cstream = torch.cuda.Stream()

    def e2e_run(n):
        """n pipelined steps; returns their total device time in ms."""
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready, done, copied = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(comp)
        cstream.wait_event(t0)
        with torch.cuda.stream(cstream):
            dev_in[0][0].copy_(Wh, non_blocking=True)
            dev_in[0][1].copy_(Xh, non_blocking=True)
            in_ready[0].record(cstream)
        for k in range(n):
            sl = k % 2
            comp.wait_event(in_ready[sl])
            if k >= 2:
                comp.wait_event(copied[sl])  # step k-2's results have left this slot
            Wd, Xd = dev_in[sl]
            aa = awq.act_stats(Xd, ws_stats, out=a)
            r = awq.search_scales(Wd, Xd, aa, cfg, ws=ws, outputs=dev_out[sl])
            pk = awq.quantize_pack(Wd, r["s_best"], cfg, outputs=dev_pack[sl])
            done[sl].record(comp)
            with torch.cuda.stream(cstream):
                if k + 1 < n:
                    nx = (k + 1) % 2
                    if k >= 1:
                        cstream.wait_event(done[nx])  # step k-1 no longer reads that slot
                    dev_in[nx][0].copy_(Wh, non_blocking=True)
                    dev_in[nx][1].copy_(Xh, non_blocking=True)
                    in_ready[nx].record(cstream)
                cstream.wait_event(done[sl])
                for h, d in zip(host_out[sl], (r["losses"], r["best"], r["s_best"], *pk)):
                    h.copy_(d, non_blocking=True)
                copied[sl].record(cstream)
        comp.wait_event(copied[(n - 1) % 2])
        if n >= 2:
            comp.wait_event(copied[(n - 2) % 2])
        t1.record(comp)
        t1.synchronize()
        return t0.elapsed_time(t1)

    e2e_run(2)
    torch.cuda.synchronize()
    e2e_total = e2e_run(K)
    if world > 1:
        e2e_total = max_over_ranks([e2e_total], dev)[0]
    awq.workspace_error(ws)
    # the pipelined steps returned what the device-resident steps computed (deterministic kernels)
    last = host_out[(K - 1) % 2]
    if not (torch.equal(last[0], outs["losses"].cpu()) and torch.equal(last[1], outs["best"].cpu())):
        raise RuntimeError("end-to-end results differ from the device-resident run")
    h2d = Wb.nbytes + Xb.nbytes
    d2h = sum(h.numel() * h.element_size() for h in host_out[0])

    # ---- per-group clipping with the chosen scales (a follow-on pass, timed apart from the step)
    gclip = None
    if wl.group >= 32 and not args.no_group_clip:
        ccfg = awq.make_cfg(wl.bits, wl.group, wl.symmetric, len(GROUP_CLIPS))
        cws = awq.workspace(awq.group_clip_workspace_size(d_out, d_in, N, ccfg))
        best_clip = torch.empty((d_out, ng), dtype=torch.uint8, device=dev)
        cp = (ctypes.c_float * len(GROUP_CLIPS))(*GROUP_CLIPS)

        def clip_step():
            st = B._stream()
            B._check(L.awq_search_group_clip(ctypes.c_void_p(W.data_ptr()), ctypes.c_void_p(X.data_ptr()),
                                             ctypes.c_void_p(outs["s_best"].data_ptr()), ctypes.cast(cp, ctypes.c_void_p),
                                             d_out, d_in, N, ctypes.byref(ccfg), ctypes.c_void_p(cws.data_ptr()),
                                             cws.numel(), ctypes.c_void_p(best_clip.data_ptr()), None, st),
                     "awq_search_group_clip")
            awq.quantize_pack_group_clip(W, outs["s_best"], GROUP_CLIPS, best_clip, ccfg, outputs=packed)

        for _ in range(3):
            clip_step()
        torch.cuda.synchronize()
        g_ms = []
        for k in range(KB):
            flush.fill_(k & 0xFF)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            clip_step()
            e1.record()
            e1.synchronize()
            g_ms.append(e0.elapsed_time(e1))
        awq.workspace_error(cws)
        gms = float(np.mean(g_ms))
        if world > 1:
            gms = max_over_ranks([gms], dev)[0]
        gclip = {"clips": GROUP_CLIPS, "ms_per_pass": round(gms, 4),
                 "clip_group_evals_per_s": round(world * len(GROUP_CLIPS) * d_out * ng / (gms * 1e-3), 1),
                 "note": "search_group_clip + quantize_pack_group_clip with s_best, " + str(KB) + " passes, L2 flushed"}
        del cws

    # ---- inference side: the packed layer applied by the W4A16 kernel (timed apart from the step)
    w4 = None
    if d_in % 32 == 0 and not args.no_w4a16:
        pk = awq.quantize_pack(W, outs["s_best"], cfg)
        Xt = X.t().contiguous()
        awq.fold_inv_scales(outs["s_best"], Xt)  # activations carrying S^-1
        Xp_all = Xt.t().contiguous()
        del Xt
        peaks_ = load_peaks()
        hbm_ = peaks_.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        tc_ = peaks_.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        w4 = {}
        W16 = W.to(torch.float16)
        # decodes first: the product is issue-bound, so its time follows the SM
        # clock, which the power cap lowers for a while after the prefill loops
        for label, n_tok, dt in (("decode_16_f16", 16, torch.float16), ("decode_16_bf16", 16, torch.bfloat16),
                                 ("prefill_N_f16", N, torch.float16), ("prefill_N_bf16", N, torch.bfloat16)):
            Xp = Xp_all[:n_tok].to(dt).contiguous()
            Wd = W16 if dt == torch.float16 else W
            wsw = awq.workspace(awq.w4a16_workspace_size(n_tok, d_out, d_in, cfg))
            Yw = torch.empty((n_tok, d_out), dtype=dt, device=dev)

            def run_w4():
                awq.w4a16_gemm(Xp, *pk, cfg, ws=wsw, out=Yw)

            def run_dense():
                torch.matmul(Xp, Wd.t(), out=Yw)

            res = {}
            for nm, fn in (("w4a16", run_w4), ("bf16_dense_cublas", run_dense)):
                for _ in range(3):
                    fn()
                torch.cuda.synchronize()
                tms = []
                for k in range(KB):
                    flush.fill_(k & 0xFF)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    fn()
                    e1.record()
                    e1.synchronize()
                    tms.append(e0.elapsed_time(e1))
                res[nm] = float(np.mean(tms))
            awq.workspace_error(wsw)
            byts = d_out * d_in // 2 + 4 * d_out * ng + n_tok * d_in * 2 + n_tok * d_out * 2
            flops = 2.0 * n_tok * d_out * d_in
            ms = res["w4a16"]
            entry = {"tokens": n_tok, "activations": "fp16" if dt == torch.float16 else "bf16", "ms": round(ms, 4),
                     "dense_cublas_ms": round(res["bf16_dense_cublas"], 4),
                     "speedup_vs_dense": round(res["bf16_dense_cublas"] / ms, 3),
                     "gbs": round(byts / (ms * 1e-3) / 1e9, 1), "hbm_frac": round(byts / (ms * 1e-3) / 1e9 / hbm_, 4),
                     "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
                     "tensor_frac": round(flops / (ms * 1e-3) / 1e12 / tc_, 4),
                     "algorithmic_bytes": int(byts), "flops": flops}
            entry["bound"] = "hbm" if flops / byts < tc_ * 1e12 / (hbm_ * 1e9) else "tensor"
            w4[label] = entry
            del wsw, Yw, Xp
        w4["note"] = ("awq_w4a16_gemm on this layer's packed weights (s_best), activations folded by "
                      "awq_fold_inv_scales; " + str(KB) + " runs each, L2 flushed; cuBLAS dense GEMM of the "
                      "same activation type on the unquantised W for context")
        del Xp_all, pk, W16

    peaks = load_peaks()
    n_a = wl.n_alpha
    flops_direct = 2.0 * n_a * d_out * d_in * N
    tri = tri_macs_per_row(d_in)
    flops_search = flops_direct if form == "direct" else 2.0 * n_a * d_out * tri
    flops_gram = 0.0 if form == "direct" else 2.0 * N * tri
    c_ms = breakdown["contraction"]
    achieved_tflops = flops_search / (c_ms * 1e-3) / 1e12
    peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    # a step of tens of milliseconds repeated for the timed region runs under the
    # power cap: the sustained peak is its denominator; short steps run at full
    # clock against the burst peak (the other fraction is reported beside it)
    long_step = ms_per_step >= LONG_STEP_MS
    peak = peak_sustained if long_step else peak_burst
    stats_bytes = N * d_in * 2 + d_in * 4
    pack_bytes = d_out * d_in * 2 + d_out * d_in // 2 + 2 * 2 * d_out * (d_in // wl.group) + d_in * 4
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    stats_gbs = stats_bytes / (step_split["stats"] * 1e-3) / 1e9
    pack_gbs = pack_bytes / (step_split["pack"] * 1e-3) / 1e9

    line = {
        "metric": METRIC,
        "value": round(world * n_a / (ms_per_step * 1e-3), 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "ms_per_step_eager": round(eager_total_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(wl, world),
        "form": form,
        "timing": graph_note,
        "roofline": {"kernel": "gemm_pair_bf16_tcgen05 (CTA pairs, " + ("direct, sum-of-squares epilogue)" if form == "direct"
                                                                 else "block-triangular Gram, dot epilogue)"),
                     "bound": "tensor", "achieved": round(achieved_tflops, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved_tflops / peak, 4),
                     "peak_kind": (f"bf16 dense sustained ({peaks.get('source')}; step >= {LONG_STEP_MS} ms)"
                                   if long_step else f"bf16 dense burst ({peaks.get('source')})"),
                     "frac_of_burst": round(achieved_tflops / peak_burst, 4),
                     "frac_of_sustained": round(achieved_tflops / peak_sustained, 4),
                     "traffic": profiled_traffic(wl.key, form),
                     "algorithmic_flops_per_launch": flops_search},
        "step_ms": step_split,
        "breakdown_ms": breakdown,
        "breakdown_note": "breakdown_ms: each step entry point timed alone (no overlap), " + str(KB) + " steps",
        "stats_gbs": round(stats_gbs, 1), "stats_hbm_frac": round(stats_gbs / hbm, 4),
        "pack_gbs": round(pack_gbs, 1), "pack_hbm_frac": round(pack_gbs / hbm, 4),
        "gram_tflops": round(flops_gram / (breakdown["gram"] * 1e-3) / 1e12, 2) if flops_gram else None,
        "candidate_weight_evals_per_s": round(world * n_a * d_out * d_in / (ms_per_step * 1e-3), 1),
        "layers_per_s": round(world / (ms_per_step * 1e-3), 3),
        "e2e": {"value": round(world * n_a * K / (e2e_total * 1e-3), 2), "unit": UNIT,
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        "group_clip": gclip,
        "w4a16": w4,
        "e2e_note": "each step: H2D of W and X from pinned memory, the search and pack, D2H of every result; "
                    "step k+1's inputs are copied on a second stream while step k computes; working set "
                    "(the candidate stack) larger than L2, no flush",
        "parity": parity,
        "gpu_launches": launches_per_step(form, n_a, d_in, N) * K,
        "clocks": clk,
        "wall_s_timed_region": round(t_wall, 3),
    }
    return line, (Wb, Xb)


# ----------------------------------------------------------------------------- one entry point alone
ONLY = ("stats", "pack", "fake_quant", "gram", "contract", "group_clip", "fold", "per_tensor", "segmented", "w4a16")


def run_only(args):
    """One entry point of the library alone on the workload's shapes (for
    per-kernel timing and for single-kernel profiler captures): `--steps`
    timed calls after `--warmup` untimed ones, L2 flushed before each, CUDA
    events around each call on the launching stream. W and X come from the
    workload's generator; where the call needs scale vectors that the search
    would produce, it gets s = (a / mean a)^0.4 computed from the workload's
    statistics (a vector of the search's form; the time does not depend on
    which one). The JSON line gives the median time and the call's rate
    against its roofline."""
    import torch
    import weight_only_int4_act_b200 as awq
    from weight_only_int4_act_b200 import binding as B
    from awq_inputs import gen

    import ctypes
    wl = WORKLOADS[args.config]
    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    what = args.only
    d_out, d_in, N = wl.d_out, wl.d_in, wl.N
    ng = d_in // wl.group
    cfg = awq.make_cfg(wl.bits, wl.group, wl.symmetric, wl.n_alpha)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    tokens = args.tokens if what == "w4a16" else N
    W = bf16(gen.make_weight(wl.seed, d_out, d_in, wl.w_std))
    X = bf16(gen.make_activations(wl.seed, tokens, d_in, wl.x_kind, wl.x_lognormal_sigma, wl.outlier_count,
                                  wl.outlier_factor))
    a = awq.act_stats(X)
    s = ((a / a.mean()).clamp_min(1e-4) ** 0.4).contiguous()
    note, byts, flops, kernels = "", None, None, []
    keep = []  # buffers the timed call uses
    err_ws = []  # of those, the workspaces with a device error word (all but the pack's)

    if what == "stats":
        ws = awq.workspace(awq.stats_workspace_size(N, d_in))
        keep.append(ws)
        err_ws.append(ws)
        fn = lambda: awq.act_stats(X, ws, out=a)  # noqa: E731
        byts = N * d_in * 2 + d_in * 4
        kernels = ["act_absmean_partial", "act_absmean_final"]
    elif what in ("pack", "per_tensor"):
        del X
        pcfg = cfg if what == "pack" else awq.make_cfg(wl.bits, 0, wl.symmetric, 1)
        shape = (d_out, ng) if what == "pack" else (1, 1)
        outs = (torch.empty((d_out, d_in // 8), dtype=torch.int32, device=dev),
                torch.empty(shape, dtype=torch.float16, device=dev), torch.empty(shape, dtype=torch.float16, device=dev))
        ws = awq.workspace(max(awq.pack_workspace_size(d_out, d_in, pcfg), 256)) if what == "per_tensor" else None
        keep += [outs, ws]
        fn = lambda: awq.quantize_pack(W, s, pcfg, outputs=outs, ws=ws)  # noqa: E731
        byts = d_out * d_in * 2 + d_out * d_in // 2 + d_in * 4 + (4 * d_out * ng if what == "pack" else d_out * d_in * 2)
        kernels = ["quantize_pack"] if what == "pack" else ["col_minmax", "tensor_extremes", "quantize_pack"]
        if what == "per_tensor":
            note = "per tensor (group 0): W is read twice (extremes, then the pack)"
    elif what in ("fake_quant", "gram", "contract"):
        ws = awq.workspace(awq.search_workspace_size(d_out, d_in, N, cfg))
        keep.append(ws)
        err_ws.append(ws)
        awq.search_scales(W, X, a, cfg, ws=ws)
        L, cptr, st = B.lib(), ctypes.byref(cfg), B._stream()
        wsp, wsn = ctypes.c_void_p(ws.data_ptr()), ws.numel()
        form = awq.search_form(d_out, d_in, N, cfg)
        tri = tri_macs_per_row(d_in)
        if what == "fake_quant":
            fn = lambda: B._check(L.awq_step_fake_quant(ctypes.c_void_p(W.data_ptr()), d_out, d_in, N, cptr, wsp,  # noqa: E731
                                                        wsn, st), "fq")
            byts = d_out * d_in * 2 + wl.n_alpha * d_out * d_in * 2
            kernels = ["fake_quant_delta"]
        elif what == "gram":
            if form != "gram":
                raise SystemExit(f"{wl.key} runs the direct form: no Gram product")
            fn = lambda: B._check(L.awq_step_gram(ctypes.c_void_p(X.data_ptr()), d_out, d_in, N, cptr, wsp, wsn, st),  # noqa: E731
                                  "gram")
            flops = 2.0 * N * tri
            kernels = ["gemm_pair_bf16_tcgen05 (EPI_STORE, MN-major, lower block triangle)", "gram_tail_fixup"]
        else:
            fn = lambda: B._check(L.awq_step_contract(ctypes.c_void_p(X.data_ptr()), d_out, d_in, N, cptr, wsp,  # noqa: E731
                                                      wsn, st), "contract")
            flops = 2.0 * wl.n_alpha * d_out * (tri if form == "gram" else d_in * N)
            kernels = [f"gemm_pair_bf16_tcgen05 ({form} form)"]
    elif what == "group_clip":
        ccfg = awq.make_cfg(wl.bits, wl.group, wl.symmetric, len(GROUP_CLIPS))
        ws = awq.workspace(awq.group_clip_workspace_size(d_out, d_in, N, ccfg))
        keep.append(ws)
        err_ws.append(ws)
        fn = lambda: awq.search_group_clip(W, X, s, GROUP_CLIPS, ccfg, ws=ws)  # noqa: E731
        flops = 2.0 * N * 256 * d_in + 2.0 * len(GROUP_CLIPS) * d_out * 256 * d_in
        kernels = ["repeat_scales", "fake_quant_delta", "gemm_bf16_tcgen05 (EPI_STORE, TRI_DIAG_STORE)",
                   "gemm_bf16_tcgen05 (EPI_DOT32, TRI_DIAG)", "group_clip_argmin"]
        note = f"{len(GROUP_CLIPS)} clip ratios; flops are those issued (the diagonal 256-blocks)"
    elif what == "fold":
        Xt = X.t().contiguous()  # [d_in, N]: channel on the first axis, as a producer's weight
        del X
        keep.append(Xt)
        fn = lambda: awq.fold_inv_scales(s, Xt)  # noqa: E731
        byts = 4 * N * d_in + 4 * d_in
        kernels = ["fold_inv_scales_kernel"]
        note = "in place on a [d_in, N] bf16 parameter"
    elif what == "segmented":
        seg = [d_out // 3, d_out // 3, d_out - 2 * (d_out // 3)]
        ws = awq.workspace(awq.search_workspace_size(d_out, d_in, N, cfg))
        keep.append(ws)
        err_ws.append(ws)
        fn = lambda: awq.search_scales_segmented(W, X, a, cfg, seg, ws=ws)  # noqa: E731
        kernels = ["candidate_scales", "fake_quant_delta", "gemm (Gram / contraction)", "row_loss_rows", "segment_loss_reduce",
                   "segment_argmin"]
        note = f"three layers of {seg} rows sharing X"
    elif what == "w4a16":
        dt = torch.float16 if args.dtype == "f16" else torch.bfloat16
        pk = awq.quantize_pack(W, torch.ones(d_in, dtype=torch.float32, device=dev), cfg)
        Xp = X.to(dt).contiguous()
        wsw = awq.workspace(awq.w4a16_workspace_size(tokens, d_out, d_in, cfg))
        Y = torch.empty((tokens, d_out), dtype=dt, device=dev)
        keep += [pk, Xp, wsw, Y]
        err_ws.append(wsw)
        fn = lambda: awq.w4a16_gemm(Xp, *pk, cfg, ws=wsw, out=Y)  # noqa: E731
        byts = d_out * d_in // 2 + 4 * d_out * ng + tokens * (d_in + d_out) * 2
        flops = 2.0 * tokens * d_out * d_in
        kernels = ["w4a16_gemm_tcgen05", "w4a16_streamk_reduce"]
        note = f"{tokens} tokens, {args.dtype} activations, W packed at s = 1"
    else:
        raise SystemExit(f"unknown --only {what}")

    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    ms = []
    for k in range(args.steps):
        flush.fill_(k & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        e1.synchronize()
        ms.append(e0.elapsed_time(e1))
    for t in err_ws:  # workspaces that carry the device error word
        awq.workspace_error(t)
    t = float(np.median(ms))
    line = {"metric": f"{what} alone", "value": round(t, 4), "unit": "ms", "higher_is_better": False,
            "steps": args.steps, "warmup": args.warmup, "kernels": kernels,
            "config": {"workload": f"{wl.key}: {wl.title}", "d_out": d_out, "d_in": d_in,
                       "N": tokens, "bits": wl.bits, "group": wl.group, "symmetric": wl.symmetric,
                       "l2": "flushed before each call"}}
    if byts is not None:
        line["gbs"] = round(byts / (t * 1e-3) / 1e9, 1)
        line["hbm_frac"] = round(byts / (t * 1e-3) / 1e9 / peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]), 4)
        line["algorithmic_bytes"] = int(byts)
    if flops is not None:
        line["tflops"] = round(flops / (t * 1e-3) / 1e12, 2)
        line["tensor_frac"] = round(flops / (t * 1e-3) / 1e12 / peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]), 4)
        line["flops"] = flops
    if note:
        line["note"] = note
    return line


# ----------------------------------------------------------------------------- CPU oracle
ORACLE_ROW_COST_S = 7e-10  # single-thread oracle seconds per row per (d_in * N), 20 alphas (measured)
REF_STEP_S = 1.2  # oracle arm: single-thread seconds of work per step (100 + 10 steps in about 2-3 minutes)


def ref_sample(wl, seconds):
    """Rows and search tokens of the oracle arm's step: the rows of
    sample_rows; where the minimum of 8 rows over all tokens would still take
    longer than ``seconds``, the search runs over a token slice (a multiple of
    1024) sized to it."""
    rows = sample_rows(wl, seconds)
    per_token = ORACLE_ROW_COST_S * wl.d_in * rows
    tokens = int(min(wl.N, max(1024, seconds / per_token)))
    return rows, (tokens // 1024 * 1024 if tokens < wl.N else wl.N)


def sample_rows(wl, seconds):
    """Rows of W whose search by the single-thread oracle takes about
    ``seconds`` (the cost per row grows with d_in * N): a multiple of 8, at
    least 8, at most d_out."""
    rows = int(seconds / (ORACLE_ROW_COST_S * wl.d_in * wl.N)) // 8 * 8
    return int(min(wl.d_out, max(8, rows)))


def oracle_sample(wl, Wb, Xb, rows, r0=0, tokens=None, a_full=None, block=256, search_tokens=None):
    """Time the CPU oracle, as it stands, on a bounded sample of one layer:
    the statistics over ``tokens`` tokens (all by default), the search of
    ``rows`` rows starting at r0 over every alpha and ``search_tokens``
    tokens (all by default), and their pack; scaled to the whole layer by
    tokens and rows (the statistics' cost is linear in tokens, the search's
    in rows times tokens, the pack's in rows). With a token slice the search
    reads ``a_full``, the statistics of all tokens (computed once by the
    caller). Returns (layer seconds, seconds actually spent)."""
    from oracle import awq_oracle as O
    tokens = wl.N if tokens is None else min(tokens, wl.N)
    search_tokens = wl.N if search_tokens is None else min(search_tokens, wl.N)
    t0 = time.perf_counter()
    a = O.act_stats(Xb[:tokens])
    t_stats = time.perf_counter() - t0
    if tokens < wl.N:
        a = a_full  # the search needs the statistics of all tokens
    Xs = Xb[:search_tokens]
    t_search = t_pack = 0.0
    idx = (r0 + np.arange(rows)) % wl.d_out
    for b0 in range(0, rows, block):
        sel = idx[b0:b0 + block]
        t0 = time.perf_counter()
        res = O.search(Wb, Xs, a, wl.bits, wl.group, wl.symmetric, wl.n_alpha, rows=sel)
        t1 = time.perf_counter()
        O.pack(Wb[sel], res["s_best"], wl.bits, wl.group, wl.symmetric)
        t_pack += time.perf_counter() - t1
        t_search += t1 - t0
    t_layer = (t_stats * (wl.N / tokens) + t_search * (wl.d_out / rows) * (wl.N / search_tokens)
               + t_pack * (wl.d_out / rows))
    return t_layer, t_stats + t_search + t_pack


def single_thread():
    """The oracle is single-threaded: BLAS limited to one thread."""
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=1)


def cpu_baseline_entry(wl, Wb, Xb, rows):
    with single_thread():
        t_layer, spent = oracle_sample(wl, Wb, Xb, rows)
    part = (f"the whole layer ({rows} rows) x {wl.n_alpha} alphas" if rows == wl.d_out else
            f"{rows} of {wl.d_out} rows x {wl.n_alpha} alphas, extrapolated by rows")
    return {"value": round(wl.n_alpha / t_layer, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{wl.key}: statistics of all {wl.N} tokens, search and pack of {part} "
                      f"(float64 numpy, BLAS limited to 1 thread); {spent:.1f} s of CPU work",
            "extrapolated": rows < wl.d_out}


def run_reference(args, wl, world):
    """The oracle arm: each step times the oracle on a bounded sample of the
    layer (statistics over a token slice, search and pack of a row slice over
    all tokens and alphas, the slice moving from step to step), scaled to the
    whole layer; inputs generated once, before the steps."""
    Wb, Xb = make_inputs(wl)
    rows, search_tokens = ref_sample(wl, REF_STEP_S)
    if args.ref_rows:
        rows, search_tokens = args.ref_rows, wl.N
    tokens = min(wl.N, args.ref_tokens)
    K = args.steps
    times, spent = [], []
    with single_thread():
        from oracle import awq_oracle as O
        a_full = O.act_stats(Xb) if tokens < wl.N else None
        for k in range(args.warmup + K):
            t_layer, sp = oracle_sample(wl, Wb, Xb, rows, r0=(k * rows) % wl.d_out, tokens=tokens, a_full=a_full,
                                        search_tokens=search_tokens)
            if k >= args.warmup:
                times.append(t_layer)
                spent.append(sp)
    ms = 1e3 * sum(times) / K
    value = wl.n_alpha / (ms * 1e-3)
    over = "all tokens" if search_tokens == wl.N else f"{search_tokens} of {wl.N} tokens (scaled by tokens)"
    sample = (f"per step: statistics of {tokens} of {wl.N} tokens (scaled by tokens), search of "
              f"{rows} of {wl.d_out} rows x {wl.n_alpha} alphas over {over} and their pack (scaled by rows); "
              f"float64 numpy, BLAS limited to 1 thread")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms, 2), "extrapolated": True,
        "sample_s_per_step": round(float(np.mean(spent)), 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, world),
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="C5", choices=sorted(WORKLOADS),
                    help="workload (default C5, the 70B MLP layer: the largest single-GPU configuration)")
    ap.add_argument("--form", default="auto", choices=["auto", "direct", "gram"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=None,
                    help="rows of W per step of the oracle arm, searched over all tokens (default: about "
                         "REF_STEP_S s of single-thread work, over a token slice where 8 rows would exceed it)")
    ap.add_argument("--ref-tokens", type=int, default=8192, help="tokens of the oracle arm's statistics sample")
    ap.add_argument("--cpu-rows", type=int, default=None,
                    help="rows of W in the CPU baseline's sample (default: about 15 s of single-thread work)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-group-clip", action="store_true", help="skip the per-group clipping pass")
    ap.add_argument("--no-w4a16", action="store_true", help="skip the W4A16 inference-side timing")
    ap.add_argument("--no-graph", action="store_true", help="time the eager public calls only")
    ap.add_argument("--only", default=None, choices=ONLY, help="time one entry point alone (its own JSON line)")
    ap.add_argument("--tokens", type=int, default=16, help="tokens for --only w4a16")
    ap.add_argument("--dtype", default="f16", choices=["f16", "bf16"], help="activations for --only w4a16")
    ap.add_argument("--json-out", default=None, help="also write the JSON line to this file")
    ap.add_argument("--seed", type=int, default=None,
                    help="seed of the synthetic inputs (default: the workload's own; parity then has no stored run)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.seed is not None:  # every reader of WORKLOADS[args.config] below sees the new seed
        import dataclasses
        WORKLOADS[args.config] = dataclasses.replace(WORKLOADS[args.config], seed=args.seed)
    wl = WORKLOADS[args.config]

    def emit(line):
        text = json.dumps(line)
        print(text, flush=True)
        if args.json_out:
            with open(args.json_out, "w") as f:
                f.write(text + "\n")

    if args.only:
        if rank == 0:
            emit(run_only(args))
        return

    if args.impl == "reference":
        if rank == 0:
            emit(run_reference(args, wl, world))
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line, (Wb, Xb) = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                rows = args.cpu_rows if args.cpu_rows is not None else sample_rows(wl, 15.0)
                line["cpu_baseline"] = cpu_baseline_entry(wl, Wb, Xb, rows)
            emit(line)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
