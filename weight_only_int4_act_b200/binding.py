"""Python binding of the C ABI in include/awq.h (ctypes; argument marshalling only).

Every computation runs in the CUDA library; PyTorch only provides device
memory and the current stream. If the library is missing the calls raise:
there is no fallback.

Two builds of the library exist (see _build.py): "release" and "check", the
debug build with index checks. The environment variable AWQ_B200_LIB
(release | check) picks the one loaded at first use; select_library()
switches later calls to the other.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int32, c_int64, c_size_t, c_void_p

from ._build import VARIANTS, lib_path

AWQ_OK = 0
STATUS_NAMES = {
    0: "AWQ_OK", 1: "AWQ_ERR_INVALID_ARG", 2: "AWQ_ERR_SHAPE", 3: "AWQ_ERR_WORKSPACE",
    4: "AWQ_ERR_NONFINITE", 5: "AWQ_ERR_CUDA", 6: "AWQ_ERR_DEVICE", 7: "AWQ_ERR_UNSUPPORTED",
    8: "AWQ_ERR_BOUNDS",
}
AWQ_ERR_BOUNDS = 8
BOUNDS_SITE_SELFTEST = 0x7F
FORMS = {"auto": 0, "direct": 1, "gram": 2}
AWQ_DTYPE_BF16, AWQ_DTYPE_F16 = 0, 1

# every symbol include/awq.h declares
EXPORTED = (
    "awq_status_str", "awq_stats_workspace_size", "awq_act_stats", "awq_search_workspace_size",
    "awq_search_scales", "awq_search_form", "awq_workspace_error", "awq_quantize_pack",
    "awq_step_scales", "awq_step_fake_quant", "awq_step_gram", "awq_step_contract", "awq_step_reduce",
    "awq_debug_copy_dw", "awq_act_stats_noalloc", "awq_search_scales_segmented", "awq_search_candidates",
    "awq_quantize_pack_clipped", "awq_group_clip_workspace_size", "awq_search_group_clip",
    "awq_quantize_pack_group_clip", "awq_fold_inv_scales", "awq_w4a16_workspace_size", "awq_w4a16_gemm",
    "awq_pack_workspace_size", "awq_quantize_pack_ws", "awq_selftest_bounded_wait",
    "awq_bounds_checks_enabled", "awq_bounds_error", "awq_selftest_bounds",
)


class AwqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class QCfg(ctypes.Structure):
    _fields_ = [
        ("bits", c_int32), ("group", c_int32), ("symmetric", c_int32), ("n_alpha", c_int32),
        ("form", c_int32), ("eps_a", c_float), ("alphas", POINTER(c_float)),
    ]


def make_cfg(bits=4, group=128, symmetric=False, n_alpha=20, form="auto", eps_a=1e-4, alphas=None) -> QCfg:
    cfg = QCfg(int(bits), int(group), int(bool(symmetric)), int(n_alpha), FORMS[form], float(eps_a), None)
    if alphas is not None:
        arr = (c_float * len(alphas))(*[float(x) for x in alphas])
        cfg.alphas = ctypes.cast(arr, POINTER(c_float))
        cfg._keep = arr  # keep the host array alive with the struct
    return cfg


_libs = {}
_active = os.environ.get("AWQ_B200_LIB", "release")


def select_library(variant: str) -> str:
    """Route later calls to the given build ("release" or "check"); returns
    the previous choice."""
    global _active
    if variant not in VARIANTS:
        raise ValueError(f"unknown library build {variant!r}; one of {sorted(VARIANTS)}")
    prev, _active = _active, variant
    return prev


def lib() -> ctypes.CDLL:
    """The selected build of the CUDA library (raises if it has not been built)."""
    if _active not in VARIANTS:
        raise ValueError(f"AWQ_B200_LIB={_active!r}; one of {sorted(VARIANTS)}")
    if _active not in _libs:
        path = lib_path(_active)
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library {path} is missing; build it with __graft_entry__.build()")
        L = ctypes.CDLL(path)
        cfgp = POINTER(QCfg)
        sig = {
            "awq_status_str": (c_char_p, [c_int32]),
            "awq_stats_workspace_size": (c_size_t, [c_int64, c_int64]),
            "awq_act_stats": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, c_void_p, c_size_t, c_void_p]),
            "awq_act_stats_noalloc": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, c_void_p]),
            "awq_search_workspace_size": (c_size_t, [c_int64, c_int64, c_int64, cfgp]),
            "awq_search_form": (c_int32, [c_int64, c_int64, c_int64, cfgp]),
            "awq_search_scales": (c_int32, [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64, cfgp,
                                            c_void_p, c_size_t, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
            "awq_search_scales_segmented": (c_int32, [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64, cfgp,
                                                      c_int32, c_void_p, c_void_p, c_size_t, c_void_p, c_void_p,
                                                      c_void_p, c_void_p, c_void_p]),
            "awq_search_candidates": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64,
                                                cfgp, c_void_p, c_size_t, c_void_p, c_void_p, c_void_p, c_void_p,
                                                c_void_p]),
            "awq_quantize_pack_clipped": (c_int32, [c_void_p, c_void_p, c_int64, c_int64, cfgp, c_float, c_void_p,
                                                    c_void_p, c_void_p, c_void_p]),
            "awq_group_clip_workspace_size": (c_size_t, [c_int64, c_int64, c_int64, cfgp]),
            "awq_search_group_clip": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64,
                                                cfgp, c_void_p, c_size_t, c_void_p, c_void_p, c_void_p]),
            "awq_quantize_pack_group_clip": (c_int32, [c_void_p, c_void_p, c_void_p, c_int32, c_void_p, c_int64,
                                                       c_int64, cfgp, c_void_p, c_void_p, c_void_p, c_void_p]),
            "awq_fold_inv_scales": (c_int32, [c_void_p, c_int64, c_void_p, c_int32, c_int64, c_void_p]),
            "awq_w4a16_workspace_size": (c_size_t, [c_int64, c_int64, c_int64, cfgp]),
            "awq_w4a16_gemm": (c_int32, [c_void_p, c_int32, c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64,
                                         cfgp, c_void_p, c_void_p, c_size_t, c_void_p]),
            "awq_pack_workspace_size": (c_size_t, [c_int64, c_int64, cfgp]),
            "awq_quantize_pack_ws": (c_int32, [c_void_p, c_void_p, c_int64, c_int64, cfgp, c_float, c_void_p,
                                               c_size_t, c_void_p, c_void_p, c_void_p, c_void_p]),
            "awq_selftest_bounded_wait": (c_int32, [c_void_p, c_void_p]),
            "awq_bounds_checks_enabled": (c_int32, []),
            "awq_bounds_error": (c_int32, [POINTER(c_int32), c_void_p]),
            "awq_selftest_bounds": (c_int32, [c_void_p, c_size_t, c_void_p]),
            "awq_workspace_error": (c_int32, [c_void_p, c_void_p]),
            "awq_quantize_pack": (c_int32, [c_void_p, c_void_p, c_int64, c_int64, cfgp, c_void_p, c_void_p,
                                            c_void_p, c_void_p]),
            "awq_step_scales": (c_int32, [c_void_p, c_int64, c_int64, c_int64, cfgp, c_void_p, c_size_t, c_void_p]),
            "awq_step_fake_quant": (c_int32, [c_void_p, c_int64, c_int64, c_int64, cfgp, c_void_p, c_size_t,
                                              c_void_p]),
            "awq_step_gram": (c_int32, [c_void_p, c_int64, c_int64, c_int64, cfgp, c_void_p, c_size_t, c_void_p]),
            "awq_step_contract": (c_int32, [c_void_p, c_int64, c_int64, c_int64, cfgp, c_void_p, c_size_t,
                                            c_void_p]),
            "awq_step_reduce": (c_int32, [c_int64, c_int64, c_int64, cfgp, c_void_p, c_size_t, c_void_p, c_void_p,
                                          c_void_p, c_void_p, c_void_p]),
            "awq_debug_copy_dw": (c_int32, [c_void_p, c_int64, c_int64, c_int64, cfgp, c_int32, c_void_p,
                                            c_void_p]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _libs[_active] = L
    return _libs[_active]


def status_str(status: int) -> str:
    return lib().awq_status_str(status).decode()


def _check(status: int, what: str):
    if status != AWQ_OK:
        raise AwqError(status, what)


def _torch():
    import torch
    return torch


def _stream():
    return c_void_p(_torch().cuda.current_stream().cuda_stream)


def _req(t, dtype, shape, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _ptr(t):
    return c_void_p(t.data_ptr()) if t is not None else None


# --------------------------------------------------------------------------- sizes
def stats_workspace_size(N: int, d_in: int) -> int:
    return int(lib().awq_stats_workspace_size(N, d_in))


def search_workspace_size(d_out: int, d_in: int, N: int, cfg: QCfg) -> int:
    return int(lib().awq_search_workspace_size(d_out, d_in, N, ctypes.byref(cfg)))


def search_form(d_out: int, d_in: int, N: int, cfg: QCfg) -> str:
    f = int(lib().awq_search_form(d_out, d_in, N, ctypes.byref(cfg)))
    return {1: "direct", 2: "gram"}.get(f, "invalid")


def workspace(nbytes: int):
    torch = _torch()
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device="cuda")


# --------------------------------------------------------------------------- a1
def act_stats(X, ws=None, out=None):
    """a[i] = mean_t |X[t, i]| for bf16 X [N, d_in] (float32 [d_in])."""
    torch = _torch()
    _req(X, torch.bfloat16, None, "X")
    N, d_in = X.shape
    if ws is None:
        ws = workspace(stats_workspace_size(N, d_in))
    a = out if out is not None else torch.empty(d_in, dtype=torch.float32, device=X.device)
    _check(lib().awq_act_stats(_ptr(X), N, d_in, _ptr(a), _ptr(ws), ws.numel(), _stream()), "awq_act_stats")
    return a


# --------------------------------------------------------------------------- a2-a6
def search_scales(W, X, a, cfg: QCfg, ws=None, row_losses=False, outputs=None):
    """Loss of every alpha, the chosen index and its scales (device tensors).

    Returns dict(losses float32[n_alpha], best int32[1], s_best float32[d_in],
    row_losses float32[n_alpha, d_out] or None, ws)."""
    torch = _torch()
    _req(W, torch.bfloat16, None, "W")
    d_out, d_in = W.shape
    _req(X, torch.bfloat16, None, "X")
    N = X.shape[0]
    if X.shape[1] != d_in:
        raise ValueError("X must have d_in columns")
    _req(a, torch.float32, (d_in,), "a")
    if ws is None:
        ws = workspace(search_workspace_size(d_out, d_in, N, cfg))
    if outputs is None:
        outputs = dict(
            losses=torch.empty(cfg.n_alpha, dtype=torch.float32, device=W.device),
            best=torch.empty(1, dtype=torch.int32, device=W.device),
            s_best=torch.empty(d_in, dtype=torch.float32, device=W.device),
            row_losses=torch.empty((cfg.n_alpha, d_out), dtype=torch.float32, device=W.device) if row_losses else None,
        )
    o = outputs
    _check(lib().awq_search_scales(_ptr(W), _ptr(X), _ptr(a), d_out, d_in, N, ctypes.byref(cfg), _ptr(ws),
                                   ws.numel(), _ptr(o["losses"]), _ptr(o["best"]), _ptr(o["s_best"]),
                                   _ptr(o["row_losses"]), _stream()), "awq_search_scales")
    return dict(o, ws=ws)


def search_scales_segmented(W, X, a, cfg: QCfg, seg_rows, ws=None, row_losses=False):
    """Per-layer search for layers sharing X; W is their row concatenation and
    seg_rows the row count of each layer. Returns dict(losses float32[n_seg,
    n_alpha], best int32[n_seg], s_best float32[n_seg, d_in], row_losses, ws)."""
    torch = _torch()
    _req(W, torch.bfloat16, None, "W")
    d_out, d_in = W.shape
    _req(X, torch.bfloat16, None, "X")
    N = X.shape[0]
    if X.shape[1] != d_in:
        raise ValueError("X must have d_in columns")
    _req(a, torch.float32, (d_in,), "a")
    n_seg = len(seg_rows)
    rows = (ctypes.c_int64 * max(n_seg, 1))(*[int(r) for r in seg_rows])
    if ws is None:
        ws = workspace(search_workspace_size(d_out, d_in, N, cfg))
    o = dict(losses=torch.empty((n_seg, cfg.n_alpha), dtype=torch.float32, device=W.device),
             best=torch.empty(n_seg, dtype=torch.int32, device=W.device),
             s_best=torch.empty((n_seg, d_in), dtype=torch.float32, device=W.device),
             row_losses=torch.empty((cfg.n_alpha, d_out), dtype=torch.float32, device=W.device) if row_losses else None)
    _check(lib().awq_search_scales_segmented(_ptr(W), _ptr(X), _ptr(a), d_out, d_in, N, ctypes.byref(cfg), n_seg,
                                             ctypes.cast(rows, c_void_p), _ptr(ws), ws.numel(), _ptr(o["losses"]),
                                             _ptr(o["best"]), _ptr(o["s_best"]), _ptr(o["row_losses"]), _stream()),
           "awq_search_scales_segmented")
    return dict(o, ws=ws)


def search_candidates(W, X, s_cand, cfg: QCfg, clips=None, ws=None, row_losses=False):
    """Losses of explicit candidates: scale vectors s_cand float32 [n, d_in] (CUDA)
    and optional clip ratios (host sequence of n floats in (0, 1]); n must equal
    cfg.n_alpha. Returns dict(losses, best, s_best, row_losses, ws)."""
    torch = _torch()
    _req(W, torch.bfloat16, None, "W")
    d_out, d_in = W.shape
    _req(X, torch.bfloat16, None, "X")
    N = X.shape[0]
    _req(s_cand, torch.float32, (cfg.n_alpha, d_in), "s_cand")
    carr = None
    if clips is not None:
        if len(clips) != cfg.n_alpha:
            raise ValueError("need one clip ratio per candidate")
        carr = (c_float * len(clips))(*[float(c) for c in clips])
    if ws is None:
        ws = workspace(search_workspace_size(d_out, d_in, N, cfg))
    o = dict(losses=torch.empty(cfg.n_alpha, dtype=torch.float32, device=W.device),
             best=torch.empty(1, dtype=torch.int32, device=W.device),
             s_best=torch.empty(d_in, dtype=torch.float32, device=W.device),
             row_losses=torch.empty((cfg.n_alpha, d_out), dtype=torch.float32, device=W.device) if row_losses else None)
    _check(lib().awq_search_candidates(_ptr(W), _ptr(X), _ptr(s_cand), ctypes.cast(carr, c_void_p) if carr else None,
                                       d_out, d_in, N, ctypes.byref(cfg), _ptr(ws), ws.numel(), _ptr(o["losses"]),
                                       _ptr(o["best"]), _ptr(o["s_best"]), _ptr(o["row_losses"]), _stream()),
           "awq_search_candidates")
    return dict(o, ws=ws)


def group_clip_workspace_size(d_out, d_in, N, cfg: QCfg) -> int:
    return int(lib().awq_group_clip_workspace_size(d_out, d_in, N, ctypes.byref(cfg)))


def _clip_array(clips, n):
    if len(clips) != n:
        raise ValueError("need one clip ratio per candidate")
    return (c_float * n)(*[float(c) for c in clips])


def search_group_clip(W, X, s, clips, cfg: QCfg, ws=None, group_err=False):
    """Per-(row, group) clip choice with the scales s fixed: clips is a host
    sequence of cfg.n_alpha ratios. Returns dict(best_clip uint8 [d_out, d_in/g],
    group_err float32 [n, d_out, d_in/g] or None, ws)."""
    torch = _torch()
    _req(W, torch.bfloat16, None, "W")
    d_out, d_in = W.shape
    _req(X, torch.bfloat16, None, "X")
    N = X.shape[0]
    _req(s, torch.float32, (d_in,), "s")
    carr = _clip_array(clips, cfg.n_alpha)
    if ws is None:
        ws = workspace(group_clip_workspace_size(d_out, d_in, N, cfg))
    ng = d_in // cfg.group if cfg.group > 0 else 0
    o = dict(best_clip=torch.empty((d_out, ng), dtype=torch.uint8, device=W.device),
             group_err=torch.empty((cfg.n_alpha, d_out, ng), dtype=torch.float32, device=W.device)
             if group_err else None)
    _check(lib().awq_search_group_clip(_ptr(W), _ptr(X), _ptr(s), ctypes.cast(carr, c_void_p), d_out, d_in, N,
                                       ctypes.byref(cfg), _ptr(ws), ws.numel(), _ptr(o["best_clip"]),
                                       _ptr(o["group_err"]), _stream()), "awq_search_group_clip")
    return dict(o, ws=ws)


def quantize_pack_group_clip(W, s, clips, best_clip, cfg: QCfg, outputs=None):
    """quantize_pack with group j of row r clipped at clips[best_clip[r, j]]."""
    torch = _torch()
    _req(W, torch.bfloat16, None, "W")
    d_out, d_in = W.shape
    _req(s, torch.float32, (d_in,), "s")
    ng = d_in // cfg.group if cfg.group > 0 else 0
    _req(best_clip, torch.uint8, (d_out, ng), "best_clip")
    carr = _clip_array(clips, len(clips))
    if outputs is None:
        outputs = (torch.empty((d_out, d_in // 8), dtype=torch.int32, device=W.device),
                   torch.empty((d_out, ng), dtype=torch.float16, device=W.device),
                   torch.empty((d_out, ng), dtype=torch.float16, device=W.device))
    q, sc, zr = outputs
    _check(lib().awq_quantize_pack_group_clip(_ptr(W), _ptr(s), ctypes.cast(carr, c_void_p), len(clips),
                                              _ptr(best_clip), d_out, d_in, ctypes.byref(cfg), _ptr(q), _ptr(sc),
                                              _ptr(zr), _stream()), "awq_quantize_pack_group_clip")
    return q, sc, zr


# --------------------------------------------------------------------------- inference side
def _dtype_code(t, name):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return AWQ_DTYPE_BF16
    if t.dtype == torch.float16:
        return AWQ_DTYPE_F16
    raise ValueError(f"{name} must be bfloat16 or float16, got {t.dtype}")


def fold_inv_scales(s, p):
    """In place: row i of p (bf16 or fp16 [d_in] or [d_in, inner], CUDA) becomes p / s_i."""
    torch = _torch()
    _req(s, torch.float32, None, "s")
    dt = _dtype_code(p, "p")
    _req(p, p.dtype, None, "p")
    d_in = s.numel()
    if p.shape[0] != d_in:
        raise ValueError("p must have the channel (length of s) on its first axis")
    inner = p.numel() // d_in if d_in else 0
    _check(lib().awq_fold_inv_scales(_ptr(s), d_in, _ptr(p), dt, inner, _stream()), "awq_fold_inv_scales")
    return p


def w4a16_workspace_size(N, d_out, d_in, cfg: QCfg) -> int:
    return int(lib().awq_w4a16_workspace_size(N, d_out, d_in, ctypes.byref(cfg)))


def w4a16_gemm(Xp, qweight, scales, zeros, cfg: QCfg, ws=None, out=None):
    """Y [N, d_out] = X' ([N, d_in], fp16 or bf16) times the dequantised packed
    weights, in the activations' type."""
    torch = _torch()
    dt = _dtype_code(Xp, "X")
    _req(Xp, Xp.dtype, None, "X")
    N, d_in = Xp.shape
    _req(qweight, torch.int32, None, "qweight")
    d_out = qweight.shape[0]
    if qweight.shape != (d_out, d_in // 8):
        raise ValueError("qweight must be [d_out, d_in/8]")
    ng = d_in // cfg.group if cfg.group > 0 else 0
    _req(scales, torch.float16, (d_out, ng), "scales")
    _req(zeros, torch.float16, (d_out, ng), "zeros")
    if ws is None:
        ws = workspace(max(w4a16_workspace_size(N, d_out, d_in, cfg), 256))
    if out is None:
        out = torch.empty((N, d_out), dtype=Xp.dtype, device=Xp.device)
    _req(out, Xp.dtype, (N, d_out), "out")
    _check(lib().awq_w4a16_gemm(_ptr(Xp), dt, _ptr(qweight), _ptr(scales), _ptr(zeros), N, d_out, d_in,
                                ctypes.byref(cfg), _ptr(out), _ptr(ws), ws.numel(), _stream()), "awq_w4a16_gemm")
    return out


def selftest_bounded_wait(ws):
    """Launch the bounded-wait failure path (see include/awq.h); the error lands in ws."""
    _check(lib().awq_selftest_bounded_wait(_ptr(ws), _stream()), "awq_selftest_bounded_wait")


def bounds_checks_enabled() -> bool:
    """True if the selected build carries the index checks."""
    return bool(lib().awq_bounds_checks_enabled())


def bounds_error():
    """(status, site) of the index checks since the last call; reading clears
    the device word (synchronises). Always (AWQ_OK, 0) in the release build."""
    site = c_int32(0)
    st = int(lib().awq_bounds_error(ctypes.byref(site), _stream()))
    if st not in (AWQ_OK, AWQ_ERR_BOUNDS):
        raise AwqError(st, "awq_bounds_error")
    return st, int(site.value)


def selftest_bounds(ws):
    """Launch the index checks' failure path (see include/awq.h)."""
    _check(lib().awq_selftest_bounds(_ptr(ws), ws.numel() * ws.element_size(), _stream()), "awq_selftest_bounds")


def workspace_error(ws):
    """Raise AwqError if a kernel recorded an error in the workspace (synchronises)."""
    _check(lib().awq_workspace_error(_ptr(ws), _stream()), "device")


def step(name: str, *args):
    """Call one awq_step_* entry point with already-marshalled arguments."""
    fn = getattr(lib(), "awq_step_" + name)
    _check(fn(*args), "awq_step_" + name)


def debug_dw(ws, d_out, d_in, N, cfg, k):
    """bf16 [d_out, d_in] copy of the candidate dW for grid index k."""
    torch = _torch()
    dst = torch.empty((d_out, d_in), dtype=torch.bfloat16, device="cuda")
    _check(lib().awq_debug_copy_dw(_ptr(ws), d_out, d_in, N, ctypes.byref(cfg), k, _ptr(dst), _stream()),
           "awq_debug_copy_dw")
    return dst


# --------------------------------------------------------------------------- a7
def pack_workspace_size(d_out, d_in, cfg: QCfg) -> int:
    return int(lib().awq_pack_workspace_size(d_out, d_in, ctypes.byref(cfg)))


def quantize_pack(W, s, cfg: QCfg, outputs=None, clip=1.0, ws=None):
    """(qweight int32 view of uint32 [d_out, d_in/8], scales fp16 [d_out, d_in/g], zeros fp16 [d_out, d_in/g]);
    per tensor (cfg.group == 0): scales and zeros are [1, 1] and a workspace is used."""
    torch = _torch()
    _req(W, torch.bfloat16, None, "W")
    d_out, d_in = W.shape
    _req(s, torch.float32, (d_in,), "s")
    if outputs is None:
        shape = (d_out, d_in // cfg.group) if cfg.group > 0 else (1, 1)
        outputs = (torch.empty((d_out, d_in // 8), dtype=torch.int32, device=W.device),
                   torch.empty(shape, dtype=torch.float16, device=W.device),
                   torch.empty(shape, dtype=torch.float16, device=W.device))
    q, sc, zr = outputs
    if cfg.group == 0 or ws is not None:
        if ws is None:
            ws = workspace(pack_workspace_size(d_out, d_in, cfg))
        _check(lib().awq_quantize_pack_ws(_ptr(W), _ptr(s), d_out, d_in, ctypes.byref(cfg), float(clip), _ptr(ws),
                                          ws.numel(), _ptr(q), _ptr(sc), _ptr(zr), _stream()), "awq_quantize_pack_ws")
    elif clip == 1.0:
        _check(lib().awq_quantize_pack(_ptr(W), _ptr(s), d_out, d_in, ctypes.byref(cfg), _ptr(q), _ptr(sc), _ptr(zr),
                                       _stream()), "awq_quantize_pack")
    else:
        _check(lib().awq_quantize_pack_clipped(_ptr(W), _ptr(s), d_out, d_in, ctypes.byref(cfg), float(clip), _ptr(q),
                                               _ptr(sc), _ptr(zr), _stream()), "awq_quantize_pack_clipped")
    return q, sc, zr
