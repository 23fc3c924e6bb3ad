"""The C ABI without a GPU: the library loads, exports what include/awq.h
declares, sizes its workspaces on the host, and rejects bad arguments before
touching the device. No test here enqueues GPU work."""
import ctypes
import pathlib
import re

import pytest

import weight_only_int4_act_b200 as awq
from weight_only_int4_act_b200 import binding

HEADER = pathlib.Path(__file__).resolve().parents[1] / "include" / "awq.h"
FAKE = ctypes.c_void_p(0x10000)  # aligned, never dereferenced: every call below fails validation first


def declared_symbols():
    text = HEADER.read_text()
    return sorted(set(re.findall(r"\b(awq_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(params=["release", "check"])
def build_lib(request):
    """The ctypes library of one build; the binding's choice is restored after."""
    prev = binding.select_library(request.param)
    try:
        yield request.param, awq.lib()
    finally:
        binding.select_library(prev)


def test_header_declarations_match_exports(build_lib):
    _, lib = build_lib
    names = declared_symbols()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), f"{n} declared in awq.h but not exported"
    assert sorted(binding.EXPORTED) == names


def test_bounds_entry_points_without_gpu(build_lib):
    """Which build carries the index checks, and the checks' entry points up
    to the point where they would need the device."""
    variant, lib = build_lib
    assert lib.awq_bounds_checks_enabled() == (1 if variant == "check" else 0)
    assert lib.awq_selftest_bounds(None, 256, None) == 1  # AWQ_ERR_INVALID_ARG
    assert lib.awq_selftest_bounds(ctypes.c_void_p(0x10010), 256, None) == 1  # not 256-byte aligned
    assert lib.awq_selftest_bounds(FAKE, 64, None) == 3  # AWQ_ERR_WORKSPACE
    if variant == "release":
        # nothing to read back and no self-test to launch
        site = ctypes.c_int32(5)
        assert lib.awq_bounds_error(ctypes.byref(site), None) == 0 and site.value == 0
        assert lib.awq_selftest_bounds(FAKE, 256, None) == 7  # AWQ_ERR_UNSUPPORTED, nothing launched


def test_status_strings():
    for s in range(9):
        txt = awq.status_str(s)
        assert txt.startswith(binding.STATUS_NAMES[s])
    assert awq.status_str(99) == "AWQ_ERR_UNKNOWN"


def test_workspace_sizes_and_form():
    cfg = awq.make_cfg(4, 128, False, 20)
    # C2 shape: the stack of 20 x 4096 x 4096 bf16 dominates; N = d_in, so the
    # block-triangular Gram form needs about half the multiply-adds of the direct one
    n = awq.search_workspace_size(4096, 4096, 4096, cfg)
    assert n >= 20 * 4096 * 4096 * 2
    assert awq.search_form(4096, 4096, 4096, cfg) == "gram"
    assert awq.search_form(4096, 4096, 1024, cfg) == "direct"
    assert awq.search_form(11008, 4096, 16384, cfg) == "gram"
    assert awq.search_form(28672, 8192, 65536, cfg) == "gram"
    assert awq.search_form(4096, 11008, 16384, awq.make_cfg(3, 64, True, 20)) == "gram"
    assert awq.search_form(256, 512, 256, cfg) == "direct"
    forced = awq.make_cfg(4, 128, False, 20, form="gram")
    assert awq.search_form(256, 512, 256, forced) == "gram"
    assert awq.search_workspace_size(256, 512, 256, forced) > awq.search_workspace_size(256, 512, 256, cfg)
    # ragged rows pad to 128
    assert awq.search_workspace_size(200, 512, 256, cfg) == awq.search_workspace_size(256, 512, 256, cfg)
    assert awq.stats_workspace_size(65536, 8192) > 0
    # invalid configurations size to 0
    assert awq.search_workspace_size(256, 500, 256, cfg) == 0
    assert awq.search_workspace_size(256, 512, 0, cfg) == 0
    assert awq.stats_workspace_size(0, 512) == 0


@pytest.mark.parametrize("field,value", [
    ("bits", 1), ("bits", 5), ("group", 96), ("group", 4), ("group", 512), ("symmetric", 2),
    ("n_alpha", 0), ("n_alpha", 65), ("form", 3),
])
def test_bad_config_rejected(field, value):
    cfg = awq.make_cfg(4, 128, False, 20)
    setattr(cfg, field, value)
    lib = awq.lib()
    st = lib.awq_search_scales(FAKE, FAKE, FAKE, 256, 512, 256, ctypes.byref(cfg), FAKE, 1 << 40,
                               FAKE, FAKE, FAKE, None, None)
    assert st == 1  # AWQ_ERR_INVALID_ARG
    assert awq.search_workspace_size(256, 512, 256, cfg) == 0


def test_bad_alpha_grid_rejected():
    cfg = awq.make_cfg(4, 128, False, 3, alphas=[0.0, 0.5, 1.5])
    assert awq.search_workspace_size(256, 512, 256, cfg) == 0


def test_shape_and_pointer_errors():
    lib = awq.lib()
    cfg = awq.make_cfg(4, 128, False, 20)
    c = ctypes.byref(cfg)
    big = 1 << 40
    # d_in not a multiple of the group
    assert lib.awq_search_scales(FAKE, FAKE, FAKE, 256, 500, 256, c, FAKE, big, FAKE, FAKE, FAKE, None, None) == 2
    # no tokens / no rows
    assert lib.awq_search_scales(FAKE, FAKE, FAKE, 256, 512, 0, c, FAKE, big, FAKE, FAKE, FAKE, None, None) == 2
    assert lib.awq_search_scales(FAKE, FAKE, FAKE, 0, 512, 256, c, FAKE, big, FAKE, FAKE, FAKE, None, None) == 2
    # null pointers
    assert lib.awq_search_scales(None, FAKE, FAKE, 256, 512, 256, c, FAKE, big, FAKE, FAKE, FAKE, None, None) == 1
    assert lib.awq_search_scales(FAKE, FAKE, FAKE, 256, 512, 256, c, None, big, FAKE, FAKE, FAKE, None, None) == 1
    assert lib.awq_search_scales(FAKE, FAKE, FAKE, 256, 512, 256, c, FAKE, big, None, FAKE, FAKE, None, None) == 1
    # misaligned pointers
    odd = ctypes.c_void_p(0x10002)
    assert lib.awq_search_scales(odd, FAKE, FAKE, 256, 512, 256, c, FAKE, big, FAKE, FAKE, FAKE, None, None) == 1
    assert lib.awq_search_scales(FAKE, FAKE, FAKE, 256, 512, 256, c, odd, big, FAKE, FAKE, FAKE, None, None) == 1
    # workspace too small
    need = awq.search_workspace_size(256, 512, 256, cfg)
    assert lib.awq_search_scales(FAKE, FAKE, FAKE, 256, 512, 256, c, FAKE, need - 1, FAKE, FAKE, FAKE, None,
                                 None) == 3
    # stats
    assert lib.awq_act_stats(None, 16, 512, FAKE, FAKE, big, None) == 1
    assert lib.awq_act_stats(FAKE, 0, 512, FAKE, FAKE, big, None) == 2
    assert lib.awq_act_stats(FAKE, 16, 500, FAKE, FAKE, big, None) == 2
    assert lib.awq_act_stats(FAKE, 16, 512, FAKE, FAKE, 8, None) == 3
    # pack
    assert lib.awq_quantize_pack(FAKE, FAKE, 256, 500, c, FAKE, FAKE, FAKE, None) == 2
    assert lib.awq_quantize_pack(FAKE, None, 256, 512, c, FAKE, FAKE, FAKE, None) == 1
    # workspace error read-back needs a workspace
    assert lib.awq_workspace_error(None, None) == 1


def test_python_binding_refuses_cpu_tensors():
    import torch
    X = torch.zeros((4, 16), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        awq.act_stats(X)


def test_segmented_search_validation():
    lib = awq.lib()
    cfg = awq.make_cfg(4, 128, False, 20)
    c = ctypes.byref(cfg)
    big = 1 << 40

    def call(rows, d_out=256):
        arr = (ctypes.c_int64 * max(len(rows), 1))(*rows)
        return lib.awq_search_scales_segmented(FAKE, FAKE, FAKE, d_out, 512, 256, c, len(rows), ctypes.cast(arr, ctypes.c_void_p),
                                               FAKE, big, FAKE, FAKE, FAKE, None, None)
    assert call([]) == 1                      # n_seg < 1
    assert call([16] * 17, d_out=272) == 1    # n_seg > 16
    assert call([100, 100]) == 2              # rows do not sum to d_out
    assert call([200, 100]) == 2              # overshoot
    assert call([256, 0]) == 2                # empty layer
    assert lib.awq_search_scales_segmented(FAKE, FAKE, FAKE, 256, 512, 256, c, 1, None, FAKE, big, FAKE, FAKE, FAKE,
                                           None, None) == 1


def test_group_clip_validation():
    lib = awq.lib()
    big = 1 << 40
    cfg = awq.make_cfg(4, 128, False, 4)
    c = ctypes.byref(cfg)
    clips = (ctypes.c_float * 4)(1.0, 0.9, 0.8, 0.7)
    cp = ctypes.cast(clips, ctypes.c_void_p)
    need = awq.group_clip_workspace_size(256, 512, 256, cfg)
    # the candidate stack of 4 x 256 x 512 bf16 and the 512 x 256 diagonal blocks of G
    assert need >= 4 * 256 * 512 * 2 + 512 * 256 * 2
    assert awq.group_clip_workspace_size(200, 512, 256, cfg) == need  # rows pad to 128
    assert awq.group_clip_workspace_size(256, 512, 256, awq.make_cfg(4, 16, False, 4)) == 0  # g < 32

    def call(cfg_=cfg, clips_=cp, ws_bytes=big, best=FAKE, d_in=512):
        return lib.awq_search_group_clip(FAKE, FAKE, FAKE, clips_, 256, d_in, 256, ctypes.byref(cfg_), FAKE,
                                         ws_bytes, best, None, None)
    assert call(cfg_=awq.make_cfg(4, 16, False, 4)) == 7          # AWQ_ERR_UNSUPPORTED
    assert call(ws_bytes=need - 1) == 3                           # AWQ_ERR_WORKSPACE
    assert call(best=None) == 1
    assert call(clips_=None) == 1
    assert call(d_in=500) == 2
    bad = (ctypes.c_float * 4)(1.0, 0.9, 1.5, 0.7)
    assert call(clips_=ctypes.cast(bad, ctypes.c_void_p)) == 1
    # pack with a clip per group
    pk = lib.awq_quantize_pack_group_clip
    assert pk(FAKE, FAKE, None, 4, FAKE, 256, 512, c, FAKE, FAKE, FAKE, None) == 1
    assert pk(FAKE, FAKE, cp, 0, FAKE, 256, 512, c, FAKE, FAKE, FAKE, None) == 1
    assert pk(FAKE, FAKE, cp, 65, FAKE, 256, 512, c, FAKE, FAKE, FAKE, None) == 1
    assert pk(FAKE, FAKE, cp, 4, None, 256, 512, c, FAKE, FAKE, FAKE, None) == 1
    assert pk(FAKE, FAKE, ctypes.cast(bad, ctypes.c_void_p), 4, FAKE, 256, 512, c, FAKE, FAKE, FAKE, None) == 1
    assert pk(FAKE, FAKE, cp, 4, FAKE, 256, 500, c, FAKE, FAKE, FAKE, None) == 2


def test_w4a16_and_fold_validation():
    lib = awq.lib()
    big = 1 << 40
    cfg = awq.make_cfg(4, 128, False, 1)
    c = ctypes.byref(cfg)
    # decode shape: few output tiles, so K is split and the workspace holds fp32 partials
    small = awq.w4a16_workspace_size(1, 256, 4096, cfg)
    assert small > 1024 + 256 * 4
    assert awq.w4a16_workspace_size(4096, 4096, 4096, cfg) == 1024  # enough tiles: no split, error word only
    assert awq.w4a16_workspace_size(16, 256, 4112, cfg) == 0      # d_in not a multiple of 32 / of g
    assert awq.w4a16_workspace_size(16, 256, 4096, awq.make_cfg(5, 128, False, 1)) == 0
    assert awq.w4a16_workspace_size(0, 256, 4096, cfg) == 0

    def call(X=FAKE, q=FAKE, sc=FAKE, zr=FAKE, N=1, d_out=256, d_in=4096, cfg_=cfg, Y=FAKE, ws=FAKE, wsb=big, dt=0):
        return lib.awq_w4a16_gemm(X, dt, q, sc, zr, N, d_out, d_in, ctypes.byref(cfg_), Y, ws, wsb, None)
    assert call(d_in=4000) == 2
    assert call(N=0) == 2
    assert call(cfg_=awq.make_cfg(4, 96, False, 1)) == 1
    assert call(cfg_=awq.make_cfg(4, 0, False, 1)) == 1   # the per-tensor layout is not read by this kernel
    assert awq.w4a16_workspace_size(16, 256, 4096, awq.make_cfg(4, 0, False, 1)) == 0
    assert call(X=None) == 1
    assert call(Y=None) == 1
    assert call(ws=None) == 1
    assert call(X=ctypes.c_void_p(0x10008)) == 1   # activations must be 16-byte aligned (TMA)
    assert call(wsb=small - 1) == 3
    assert call(dt=2) == 1                          # activation type: 0 bf16, 1 fp16
    assert call(dt=1, wsb=small - 1) == 3
    # fold
    assert lib.awq_fold_inv_scales(None, 16, FAKE, 0, 1, None) == 1
    assert lib.awq_fold_inv_scales(FAKE, 16, FAKE, 2, 1, None) == 1
    assert lib.awq_fold_inv_scales(FAKE, 0, FAKE, 1, 1, None) == 2
    assert lib.awq_fold_inv_scales(FAKE, 16, FAKE, 0, 0, None) == 2


def test_per_tensor_validation():
    lib = awq.lib()
    big = 1 << 40
    cfg = awq.make_cfg(4, 0, True, 20)
    assert awq.search_workspace_size(256, 512, 256, cfg) > 0
    assert awq.search_workspace_size(256, 520, 256, cfg) == 0          # d_in % 16 for one step per layer
    assert awq.pack_workspace_size(256, 512, cfg) >= 2 * 512 * 4
    c = ctypes.byref(cfg)
    # the pack without a workspace cannot take the layer-wide extremes
    assert lib.awq_quantize_pack(FAKE, FAKE, 256, 512, c, FAKE, FAKE, FAKE, None) == 3
    need = awq.pack_workspace_size(256, 512, cfg)
    assert lib.awq_quantize_pack_ws(FAKE, FAKE, 256, 512, c, 1.0, FAKE, need - 1, FAKE, FAKE, FAKE, None) == 3
    # one step per layer does not apply to concatenated layers, per-group clipping or the W4A16 product
    arr = (ctypes.c_int64 * 2)(128, 128)
    assert lib.awq_search_scales_segmented(FAKE, FAKE, FAKE, 256, 512, 256, c, 2, ctypes.cast(arr, ctypes.c_void_p),
                                           FAKE, big, FAKE, FAKE, FAKE, None, None) == 7
    assert awq.group_clip_workspace_size(256, 512, 256, cfg) == 0
    assert awq.w4a16_workspace_size(16, 256, 512, cfg) == 0


# ---------------------------------------------------------------- W4A16 work split (host plan)
def _w4_split(N, d_out, d_in, group, ctas=148):
    """The W4A16 plan's work split, restated: 128-row tiles of bn tokens,
    K steps of 256 channels at decode widths (bn <= 64, g > 8) else 128;
    with fewer than two waves of tiles, G = min(ctas, units // 4) equal
    ranges of the tile-major (tile, K step) units. Returns (segments per
    CTA, slots, G): a segment is (tile, k0, k1, slab, whole)."""
    bn = next(b for b in (16, 32, 64, 128, 256) if N <= b) if N <= 256 else 256
    bk = 256 if bn <= 64 and group > 8 else 128
    tiles = -(-d_out // 128) * -(-N // bn)
    n_kb = -(-d_in // bk)
    units = tiles * n_kb
    if not (tiles < 2 * ctas and n_kb > 1):
        return None, 1, min(tiles, ctas)
    G = max(1, min(units // 4, ctas))
    begin = lambda c: c * units // G  # noqa: E731
    cta = lambda u: ((u + 1) * G - 1) // units  # noqa: E731
    segs = []
    for c in range(G):
        u, u1, mine = begin(c), begin(c + 1), []
        while u < u1:
            t = u // n_kb
            k0 = u - t * n_kb
            k1 = min(n_kb, k0 + (u1 - u))
            first, last = cta(t * n_kb), cta(t * n_kb + n_kb - 1)
            mine.append((t, k0, k1, c - first, first == last))
            u += k1 - k0
        segs.append(mine)
    slots = max(cta(t * n_kb + n_kb - 1) - cta(t * n_kb) + 1 for t in range(tiles))
    return segs, slots, G


@pytest.mark.parametrize("shape", [(16, 28672, 8192, 128), (64, 28672, 8192, 128), (16, 4096, 4096, 128),
                                   (1, 256, 4096, 128), (8, 128, 16384, 128), (37, 200, 352, 32),
                                   (17, 384, 1216, 64), (256, 4096, 4096, 128), (4096, 4096, 4096, 128),
                                   (16, 512, 1024, 128), (64, 128, 512, 8)])
def test_w4a16_stream_k_split(shape):
    """Every (tile, K step) unit is taken exactly once, a tile that one CTA
    covers is written whole, a split tile's CTAs fill slabs 0 .. n-1, and the
    library's workspace holds exactly the error word plus those slabs."""
    N, d_out, d_in, g = shape
    cfg = awq.make_cfg(4, g, False, 1)
    segs, slots, G = _w4_split(N, d_out, d_in, g)
    p_stride = (N * d_out + 3) // 4 * 4
    want = 1024 + ((slots * p_stride * 4 + 1023) // 1024 * 1024 if slots > 1 else 0)
    assert awq.w4a16_workspace_size(N, d_out, d_in, cfg) == want
    if segs is None:
        return
    seen, slabs = {}, {}
    for c, mine in enumerate(segs):
        for t, k0, k1, slab, whole in mine:
            assert 0 <= slab < slots and k0 < k1
            if whole:
                assert slab == 0
            for k in range(k0, k1):
                assert (t, k) not in seen
                seen[(t, k)] = whole
            slabs.setdefault(t, set()).add(slab)
    n_kb = max(k for _, k in seen) + 1
    assert len(seen) == len({t for t, _ in seen}) * n_kb
    for t, s in slabs.items():
        assert s == set(range(len(s)))
    if shape == (16, 28672, 8192, 128):
        assert (G, slots) == (148, 2)  # 224 tiles x 32 steps: 48 or 49 steps per CTA
