"""AWQ calibration and scale search on B200 (sm_100a): a C-ABI CUDA library
(include/awq.h) and its Python binding."""
from .binding import (  # noqa: F401
    AwqError, QCfg, make_cfg, lib, act_stats, search_scales, search_scales_segmented, search_candidates, quantize_pack, workspace_error,
    group_clip_workspace_size, search_group_clip, quantize_pack_group_clip,
    fold_inv_scales, w4a16_workspace_size, w4a16_gemm, pack_workspace_size, selftest_bounded_wait,
    select_library, bounds_checks_enabled, bounds_error, selftest_bounds, AWQ_ERR_BOUNDS,
    stats_workspace_size, search_workspace_size, search_form, workspace, debug_dw, step, status_str,
)
