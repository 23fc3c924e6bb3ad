"""awq_act_stats_noalloc: activation statistics for callers that cannot
allocate device memory (for example code running inside an allocator or
memory pool it does not own, or a plugin host that only hands out its own
buffers). It keeps its scratch in a fixed array compiled into the library.

Checked through the C ABI against awq_act_stats (which takes a caller
workspace), within the statistics tolerance of the other parity tests, on two
calls in a row of different sizes (the second must not see the first's
leftovers). This file is collected last so that a run stopping at its first
failure has already run every other test; it passes alone in a fresh process
as well.
"""
import ctypes

import numpy as np
import pytest

from awq_inputs import custom, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import weight_only_int4_act_b200 as awq  # noqa: E402

A_RTOL = 1e-5


def _noalloc(X):
    N, d_in = X.shape
    a = torch.empty(d_in, dtype=torch.float32, device=X.device)
    st = awq.lib().awq_act_stats_noalloc(ctypes.c_void_p(X.data_ptr()), N, d_in, ctypes.c_void_p(a.data_ptr()),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, a


def _device_x(N, d_in, seed):
    _, Xb = make_inputs(custom(8, d_in, N, seed=seed))
    return torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).cuda()


def test_noalloc_stats_match_workspace_version_twice():
    for N, d_in, seed in ((20000, 4096, 31), (257, 1032, 32)):
        X = _device_x(N, d_in, seed)
        ref = awq.act_stats(X)
        st, got = _noalloc(X)
        assert st == 0, awq.status_str(st)
        torch.cuda.synchronize()
        r = ref.cpu().numpy().astype(np.float64)
        g = got.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(g - r) <= A_RTOL * np.abs(r)), (N, d_in, np.max(np.abs(g - r) / np.abs(r)))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    X = torch.zeros((2, 8), dtype=torch.bfloat16, device="cuda")
    a = torch.empty(8, dtype=torch.float32, device="cuda")
    too_wide = 524288 + 8
    st = awq.lib().awq_act_stats_noalloc(ctypes.c_void_p(X.data_ptr()), 2, too_wide, ctypes.c_void_p(a.data_ptr()),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 2  # AWQ_ERR_SHAPE, before anything is launched
