import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU-side oracle work")


@pytest.fixture(autouse=True)
def _no_index_check_fired(request):
    """After a GPU test on the debug build (AWQ_B200_LIB=check), no index
    check may have fired; on the release build there is nothing to read."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import weight_only_int4_act_b200 as awq
    if not awq.bounds_checks_enabled():
        return
    st, site = awq.bounds_error()
    assert st == 0, f"an index check failed at site {site:#x}"
