"""Seeded synthetic inputs (no method arithmetic); shared by the oracle and the CUDA path's tests."""
from .configs import WORKLOADS, Workload, custom, make_inputs, make_weight_rows  # noqa: F401
from . import gen  # noqa: F401
