"""The synthetic linear-layer workloads of the AWQ search path.

Each workload is one linear layer: W[d_out, d_in] (rows = output channels),
calibration activations X[N, d_in] (tokens x input channels), and the
quantiser settings (bits, group size g along d_in, symmetric or with zero
point, alpha grid of n_alpha points). Synthetic inputs stand in for the real
calibration text and trained Llama weights the pages use, neither of which is
available: the shapes are those of Llama-7B / Llama-3-70B projections, the
value distributions are Gaussian weights and activations whose per-channel
scale is lognormal, with a small fraction of outlier channels (the pages put
the salient fraction at 0.1-1% of channels).
"""
from __future__ import annotations

from dataclasses import dataclass, asdict

import numpy as np

from . import gen


@dataclass(frozen=True)
class Workload:
    key: str
    title: str
    d_out: int
    d_in: int
    N: int
    bits: int
    symmetric: bool
    group: int
    n_alpha: int
    w_std: float
    x_kind: str                 # "normal" or "absnormal"
    x_lognormal_sigma: float | None
    outlier_count: int
    outlier_factor: float
    seed: int

    def as_dict(self):
        return asdict(self)


WORKLOADS = {
    "C1": Workload("C1", "single linear 256x512, 256 tokens, INT4 asym g128",
                   256, 512, 256, 4, False, 128, 20, 0.02,
                   "normal", None, 5, 20.0, 20260001),
    "C2": Workload("C2", "Llama-7B attn proj 4096x4096, 4096 tokens (8x512), INT4 asym g128",
                   4096, 4096, 4096, 4, False, 128, 20, 0.02,
                   "normal", 1.0, 41, 30.0, 20260002),
    "C3": Workload("C3", "MLP gate/up 11008x4096, 16384 tokens, INT4 asym g128",
                   11008, 4096, 16384, 4, False, 128, 20, 0.02,
                   "normal", 1.5, 41, 50.0, 20260003),
    "C4": Workload("C4", "MLP down 4096x11008, 16384 tokens post-SiLU-like, INT3 sym g64",
                   4096, 11008, 16384, 3, True, 64, 20, 0.015,
                   "absnormal", None, 55, 40.0, 20260004),
    "C5": Workload("C5", "70B MLP 28672x8192, 65536 tokens (128x512), INT4 asym g128",
                   28672, 8192, 65536, 4, False, 128, 20, 0.01,
                   "normal", 1.0, 82, 30.0, 20260005),
}


def custom(d_out, d_in, N, bits=4, symmetric=False, group=128, n_alpha=20,
           w_std=0.02, x_kind="normal", x_lognormal_sigma=1.0,
           outlier_count=None, outlier_factor=30.0, seed=7) -> Workload:
    """A workload of arbitrary shape with the C2-style recipe (for parity tests)."""
    if outlier_count is None:
        outlier_count = max(1, int(round(0.01 * d_in)))
    return Workload(f"custom-{d_out}x{d_in}x{N}", "custom", d_out, d_in, N, bits,
                    symmetric, group, n_alpha, w_std, x_kind, x_lognormal_sigma,
                    outlier_count, outlier_factor, seed)


def make_inputs(wl: Workload):
    """(W_bits[d_out, d_in], X_bits[N, d_in]) as uint16 bf16 bit patterns."""
    W = gen.make_weight(wl.seed, wl.d_out, wl.d_in, wl.w_std)
    X = gen.make_activations(wl.seed, wl.N, wl.d_in, wl.x_kind, wl.x_lognormal_sigma,
                             wl.outlier_count, wl.outlier_factor)
    return W, X


def make_weight_rows(wl: Workload, rows) -> np.ndarray:
    """Selected rows of W only (bf16 bits), without generating the rest."""
    key = gen.stream_key(wl.seed, gen.STREAM_W)
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), wl.d_in), dtype=np.uint16)
    for j, r in enumerate(rows):
        z = gen.normal(key, int(r) * wl.d_in, wl.d_in)
        out[j] = gen.f64_to_bf16_bits(wl.w_std * z)
    return out
