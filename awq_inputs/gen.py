"""Seeded, synthetic inputs for the AWQ calibration and scale-search path.

This module is shared by the CUDA path's tests and bench and by the CPU
oracle. It holds none of the method's arithmetic: only a counter-based
random-number generator, its transformation to normal samples, and the
recipes (shapes, value distributions, outlier channels) of the workloads,
rounded once to bf16. The same bf16 bytes go to the oracle and to the GPU.

Generator
---------
* splitmix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): the i-th 64-bit word of a stream with key ``k``
  is ``mix(k + (i + 1) * 0x9E3779B97F4A7C15)`` (arithmetic mod 2**64), where
  ``mix`` is the splitmix64 finaliser. A stream's key is
  ``mix(seed * 0x9E3779B97F4A7C15 + stream_id)``.
* uniform in (0, 1): ``((word >> 11) + 0.5) * 2**-53``; never 0 or 1.
* normal: Box-Muller on the pair (u[2p], u[2p+1]);
  sample 2p is ``r cos(2 pi u2)``, sample 2p+1 is ``r sin(2 pi u2)``,
  ``r = sqrt(-2 ln u1)``; computed in float64.
* values are formed in float64, rounded to float32 (round to nearest even),
  then to bf16 (round to nearest even on the float32 bits).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# stream ids: one independent stream per random quantity of a workload
STREAM_W = 1
STREAM_X = 2
STREAM_X2 = 3
STREAM_CHANNEL_STD = 4
STREAM_OUTLIER = 5

_CHUNK = 1 << 22  # samples per vectorised chunk (bounds temporary memory)
_THREADS = min(8, os.cpu_count() or 1)  # chunks are independent: filled by a thread pool


def _fill_rows(n_rows, rows_per, fill):
    """Call fill(r0, r1) over [0, n_rows) in blocks of rows_per rows, on a
    thread pool (numpy releases the GIL in its array loops). Every sample
    depends only on its position in its stream, so the bytes do not depend on
    the blocking or the order."""
    blocks = [(r0, min(n_rows, r0 + rows_per)) for r0 in range(0, n_rows, rows_per)]
    if len(blocks) <= 1 or _THREADS <= 1:
        for r0, r1 in blocks:
            fill(r0, r1)
        return
    with ThreadPoolExecutor(_THREADS) as ex:
        for f in [ex.submit(fill, r0, r1) for r0, r1 in blocks]:
            f.result()


def _mix64(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        base = np.array([seed], dtype=np.uint64) * _GOLDEN + np.uint64(stream)
    return _mix64(base)[0]


def words(key: np.uint64, start: int, count: int) -> np.ndarray:
    """64-bit words ``start .. start+count-1`` of the stream with ``key``."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(key + idx * _GOLDEN)


def uniform(key: np.uint64, start: int, count: int) -> np.ndarray:
    w = words(key, start, count)
    return ((w >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(key: np.uint64, start: int, count: int) -> np.ndarray:
    """Standard normal samples ``start .. start+count-1`` of a stream (float64)."""
    out = np.empty(count, dtype=np.float64)
    done = 0
    while done < count:
        n = min(_CHUNK, count - done)
        s = start + done
        p0 = s // 2
        p1 = (s + n - 1) // 2 + 1
        u = uniform(key, 2 * p0, 2 * (p1 - p0)).reshape(-1, 2)
        r = np.sqrt(-2.0 * np.log(u[:, 0]))
        th = 2.0 * np.pi * u[:, 1]
        z = np.empty(2 * (p1 - p0), dtype=np.float64)
        z[0::2] = r * np.cos(th)
        z[1::2] = r * np.sin(th)
        off = s - 2 * p0
        out[done:done + n] = z[off:off + n]
        done += n
    return out


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 (RNE) -> bf16 (RNE) bit patterns, as uint16."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    with np.errstate(over="ignore"):
        r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def pick_channels(seed: int, d_in: int, count: int) -> np.ndarray:
    """``count`` distinct channels of ``range(d_in)``, by a partial Fisher-Yates
    shuffle driven by the outlier stream; returned sorted."""
    if count <= 0:
        return np.zeros(0, dtype=np.int64)
    key = stream_key(seed, STREAM_OUTLIER)
    u = uniform(key, 0, count)
    perm = np.arange(d_in, dtype=np.int64)
    for j in range(count):
        r = j + int(np.floor(u[j] * (d_in - j)))
        r = min(r, d_in - 1)
        perm[j], perm[r] = perm[r], perm[j]
    return np.sort(perm[:count])


def make_weight(seed: int, d_out: int, d_in: int, w_std: float) -> np.ndarray:
    """W[d_out, d_in] ~ N(0, w_std^2), bf16 bits, row-major."""
    key = stream_key(seed, STREAM_W)
    out = np.empty((d_out, d_in), dtype=np.uint16)

    def fill(r0, r1):
        z = normal(key, r0 * d_in, (r1 - r0) * d_in)
        out[r0:r1] = f64_to_bf16_bits(w_std * z).reshape(r1 - r0, d_in)

    _fill_rows(d_out, max(1, _CHUNK // max(d_in, 1)), fill)
    return out


def make_activations(seed: int, N: int, d_in: int, kind: str,
                     lognormal_sigma: float | None,
                     outlier_count: int, outlier_factor: float) -> np.ndarray:
    """X[N, d_in] (tokens x input channels), bf16 bits, row-major.

    kind ``normal``:   X[t,i] = c_i * sigma_i * z[t,i]
    kind ``absnormal``: X[t,i] = c_i * |z1[t,i]| * z2[t,i]   (post-SiLU-like)
    sigma_i = exp(lognormal_sigma * zc[i]) when ``lognormal_sigma`` is given,
    else 1; c_i = outlier_factor on the picked outlier channels, else 1.
    """
    key_x = stream_key(seed, STREAM_X)
    key_x2 = stream_key(seed, STREAM_X2)
    chan = np.ones(d_in, dtype=np.float64)
    if lognormal_sigma is not None:
        chan = np.exp(lognormal_sigma * normal(stream_key(seed, STREAM_CHANNEL_STD), 0, d_in))
    outl = pick_channels(seed, d_in, outlier_count)
    chan[outl] *= outlier_factor
    out = np.empty((N, d_in), dtype=np.uint16)

    def fill(t0, t1):
        n = (t1 - t0) * d_in
        z = normal(key_x, t0 * d_in, n).reshape(t1 - t0, d_in)
        if kind == "absnormal":
            z = np.abs(z) * normal(key_x2, t0 * d_in, n).reshape(t1 - t0, d_in)
        out[t0:t1] = f64_to_bf16_bits(z * chan[None, :])

    if kind not in ("normal", "absnormal"):
        raise ValueError(f"unknown activation kind {kind!r}")
    _fill_rows(N, max(1, _CHUNK // max(d_in, 1)), fill)
    return out
