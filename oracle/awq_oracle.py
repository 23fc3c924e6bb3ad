"""CPU oracle for the AWQ calibration / scale-search / pack path.

TEST INFRASTRUCTURE. This module is the plain, slow, float64 statement of
what the path computes; it exists to check the CUDA library. Only the tests,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and reference
legs may import it. The product path never calls it, and it shares no code
with the CUDA library (it reads only the bf16 bit patterns the seeded input
generator produces).

Pages cited (by title and section):
  [P1] "AWQ量化" tutorial (aiqz.cc): 量化基础 (uniform quantiser), 激活感知
       (importance Omega_i), 缩放保护 (scale-quantise-restore), 误差分析,
       GPTQ对比 (AWQ objective).
  [P2] "AWQ量化技术解析：激活感知的权重量化革命" (kwkr.cn): §1.2 (dequantise
       on the fly, W_int4 x scale_fp16), §2.1 (INT4 clip to [-8, 7], fp16
       scale), §4.2 (two 4-bit values per byte).
  [P3] "大模型的开发应用（十八）：大模型量化：GPTQ与AWQ" (ewbang.com): AWQ 二.1
       (the layer computes Q(W s)(X / s)), 二.2 (grid search of alpha on
       [0, 1]), 二.3 (INT4 storage, dequantised for the product).
  [P4] "AWQ 量化全流程拆解：将 70B 大模型塞进单张消费级 GPU" (lnrq.cn): §三
       quant_config (zero_point, q_group_size = 128, w_bit = 4).
  [P5] "AWQ" (scholia-log, inference-quantization/2_AWQ): §1.1 (Delta Y =
       Delta W X), §1.2 (a_i = E|x_i|), §2.1 (W X = (W S)(S^-1 X)), §2.3
       (Q(w) = Delta round(w / Delta)), §3.1-3.3 (worked examples, groups),
       §4.1 (s_i = a_i^alpha and the boxed objective), §4.3 (diagonal S:
       S^-1 folds into the adjacent norm or linear layer).

Conventions. W is [d_out, d_in] (rows are output channels), X is [N, d_in]
(tokens x input channels), so the layer output for token t is W x_t and the
output error over the calibration set is Delta W X^T. Groups are g consecutive
input channels within one row. Readings taken where the pages are silent are
listed with each function.

Every function here is pinned by tests/test_oracle_pins.py against values the
pages print, closed forms, brute force or invariants; nothing is "parity
unpinned".
"""
from __future__ import annotations

import numpy as np

EPS_A = 1e-4       # floor on a_i before the power (dead channels; s_i > 0 required by [P5] §2.1)
EPS_DELTA = 1e-8   # floor on a group's range (all-equal groups)

_ROW_CHUNK = 1024
_TOKEN_CHUNK = 8192


# ---------------------------------------------------------------------------
# inputs
# ---------------------------------------------------------------------------
def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# step a1: activation statistics
# ---------------------------------------------------------------------------
def act_stats(X_bits: np.ndarray) -> np.ndarray:
    """a_i = (1/N) sum_t |X[t, i]|.

    [P1] 激活感知: Omega_i is the mean absolute activation of channel i over
    the N calibration samples; [P5] §1.2: a_i = E[|x_i|]. Summed in float64
    over token chunks.
    """
    N, d_in = X_bits.shape
    acc = np.zeros(d_in, dtype=np.float64)
    for t0 in range(0, N, _TOKEN_CHUNK):
        acc += np.abs(widen_bf16(X_bits[t0:t0 + _TOKEN_CHUNK])).sum(axis=0)
    return acc / N


# ---------------------------------------------------------------------------
# step a2: candidate scales
# ---------------------------------------------------------------------------
def alpha_grid(n_alpha: int) -> np.ndarray:
    """alpha_k = k / n_alpha, k = 0 .. n_alpha-1 (a grid on [0, 1), [P3] AWQ 二.2)."""
    return np.arange(n_alpha, dtype=np.float64) / n_alpha


def candidate_scales(a: np.ndarray, alpha: float, eps_a: float = EPS_A,
                     normalise: bool = True) -> np.ndarray:
    """s_i = max(a_i, eps_a)^alpha, divided by sqrt(max_j s_j * min_j s_j).

    [P5] §4.1: s_i = a_i^alpha, alpha = 0 gives s = 1 (no activation-aware
    scaling). The sqrt(max * min) normalisation is not on the pages; it is part
    of the stated task and, since both quantisers are scale-equivariant, it
    moves the loss only by rounding. Reading: a_i is floored at eps_a before the
    power so that a dead channel still gets s_i > 0.
    """
    t = np.maximum(np.asarray(a, dtype=np.float64), eps_a) ** float(alpha)
    if not normalise:
        return t
    return t / np.sqrt(t.max() * t.min())


# ---------------------------------------------------------------------------
# step a3: group-wise quantiser and fake quantisation
# ---------------------------------------------------------------------------
def quantize_groups(V: np.ndarray, bits: int, group: int, symmetric: bool,
                    eps_delta: float = EPS_DELTA, clip: float = 1.0):
    """Uniform group-wise quantisation of V[rows, d_in] along d_in.

    Returns (V_hat, codes, delta, zero): V_hat the dequantised values, codes
    the stored unsigned codes (one per element), delta[rows, groups] the step,
    zero[rows, groups] the stored zero point.

    Symmetric ([P1] 量化基础: q = round(W/s), s = max|W| / (2^(b-1) - 1);
    [P2] §2.1: clip to [-8, 7] for INT4; [P5] §3.1: Delta = 1/7 for a group
    maximum of 1 at INT4):
        Delta = max(max_i |v_i|, eps) / (2^(b-1) - 1)
        q_i   = clamp(rne(v_i / Delta), -2^(b-1), 2^(b-1) - 1)
        v_hat = q_i * Delta;  stored code = q_i + 2^(b-1), stored zero = 2^(b-1).
    Asymmetric with zero point ([P4] §三 zero_point = True; the pages give no
    formula, this is the min/max affine reading):
        Delta = max(max v - min v, eps) / (2^b - 1)
        z     = clamp(rne(-min v / Delta), 0, 2^b - 1)
        q_i   = clamp(rne(v_i / Delta) + z, 0, 2^b - 1)
        v_hat = (q_i - z) * Delta.
    rne = round half to even ([P5] §2.3 "round"; the demo's np.round is
    half-to-even too).

    Clipping ([P5] 参考资料 note: the practical algorithm searches a restricted
    parameterisation "possibly combined with clipping"; the pages give no
    formula): with clip ratio c in (0, 1], the group's range is shrunk before
    the step is taken — max|v| -> c max|v| (symmetric), max v -> c max v and
    min v -> c min v (asymmetric) — and values outside the shrunk range clip to
    the extreme codes. c = 1 is the plain quantiser.

    group = 0 is per-tensor quantisation ([P1] 量化基础: one step s = max|W|
    / (2^(b-1) - 1) for the whole matrix): the flattened matrix is one group,
    and delta / zero are [1, 1].
    """
    V = np.asarray(V, dtype=np.float64)
    if group == 0:
        Vh, codes, delta, zero = quantize_groups(V.reshape(1, -1), bits, V.size, symmetric, eps_delta, clip)
        return Vh.reshape(V.shape), codes.reshape(V.shape), delta, zero
    rows, d_in = V.shape
    if d_in % group:
        raise ValueError("d_in must be a multiple of the group size")
    G = V.reshape(rows, d_in // group, group)
    clip = np.broadcast_to(np.asarray(clip, dtype=np.float64), (rows, d_in // group))  # scalar or per group
    if symmetric:
        qmax = 2 ** (bits - 1) - 1
        qmin = -(2 ** (bits - 1))
        delta = np.maximum(clip * np.abs(G).max(axis=-1), eps_delta) / qmax
        q = np.clip(np.rint(G / delta[..., None]), qmin, qmax)
        Vh = q * delta[..., None]
        codes = (q - qmin).astype(np.int64)
        zero = np.full(delta.shape, float(-qmin))
    else:
        levels = 2 ** bits - 1
        mx = clip * G.max(axis=-1)
        mn = clip * G.min(axis=-1)
        delta = np.maximum(mx - mn, eps_delta) / levels
        zero = np.clip(np.rint(-mn / delta), 0, levels)
        q = np.clip(np.rint(G / delta[..., None]) + zero[..., None], 0, levels)
        Vh = (q - zero[..., None]) * delta[..., None]
        codes = q.astype(np.int64)
    return Vh.reshape(rows, d_in), codes.reshape(rows, d_in), delta, zero


def fake_quant(W: np.ndarray, s: np.ndarray, bits: int, group: int, symmetric: bool, clip: float = 1.0):
    """W_hat = Q(W S) S^-1 for W[rows, d_in] (float64) and scales s[d_in].

    [P1] 缩放保护: W~_i = s_i W_i, W^_i = Q(W~_i) / s_i; [P5] §2.2: Q(WS)S^-1.
    Returns (W_hat, codes, delta, zero) with the quantiser of quantize_groups.
    """
    s = np.asarray(s, dtype=np.float64)
    V = W * s[None, :]
    Vh, codes, delta, zero = quantize_groups(V, bits, group, symmetric, clip=clip)
    return Vh / s[None, :], codes, delta, zero


def delta_weight(W: np.ndarray, s: np.ndarray, bits: int, group: int, symmetric: bool,
                 clip: float = 1.0) -> np.ndarray:
    """Delta W = Q(W S) S^-1 - W, formed before any contraction."""
    What = fake_quant(W, s, bits, group, symmetric, clip)[0]
    return What - W


# ---------------------------------------------------------------------------
# steps a4/a5: output error and its squared Frobenius norm
# ---------------------------------------------------------------------------
def output_error(dW: np.ndarray, X: np.ndarray) -> np.ndarray:
    """Delta Y = Delta W X^T ([P5] §1.1 boxed: Delta Y = Delta W X), [rows, N]."""
    return dW @ X.T


def loss_direct(dW: np.ndarray, X_bits: np.ndarray) -> float:
    """||Delta W X^T||_F^2 = sum_r sum_t (sum_i dW[r,i] X[t,i])^2.

    [P5] §4.1 boxed objective ||W X - Q(WS) S^-1 X||_F^2; [P1] GPTQ对比 writes
    the same objective as an expectation over x (equal up to the constant 1/N).
    """
    return float(row_losses_direct(dW, X_bits).sum())


def row_losses_direct(dW: np.ndarray, X_bits: np.ndarray) -> np.ndarray:
    """Per-row losses l_r = sum_t (sum_i dW[r,i] X[t,i])^2, float64 [rows]."""
    out = np.zeros(dW.shape[0], dtype=np.float64)
    for t0 in range(0, X_bits.shape[0], _TOKEN_CHUNK):
        Xc = widen_bf16(X_bits[t0:t0 + _TOKEN_CHUNK])
        for r0 in range(0, dW.shape[0], _ROW_CHUNK):
            D = output_error(dW[r0:r0 + _ROW_CHUNK], Xc)
            out[r0:r0 + _ROW_CHUNK] += np.einsum("rt,rt->r", D, D)
    return out


def gram(X_bits: np.ndarray) -> np.ndarray:
    """G = X^T X (float64, [d_in, d_in]); the loss is then sum_r dW_r G dW_r^T."""
    d_in = X_bits.shape[1]
    G = np.zeros((d_in, d_in), dtype=np.float64)
    for t0 in range(0, X_bits.shape[0], _TOKEN_CHUNK):
        Xc = widen_bf16(X_bits[t0:t0 + _TOKEN_CHUNK])
        G += Xc.T @ Xc
    return G


def row_losses_gram(dW: np.ndarray, G: np.ndarray) -> np.ndarray:
    """Per-row losses through the Gram matrix: l_r = dW_r G dW_r^T."""
    out = np.empty(dW.shape[0], dtype=np.float64)
    for r0 in range(0, dW.shape[0], _ROW_CHUNK):
        blk = dW[r0:r0 + _ROW_CHUNK]
        out[r0:r0 + _ROW_CHUNK] = np.einsum("ri,ri->r", blk @ G, blk)
    return out


# ---------------------------------------------------------------------------
# steps a2-a6 together: the search
# ---------------------------------------------------------------------------
def search(W_bits: np.ndarray, X_bits: np.ndarray, a: np.ndarray, bits: int, group: int,
           symmetric: bool, n_alpha: int, form: str = "direct", G: np.ndarray | None = None,
           rows=None):
    """Loss of every alpha candidate and the chosen one.

    For alpha_k in the grid: s = candidate_scales(a, alpha_k), dW = Q(WS)S^-1 - W,
    L(alpha_k) = ||dW X^T||_F^2 ([P5] §4.1). k* = argmin_k L, the lowest k on
    exact ties. ``form`` = "direct" contracts with X, "gram" with G = X^T X (the
    same sum, reassociated). ``rows`` restricts to a subset of W's rows and then
    also returns the per-row losses [n_alpha, len(rows)].

    Returns dict(losses[n_alpha] float64, best k, s_best[d_in], alphas,
    row_losses or None).
    """
    alphas = alpha_grid(n_alpha)
    Wsel = W_bits if rows is None else W_bits[np.asarray(rows)]
    W = widen_bf16(Wsel)
    if form == "gram" and G is None:
        G = gram(X_bits)
    per_row = np.zeros((n_alpha, W.shape[0]), dtype=np.float64)
    if form == "gram":
        for k, al in enumerate(alphas):
            per_row[k] = row_losses_gram(delta_weight(W, candidate_scales(a, al), bits, group, symmetric), G)
    elif rows is not None:
        # few rows: stack every candidate's dW and pass over X once
        dWs = np.concatenate([delta_weight(W, candidate_scales(a, al), bits, group, symmetric)
                              for al in alphas])
        per_row = row_losses_direct(dWs, X_bits).reshape(n_alpha, W.shape[0])
    else:
        for k, al in enumerate(alphas):
            per_row[k] = row_losses_direct(delta_weight(W, candidate_scales(a, al), bits, group, symmetric),
                                           X_bits)
    losses = per_row.sum(axis=1)
    best = choose(losses)
    return dict(losses=losses, best=best, s_best=candidate_scales(a, alphas[best]),
                alphas=alphas, row_losses=per_row if rows is not None else None)


def search_candidates(W_bits: np.ndarray, X_bits: np.ndarray, s_cand: np.ndarray, bits: int, group: int,
                      symmetric: bool, clips=None, form: str = "direct", G: np.ndarray | None = None):
    """Loss of arbitrary candidates: candidate k uses scales s_cand[k] and clip
    ratio clips[k] (default 1); L_k = ||(Q(W S_k) S_k^-1 - W) X^T||_F^2 and the
    lowest-index argmin, as in search(). Covers the clipping search (the same s
    with several clip ratios) and other candidate sets (e.g. a salience mask
    with a fixed scale factor, [P1] 显著识别 and its Python demo)."""
    W = widen_bf16(W_bits)
    s_cand = np.atleast_2d(np.asarray(s_cand, dtype=np.float64))
    n = s_cand.shape[0]
    clips = np.ones(n) if clips is None else np.asarray(clips, dtype=np.float64)
    if form == "gram" and G is None:
        G = gram(X_bits)
    losses = np.zeros(n)
    for k in range(n):
        dW = delta_weight(W, s_cand[k], bits, group, symmetric, clips[k])
        losses[k] = (row_losses_gram(dW, G) if form == "gram" else row_losses_direct(dW, X_bits)).sum()
    return dict(losses=losses, best=choose(losses))


def group_clip_errors(W_bits: np.ndarray, X_bits: np.ndarray, s: np.ndarray, bits: int, group: int,
                      symmetric: bool, clips, G: np.ndarray | None = None) -> np.ndarray:
    """Per-group output error of each clip ratio, err[c, r, j] =
    sum_t (sum_{i in group j} dW_c[r, i] X[t, i])^2, i.e. the output error the
    group would cause with only its own inputs (the block-diagonal part of
    dW G dW^T), with dW_c = Q(W S; clip c) S^-1 - W. This is the per-group
    reading of the clipping search ([P5] 参考资料 note): each group of each row
    then takes the ratio with the smallest error."""
    W = widen_bf16(W_bits)
    rows, d_in = W.shape
    ng = d_in // group
    if G is None:
        G = gram(X_bits)
    out = np.zeros((len(clips), rows, ng))
    for ci, c in enumerate(clips):
        dW = delta_weight(W, s, bits, group, symmetric, c)
        for j in range(ng):
            blk = dW[:, j * group:(j + 1) * group]
            Gb = G[j * group:(j + 1) * group, j * group:(j + 1) * group]
            out[ci, :, j] = np.einsum("ri,ri->r", blk @ Gb, blk)
    return out


def group_clip_choice(err: np.ndarray) -> np.ndarray:
    """Index of the smallest error per (row, group), the lowest index on ties."""
    return np.argmin(err, axis=0)


def choose(losses: np.ndarray) -> int:
    """argmin over the grid; the lowest index among exact ties."""
    losses = np.asarray(losses, dtype=np.float64)
    return int(np.flatnonzero(losses == losses.min())[0])


def acceptable_choices(losses: np.ndarray, rel: float = 0.005) -> list[int]:
    """Indices whose loss is within ``rel`` (relative) of the minimum: any of
    them is an acceptable choice when two candidates are that close."""
    losses = np.asarray(losses, dtype=np.float64)
    m = losses.min()
    return [int(k) for k in np.flatnonzero(losses <= m * (1.0 + rel))]


# ---------------------------------------------------------------------------
# step a7: pack
# ---------------------------------------------------------------------------
def pack_codes(codes: np.ndarray) -> np.ndarray:
    """uint32 word w of a row holds codes 8w .. 8w+7, code 8w+j in bits 4j..4j+3.

    [P2] §4.2 stores two 4-bit values per byte; the 8-nibbles-per-uint32 order
    (lowest input channel in the lowest nibble) is this library's stated
    layout. 2- and 3-bit codes also take one nibble each.
    """
    codes = np.asarray(codes, dtype=np.uint64)
    rows, d_in = codes.shape
    if d_in % 8:
        raise ValueError("d_in must be a multiple of 8")
    c = codes.reshape(rows, d_in // 8, 8)
    word = np.zeros((rows, d_in // 8), dtype=np.uint64)
    for j in range(8):
        word |= (c[:, :, j] & np.uint64(0xF)) << np.uint64(4 * j)
    return word.astype(np.uint32)


def to_fp16(x: np.ndarray) -> np.ndarray:
    """float64 -> IEEE binary16, round to nearest even ([P2] §2.1 fp16 scale)."""
    return np.asarray(x, dtype=np.float64).astype(np.float16)


def pack(W_bits: np.ndarray, s: np.ndarray, bits: int, group: int, symmetric: bool, clip: float = 1.0):
    """Codes of Q(W S) at the chosen scales, packed; fp16 step and zero point.

    Returns (qweight uint32[rows, d_in/8], scales fp16[rows, d_in/g],
    zeros fp16[rows, d_in/g], codes int64[rows, d_in], delta float64,
    zero float64). The search uses the float64 step; only the stored copy is
    rounded to fp16 (reading: the pages give an fp16 scale, [P2] §2.1).
    """
    W = widen_bf16(W_bits)
    _, codes, delta, zero = fake_quant(W, s, bits, group, symmetric, clip)
    return pack_codes(codes), to_fp16(delta), to_fp16(zero), codes, delta, zero


def boundary_mask(W_bits: np.ndarray, s: np.ndarray, bits: int, group: int, symmetric: bool,
                  band: float = 1e-4, clip: float = 1.0, parts: bool = False):
    """Elements whose code the float64 oracle decides within ``band`` of a
    rounding boundary. Rounding to the nearest grid point ([P5] §2.3,
    Q(w) = Delta round(w / Delta)) changes its answer only where w / Delta
    crosses a half-integer, so an element is flagged when its own v / Delta
    lies within ``band`` of one; with a zero point (asymmetric) every element
    of a group also depends on z = round(-min v / Delta), so the whole group is
    flagged when -min v / Delta lies within ``band`` of a half-integer. A
    float32 computation may round flagged elements either way; everything else
    must match.

    Returns the combined [rows, d_in] mask, or with ``parts`` the pair
    (element flags [rows, d_in], zero-point flags [rows, groups]) (for
    group = 0: [1, 1] zero-point flags)."""
    W = widen_bf16(W_bits)
    V = W * np.asarray(s, dtype=np.float64)[None, :]
    if group == 0:  # per tensor: one group of all elements
        flat = W_bits.reshape(1, -1)
        s_flat = np.tile(np.asarray(s, dtype=np.float64), W_bits.shape[0])
        el, zn = boundary_mask(flat, s_flat, bits, flat.shape[1], symmetric, band, clip, parts=True)
        el = el.reshape(W_bits.shape)
        return (el, zn) if parts else (el | zn[0, 0])
    rows, d_in = V.shape
    G = V.reshape(rows, d_in // group, group)

    def near_half(r):
        return np.abs(r - np.floor(r) - 0.5) < band

    if symmetric:
        delta = np.maximum(clip * np.abs(G).max(axis=-1), EPS_DELTA) / (2 ** (bits - 1) - 1)
        el = near_half(G / delta[..., None])
        zn = np.zeros(delta.shape, dtype=bool)   # the zero point is fixed
    else:
        mx, mn = clip * G.max(axis=-1), clip * G.min(axis=-1)
        delta = np.maximum(mx - mn, EPS_DELTA) / (2 ** bits - 1)
        el = near_half(G / delta[..., None])
        zn = near_half(-mn / delta)
    el = el.reshape(rows, d_in)
    if parts:
        return el, zn
    return el | np.repeat(zn, group, axis=1)


# ---------------------------------------------------------------------------
# inference side: S^-1 folded into the producer of X, dequantisation of the
# packed format, and the W4A16 product
# ---------------------------------------------------------------------------
def to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (NaN stays NaN)."""
    u = np.asarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    nan = np.isnan(np.asarray(x32, dtype=np.float32))
    out = rounded.astype(np.uint16)
    out[nan] = ((u[nan] >> np.uint64(16)) | np.uint64(0x40)).astype(np.uint16)
    return out


def widen_f16(bits: np.ndarray) -> np.ndarray:
    """IEEE binary16 bit patterns (uint16) -> exact float64 values."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def to_f16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> binary16 bit patterns, round to nearest even (beyond the
    fp16 range: infinity)."""
    with np.errstate(over="ignore"):
        return np.asarray(x32, dtype=np.float32).astype(np.float16).view(np.uint16)


def widen(bits: np.ndarray, dtype: str) -> np.ndarray:
    """16-bit patterns of type ``dtype`` ("bf16" or "f16") -> float64."""
    return widen_bf16(bits) if dtype == "bf16" else widen_f16(bits)


def fold_inv_scales(p_bits: np.ndarray, s: np.ndarray, dtype: str = "bf16") -> np.ndarray:
    """Absorb S^-1 into the operation that produces X.

    [P5] §4.3 (why S is diagonal): S^-1 x is a per-channel scaling that can be
    folded into the adjacent LayerNorm or Linear, so X' = X S^-1 costs nothing
    at run time; [P3] AWQ 二.1: the layer then computes Q(W s)(X / s).
    p_bits holds that producer's parameters (bf16 or fp16 bit patterns, per
    ``dtype``) with the channel on the first axis: a norm's weight or bias
    [d_in], or the previous linear layer's weight [d_in, d_prev] / bias
    [d_in]. Entry (i, ...) becomes p / s_i, rounded to the same type.
    Reading: the quotient is taken in float32 (the kernel's precision;
    float32 division is correctly rounded on both sides), so the final
    rounding decides the same value on both sides.
    """
    p = widen(p_bits, dtype).astype(np.float32)
    s32 = np.asarray(s, dtype=np.float32)
    shape = (-1,) + (1,) * (p.ndim - 1)
    q = p / s32.reshape(shape)
    return to_bf16_bits(q) if dtype == "bf16" else to_f16_bits(q)


def unpack_codes(qweight: np.ndarray, d_in: int) -> np.ndarray:
    """Inverse of pack_codes: code of channel 8w+j = bits 4j..4j+3 of word w."""
    q = np.asarray(qweight).view(np.uint32).astype(np.uint64)
    rows = q.shape[0]
    codes = np.zeros((rows, d_in), dtype=np.int64)
    for j in range(8):
        codes[:, j::8] = ((q >> np.uint64(4 * j)) & np.uint64(0xF)).astype(np.int64)
    return codes


def dequant_packed(qweight: np.ndarray, scales_f16: np.ndarray, zeros_f16: np.ndarray, group: int,
                   d_in: int) -> np.ndarray:
    """W_hat[r, i] = (code - z) * Delta of the group, from the stored format.

    [P2] §1.2: the weights are dequantised on the fly as W_int4 x scale_fp16;
    with a zero point (asymmetric, [P4] §三 zero_point) the code is first
    offset by z. Symmetric codes are stored as q + 2^(b-1) with zero 2^(b-1)
    (this library's layout), so the same formula covers both quantisers.
    The result is W_hat = Q(W S) in the scaled space (float64, exact from the
    fp16 step and zero point)."""
    codes = unpack_codes(qweight, d_in).astype(np.float64)
    delta = np.repeat(np.asarray(scales_f16, dtype=np.float64), group, axis=1)
    zero = np.repeat(np.asarray(zeros_f16, dtype=np.float64), group, axis=1)
    return (codes - zero) * delta


def w4a16_matmul(Xp_bits: np.ndarray, qweight: np.ndarray, scales_f16: np.ndarray, zeros_f16: np.ndarray,
                 group: int, dtype: str = "bf16") -> np.ndarray:
    """Y[t, o] = sum_i X'[t, i] W_hat[o, i]: the quantised layer applied to
    activations that already carry S^-1 ([P5] §2.1 W X = (W S)(S^-1 X);
    [P3] AWQ 二.3: weights stored in INT4, dequantised to FP16 for the
    product). Float64, exact products of the 16-bit activations (bf16 or fp16
    per ``dtype``) and the dequantised weights."""
    Xp = widen(Xp_bits, dtype)
    W_hat = dequant_packed(qweight, scales_f16, zeros_f16, group, Xp.shape[1])
    return Xp @ W_hat.T
