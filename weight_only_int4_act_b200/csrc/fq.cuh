// Group-wise uniform quantiser shared by the search (fake quantisation) and
// the pack kernel, so that both decide every code the same way.
//
// One thread holds CPT consecutive input channels of one row; a group of g
// channels is GL = g/CPT consecutive lanes of a warp (a power of two <= 32;
// groups never straddle warps). All 32 lanes must call fq_group together (the
// group reductions are full-warp shuffles); lanes without data pass zeros and
// belong to groups that are wholly inactive.
//
// Quantiser ([P1] 量化基础, [P2] §2.1, [P4] §三, [P5] §2.3):
//   symmetric : Delta = max(max|v|, eps) / (2^(b-1) - 1)
//               q = clamp(rne(v / Delta), -2^(b-1), 2^(b-1) - 1), v_hat = q Delta
//   asymmetric: Delta = max(max v - min v, eps) / (2^b - 1)
//               z = clamp(rne(-min v / Delta), 0, 2^b - 1)
//               q = clamp(rne(v / Delta) + z, 0, 2^b - 1),   v_hat = (q - z) Delta
// Arithmetic is fp32; Delta is the range times the fp32 constant 1/levels,
// 1/Delta is the hardware reciprocal (at most 1 ulp from the correctly rounded
// one), and rne(v / Delta) is rounded from the exact product v * (1/Delta):
// v / Delta is off by a few 1e-7 relative, so a code can differ from the
// exact decision only where v / Delta lies within ~5e-6 of a rounding
// boundary.
#pragma once
#include <cuda_runtime.h>

namespace awq {

constexpr float kEpsDelta = 1e-8f;

// 1 / (2^b - 1) rounded to fp32, for b = 1..4 (the step is range * this).
__device__ __forceinline__ float inv_levels(int b) {
  return b == 4 ? (1.0f / 15.0f) : b == 3 ? (1.0f / 7.0f) : b == 2 ? (1.0f / 3.0f) : 1.0f;
}

// Codes are kept in "magic" form c = stored code + 1.5*2^23 (see below):
// the stored code is c - 1.5*2^23 and the dequantised value is (c - off) * delta.
template <int CPT>
struct FqGroup {
  float delta;   // quantisation step of the group
  float zero;    // asymmetric: z; symmetric: 2^(b-1) (the stored zero)
  float off;     // 1.5*2^23 + z (asymmetric) or 1.5*2^23 + 2^(b-1) (symmetric)
  float c[CPT];  // magic-form codes of this thread's channels
};

// Round-to-nearest-even to an integer by the fp32 "magic number" method: for
// |x| < 2^22, x + 1.5*2^23 has no fraction bits left, so the addition itself
// rounds x to the nearest integer (ties to even), which subtracting the
// constant recovers exactly. Here the addition is fused with the product
// v * inv (one rounding of the exact product), which keeps the work on the
// full-rate FMA pipe. Larger |x| only occur in saturated (clamped) cases,
// where the ordering, which the method preserves, is all that matters.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

template <int GL>
__device__ __forceinline__ float group_max(float x) {
#pragma unroll
  for (int off = 1; off < GL; off <<= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
  return x;
}
template <int GL>
__device__ __forceinline__ float group_min(float x) {
#pragma unroll
  for (int off = 1; off < GL; off <<= 1) x = fminf(x, __shfl_xor_sync(0xffffffffu, x, off));
  return x;
}

// 1/x by the special-function unit (rcp.approx: at most 1 ulp of error; x is a
// quantisation step, normal and positive).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Three-input max / min (one instruction on sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
template <int N>
__device__ __forceinline__ float maxN(const float (&v)[N]) {
  float m = v[0];
  int j = 1;
#pragma unroll
  for (; j + 1 < N; j += 2) m = max3f(m, v[j], v[j + 1]);
  if (j < N) m = fmaxf(m, v[j]);
  return m;
}
template <int N>
__device__ __forceinline__ float minN(const float (&v)[N]) {
  float m = v[0];
  int j = 1;
#pragma unroll
  for (; j + 1 < N; j += 2) m = min3f(m, v[j], v[j + 1]);
  if (j < N) m = fminf(m, v[j]);
  return m;
}

__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Quantise this thread's CPT values of a group spread over GL lanes.
// The clamp to the code range is done on the FMA pipe: with span = 2^b - 1
// codes, y = sat((v / Delta + z) / span) is clamp(v / Delta + z, 0, span) / span,
// and fma(y, span, 1.5*2^23) rounds y * span to the nearest integer (ties to
// even) in magic form. This equals clamp(rne(v / Delta) + z, 0, span) except
// where v / Delta lies within ~1e-6 of a rounding boundary.
// clip in (0, 1] shrinks the group's range before the step is taken (1: none).
template <int CPT, int GL>
__device__ __forceinline__ void fq_group(const float (&v)[CPT], int bits, bool symmetric, FqGroup<CPT>& r,
                                         float clip = 1.0f) {
  const float span = (float)((1 << bits) - 1);
  const float inv_span = inv_levels(bits);
  float a, b;  // y = sat(v * a + b)
  if (symmetric) {
    const float amax = clip * group_max<GL>(fmaxf(maxN(v), -minN(v)));
    const float half = (float)(1 << (bits - 1));  // -qmin
    r.delta = fmaxf(amax, kEpsDelta) * inv_levels(bits - 1);
    const float inv = rcp_approx(r.delta);
    r.zero = half;
    r.off = kRoundMagic + half;
    a = inv * inv_span;
    b = half * inv_span;  // q - qmin = rne(v / Delta) + 2^(b-1)
  } else {
    const float mx = clip * group_max<GL>(maxN(v));
    const float mn = clip * group_min<GL>(minN(v));
    r.delta = fmaxf(mx - mn, kEpsDelta) * inv_span;
    const float inv = rcp_approx(r.delta);
    r.zero = fminf(fmaxf(__fmaf_rn(-mn, inv, kRoundMagic) - kRoundMagic, 0.f), span);  // clamp(rne(-min / Delta))
    r.off = kRoundMagic + r.zero;
    a = inv * inv_span;
    b = r.zero * inv_span;
  }
#pragma unroll
  for (int j = 0; j < CPT; ++j) r.c[j] = __fmaf_rn(fma_sat(v[j], a, b), span, kRoundMagic);
}

// The same quantiser with the group's extremes given (mx = max v, mn = min v;
// e.g. of the whole layer for per-tensor quantisation) instead of reduced over
// lanes: the formulas of fq_group, kept apart so that fq_group's code (the
// search's hot loop) stays as it is.
template <int CPT>
__device__ __forceinline__ void fq_from_extremes(const float (&v)[CPT], int bits, bool symmetric, FqGroup<CPT>& r,
                                                 float mx, float mn, float clip) {
  const float span = (float)((1 << bits) - 1);
  const float inv_span = inv_levels(bits);
  float a, b;
  if (symmetric) {
    const float amax = clip * fmaxf(mx, -mn);
    const float half = (float)(1 << (bits - 1));
    r.delta = fmaxf(amax, kEpsDelta) * inv_levels(bits - 1);
    const float inv = rcp_approx(r.delta);
    r.zero = half;
    r.off = kRoundMagic + half;
    a = inv * inv_span;
    b = half * inv_span;
  } else {
    mx *= clip;
    mn *= clip;
    r.delta = fmaxf(mx - mn, kEpsDelta) * inv_span;
    const float inv = rcp_approx(r.delta);
    r.zero = fminf(fmaxf(__fmaf_rn(-mn, inv, kRoundMagic) - kRoundMagic, 0.f), span);
    r.off = kRoundMagic + r.zero;
    a = inv * inv_span;
    b = r.zero * inv_span;
  }
#pragma unroll
  for (int j = 0; j < CPT; ++j) r.c[j] = __fmaf_rn(fma_sat(v[j], a, b), span, kRoundMagic);
}

// Dequantised value v_hat of element j ((q - z) Delta, or q Delta when symmetric).
template <int CPT>
__device__ __forceinline__ float fq_dequant(const FqGroup<CPT>& r, int j) {
  return (r.c[j] - r.off) * r.delta;
}

// Stored (unsigned) code of element j.
template <int CPT>
__device__ __forceinline__ unsigned fq_code(const FqGroup<CPT>& r, int j) {
  return (unsigned)(r.c[j] - kRoundMagic);
}

// Word q of the packed codes: nibble j holds the code of element 8q + j.
// A magic-form code c = 1.5*2^23 + code (0 <= code < 2^22) has the fp32 bit
// pattern 0x4B400000 + code, so sum_j bits(c_j) 16^j (mod 2^32) is the word
// plus the constant 0x4B400000 * 0x11111111: a Horner chain of integer
// multiply-adds and one subtraction, with no float-to-integer conversion.
constexpr uint32_t kMagicBits = 0x4B400000u;  // fp32 bits of kRoundMagic
constexpr uint32_t kMagicWordBias = (uint32_t)((unsigned long long)kMagicBits * 0x11111111ull);

template <int CPT>
__device__ __forceinline__ uint32_t fq_word(const FqGroup<CPT>& r, int q) {
  uint32_t acc = __float_as_uint(r.c[8 * q + 7]);
#pragma unroll
  for (int j = 6; j >= 0; --j) acc = acc * 16u + __float_as_uint(r.c[8 * q + j]);
  return acc - kMagicWordBias;
}

}  // namespace awq
