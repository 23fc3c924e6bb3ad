// Group-wise uniform quantiser shared by the search (fake quantisation) and
// the pack kernel, so that both decide every code the same way.
//
// One thread holds 8 consecutive input channels of one row; a group of g
// channels is g/8 consecutive lanes of a warp (g/8 a power of two <= 32, and
// groups never straddle warps). All 32 lanes must call fq_group8 together
// (the group reductions are full-warp shuffles); lanes without data pass
// neutral values (zeros) and belong to groups that are wholly inactive.
//
// Quantiser ([P1] 量化基础, [P2] §2.1, [P4] §三, [P5] §2.3):
//   symmetric : Delta = max(max|v|, eps) / (2^(b-1) - 1)
//               q = clamp(rne(v / Delta), -2^(b-1), 2^(b-1) - 1), v_hat = q Delta
//   asymmetric: Delta = max(max v - min v, eps) / (2^b - 1)
//               z = clamp(rne(-min v / Delta), 0, 2^b - 1)
//               q = clamp(rne(v / Delta) + z, 0, 2^b - 1),   v_hat = (q - z) Delta
// Arithmetic is fp32; Delta is the range times the fp32 constant 1/levels,
// 1/Delta is the correctly rounded reciprocal, and rne(v / Delta) is rounded
// from the exact product v * (1/Delta). GL = g/8 lanes form one group.
#pragma once
#include <cuda_runtime.h>

namespace awq {

constexpr float kEpsDelta = 1e-8f;

// 1 / (2^b - 1) rounded to fp32, for b = 1..4 (the step is range * this).
__device__ __forceinline__ float inv_levels(int b) {
  return b == 4 ? (1.0f / 15.0f) : b == 3 ? (1.0f / 7.0f) : b == 2 ? (1.0f / 3.0f) : 1.0f;
}

struct FqResult {
  float delta;  // quantisation step of the group
  float zero;   // asymmetric: z; symmetric: 2^(b-1) (the stored zero)
  float q[8];   // asymmetric: stored code in [0, 2^b-1]; symmetric: signed q
};

// Round-to-nearest-even to an integer by the fp32 "magic number" method: for
// |x| < 2^22, x + 1.5*2^23 has no fraction bits left, so the addition itself
// rounds x to the nearest integer (ties to even), which subtracting the
// constant recovers exactly. Here the addition is fused with the product
// v * inv (one rounding of the exact product), which keeps the work on the
// full-rate FMA pipe.
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

template <int GL>
__device__ __forceinline__ void fq_group8(const float (&v)[8], int bits, bool symmetric, FqResult& r) {
  if (symmetric) {
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
    amax = group_max<GL>(amax);
    const float qmax = (float)((1 << (bits - 1)) - 1);
    const float qmin = -(float)(1 << (bits - 1));
    r.delta = fmaxf(amax, kEpsDelta) * inv_levels(bits - 1);
    const float inv = __frcp_rn(r.delta);
    r.zero = -qmin;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float t = __fmaf_rn(v[j], inv, kRoundMagic) - kRoundMagic;  // rne(v / Delta)
      r.q[j] = fminf(fmaxf(t, qmin), qmax);
    }
  } else {
    float mx = v[0], mn = v[0];
#pragma unroll
    for (int j = 1; j < 8; ++j) {
      mx = fmaxf(mx, v[j]);
      mn = fminf(mn, v[j]);
    }
    mx = group_max<GL>(mx);
    mn = group_min<GL>(mn);
    const float levels = (float)((1 << bits) - 1);
    r.delta = fmaxf(mx - mn, kEpsDelta) * inv_levels(bits);
    const float inv = __frcp_rn(r.delta);
    r.zero = fminf(fmaxf(__fmaf_rn(-mn, inv, kRoundMagic) - kRoundMagic, 0.f), levels);  // rne(-min / Delta)
    const float off = kRoundMagic - r.zero;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float t = __fmaf_rn(v[j], inv, kRoundMagic) - off;  // rne(v / Delta) + z
      r.q[j] = fminf(fmaxf(t, 0.f), levels);
    }
  }
}

// Dequantised value v_hat of element j.
__device__ __forceinline__ float fq_dequant(const FqResult& r, int j, bool symmetric) {
  return symmetric ? r.q[j] * r.delta : (r.q[j] - r.zero) * r.delta;
}

// Stored (unsigned) code of element j.
__device__ __forceinline__ unsigned fq_code(const FqResult& r, int j, bool symmetric) {
  return (unsigned)(symmetric ? r.q[j] + r.zero : r.q[j]);
}

}  // namespace awq
