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
// Arithmetic is fp32; Delta is the range times the fp32 constant 1/levels and
// v / Delta is taken as v * (1 / Delta) (correctly rounded reciprocal).
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

__device__ __forceinline__ void fq_group8(const float (&v)[8], int bits, bool symmetric, int gl, FqResult& r) {
  if (symmetric) {
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
    for (int off = 1; off < gl; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float qmax = (float)((1 << (bits - 1)) - 1);
    const float qmin = -(float)(1 << (bits - 1));
    r.delta = fmaxf(amax, kEpsDelta) * inv_levels(bits - 1);
    const float inv = __frcp_rn(r.delta);
    r.zero = -qmin;
#pragma unroll
    for (int j = 0; j < 8; ++j) r.q[j] = fminf(fmaxf(rintf(v[j] * inv), qmin), qmax);
  } else {
    float mx = v[0], mn = v[0];
#pragma unroll
    for (int j = 1; j < 8; ++j) {
      mx = fmaxf(mx, v[j]);
      mn = fminf(mn, v[j]);
    }
    for (int off = 1; off < gl; off <<= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    }
    const float levels = (float)((1 << bits) - 1);
    r.delta = fmaxf(mx - mn, kEpsDelta) * inv_levels(bits);
    const float inv = __frcp_rn(r.delta);
    r.zero = fminf(fmaxf(rintf(-mn * inv), 0.f), levels);
#pragma unroll
    for (int j = 0; j < 8; ++j) r.q[j] = fminf(fmaxf(rintf(v[j] * inv) + r.zero, 0.f), levels);
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
