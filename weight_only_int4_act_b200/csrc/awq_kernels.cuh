// SIMT kernels of the AWQ search path (everything except the tensor-core
// products): activation statistics, candidate scales, the fake-quantised dW
// stack, the fixed-order loss reduction with argmin, and the pack.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "check.cuh"
#include "fq.cuh"
#include "ptx.cuh"

namespace awq {

constexpr int ERR_NONFINITE = 0x201;
constexpr int MAX_ALPHA = 64;

struct AlphaGrid {
  double v[MAX_ALPHA];
};

__device__ __forceinline__ void unpack_bf16x8(const uint4 u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    f[2 * h] = __uint_as_float(w[h] << 16);
    f[2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
  }
}

// ---------------------------------------------------------------------------
// a1: a[i] = (1/N) sum_t |X[t, i]|   ([P1] 激活感知 Omega_i, [P5] §1.2)
// Block = 256 threads covering 256 columns (each lane 8 columns, 16-byte
// loads; warps take interleaved rows) and `rows_per_chunk` rows. Each thread
// sums 8 rows in fp32, then accumulates in fp64; the 8 warps are combined in a
// fixed order and the chunk's fp64 column sums are written to `part`.
// ---------------------------------------------------------------------------
constexpr int STATS_THREADS = 256;
constexpr int STATS_COLS = 256;
constexpr int STATS_FINAL_THREADS = 256;
constexpr int STATS_UNROLL = 8;  // rows summed in fp32 (and loads in flight) per thread and step

__global__ void __launch_bounds__(STATS_THREADS) act_absmean_partial(const __nv_bfloat16* __restrict__ X, long long N,
                                                                     int d_in, int rows_per_chunk,
                                                                     double* __restrict__ part) {
  __shared__ double red[STATS_THREADS / 32][STATS_COLS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = blockIdx.x * STATS_COLS + lane * 8;
  const long long r0 = (long long)blockIdx.y * rows_per_chunk;
  const long long r1 = min(N, r0 + rows_per_chunk);
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (col < d_in) {
    const __nv_bfloat16* base = X + col;
    for (long long r = r0 + warp; r < r1; r += STATS_UNROLL * 8) {
      uint4 u[STATS_UNROLL];
#pragma unroll
      for (int k = 0; k < STATS_UNROLL; ++k) {
        const long long rr = r + 8 * k;
        u[k] = (rr < r1 && AWQ_SPAN_OK(rr * d_in + col, 8, N * d_in, BS_STATS_X))
                   ? __ldcs(reinterpret_cast<const uint4*>(base + rr * d_in))
                   : make_uint4(0, 0, 0, 0);
      }
      float s[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int k = 0; k < STATS_UNROLL; ++k) {
        float f[8];
        unpack_bf16x8(u[k], f);
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j] += fabsf(f[j]);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] += (double)s[j];
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[warp][lane * 8 + j] = acc[j];
  __syncthreads();
  const int c = blockIdx.x * STATS_COLS + threadIdx.x;
  if (c < d_in) {
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < STATS_THREADS / 32; ++w) t += red[w][threadIdx.x];
    if (AWQ_IDX_OK((long long)blockIdx.y * d_in + c, (long long)gridDim.y * d_in, BS_STATS_PART))
      part[(long long)blockIdx.y * d_in + c] = t;
  }
}

// a_i = (sum over row chunks of the partials) / N. A block takes 32 channels;
// its 8 warps each sum every 8th chunk (chunk order within a warp), and the 8
// sums are added in warp order: a fixed tree, so the result depends only on
// the shapes, with 8 times fewer dependent loads per thread than one serial
// sum per channel.
constexpr int FINAL_COLS = 32, FINAL_SLICES = STATS_FINAL_THREADS / 32;
__global__ void __launch_bounds__(STATS_FINAL_THREADS) act_absmean_final(const double* __restrict__ part, int n_chunks,
                                                                         long long N, int d_in, float* __restrict__ a) {
  __shared__ double red[FINAL_SLICES][FINAL_COLS];
  const int cl = threadIdx.x & 31, sl = threadIdx.x >> 5;
  const int c = blockIdx.x * FINAL_COLS + cl;
  double t = 0.0;
  if (c < d_in)
    for (int k = sl; k < n_chunks; k += FINAL_SLICES)
      if (AWQ_IDX_OK((long long)k * d_in + c, (long long)n_chunks * d_in, BS_STATS_PART))
        t += part[(long long)k * d_in + c];
  red[sl][cl] = t;
  __syncthreads();
  if (sl == 0 && c < d_in) {
    double u = red[0][cl];
#pragma unroll
    for (int j = 1; j < FINAL_SLICES; ++j) u += red[j][cl];
    a[c] = (float)(u / (double)N);
  }
}

// ---------------------------------------------------------------------------
// a2: s_k,i = t_k,i / sqrt(max_j t_k,j * min_j t_k,j) with t_k,i =
// max(a_i, eps)^alpha_k, and 1/s. ([P5] §4.1 s_i = a_i^alpha.) For alpha >= 0
// the power does not decrease as its base grows, so the largest and smallest
// t_k,j are the powers of the largest and smallest floored a_j: each block
// first takes those two extremes of a (d_in floats, read from L2), then each
// thread computes one element on its own. Grid: (column blocks of
// SCALES_THREADS, alpha). The power and the normalisation are taken in fp64
// and rounded once to fp32.
// ---------------------------------------------------------------------------
constexpr int SCALES_THREADS = 256;

__global__ void __launch_bounds__(SCALES_THREADS) candidate_scales(const float* __restrict__ a, int d_in,
                                                                   AlphaGrid grid, float eps_a,
                                                                   float* __restrict__ s_all,
                                                                   float* __restrict__ inv_all) {
  __shared__ double smax[SCALES_THREADS / 32], smin[SCALES_THREADS / 32];
  double mx = 0.0, mn = 1e300;
  for (int i = threadIdx.x; i < d_in; i += SCALES_THREADS) {
    const double v = fmax((double)a[i], (double)eps_a);
    mx = fmax(mx, v);
    mn = fmin(mn, v);
  }
  for (int off = 16; off > 0; off >>= 1) {
    mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, off));
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    smax[warp] = mx;
    smin[warp] = mn;
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < SCALES_THREADS / 32; ++w) {
    mx = fmax(mx, smax[w]);
    mn = fmin(mn, smin[w]);
  }
  const int k = blockIdx.y;
  const double alpha = grid.v[k];
  const double norm = sqrt(pow(mx, alpha) * pow(mn, alpha));
  const int i = blockIdx.x * SCALES_THREADS + threadIdx.x;
  if (i < d_in) {
    const double s = pow(fmax((double)a[i], (double)eps_a), alpha) / norm;
    s_all[(long long)k * d_in + i] = (float)s;
    inv_all[(long long)k * d_in + i] = (float)(1.0 / s);
  }
}

// Candidate scales given by the caller: s_all = s_cand, inv_all = 1 / s_cand;
// a non-positive or non-finite scale is recorded as a non-finite error.
__global__ void set_candidate_scales(const float* __restrict__ s_cand, long long n, float* __restrict__ s_all,
                                     float* __restrict__ inv_all, int* err) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float v = s_cand[i];
    if (!(v > 0.f) || !isfinite(v)) atomicCAS(err, 0, ERR_NONFINITE);
    s_all[i] = v;
    inv_all[i] = 1.0f / v;
  }
}

// ---------------------------------------------------------------------------
// a3: dW[k][r][:] = Q(W_r S_k) S_k^-1 - W_r as bf16, for every alpha k.
// ([P1] 缩放保护 W~ = sW, W^ = Q(W~)/s; [P5] §2.2 Q(WS)S^-1.)
// One thread = CPT consecutive channels of ROWS consecutive rows: W is read
// once and reused for every alpha, and each alpha's scales are loaded once for
// the ROWS rows. Rows d_out..d_out_pad-1 of each slice come out as zeros (their
// w = 0 dequantises to exactly 0).
// ---------------------------------------------------------------------------
#ifndef AWQ_FQ_ROWS
#define AWQ_FQ_ROWS 4
#endif
#ifndef AWQ_FQ_CPT
#define AWQ_FQ_CPT 16
#endif
constexpr int FQ_ROWS = AWQ_FQ_ROWS;
constexpr int FQ_CPT = AWQ_FQ_CPT;  // channels per thread (at most; never more than g)

template <int CPT>
__device__ __forceinline__ void load_f32(const float* __restrict__ p, float (&f)[CPT]) {
#pragma unroll
  for (int q = 0; q < CPT / 4; ++q) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(p) + q);
    f[4 * q] = x.x;
    f[4 * q + 1] = x.y;
    f[4 * q + 2] = x.z;
    f[4 * q + 3] = x.w;
  }
}

struct ClipTable {
  float c[MAX_ALPHA];  // clip ratio of each candidate (1: none)
};

// PT (per tensor): every candidate's step comes from the layer-wide extremes
// ext[2k] = max v, ext[2k+1] = min v (tensor_extremes) instead of a group.
template <int CPT, int ROWS, int GL, bool PT = false>
__global__ void __launch_bounds__(256, 2) fake_quant_delta(const __nv_bfloat16* __restrict__ W, int d_out, int d_in,
                                                           int d_out_pad, const float* __restrict__ s_all,
                                                           const float* __restrict__ inv_all, int n_alpha, int bits,
                                                           int symmetric, __nv_bfloat16* __restrict__ dW,
                                                           ClipTable clips, const float* __restrict__ ext) {
  const int chunks = d_in / CPT;
  const long long total = (long long)(d_out_pad / ROWS) * chunks;
  const long long warp_global = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  const bool sym = symmetric != 0;
  const long long slice = (long long)d_out_pad * d_in;
  for (long long base = warp_global * 32; base < total; base += n_warps * 32) {
    const long long u = base + lane;
    const bool active = u < total;
    const int rq = active ? (int)(u / chunks) : 0;
    const int c0 = active ? (int)(u - (long long)rq * chunks) * CPT : 0;
    const int row0 = rq * ROWS;
    float w[ROWS][CPT];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      const bool real = active && row0 + r < d_out;
#pragma unroll
      for (int q = 0; q < CPT / 8; ++q) {
        float f[8];
        const bool ld = real && AWQ_SPAN_OK((long long)(row0 + r) * d_in + c0 + 8 * q, 8, (long long)d_out * d_in,
                                            BS_FQ_W);
        unpack_bf16x8(ld ? __ldg(reinterpret_cast<const uint4*>(W + (long long)(row0 + r) * d_in + c0) + q)
                         : make_uint4(0, 0, 0, 0),
                      f);
#pragma unroll
        for (int j = 0; j < 8; ++j) w[r][8 * q + j] = f[j];
      }
    }
    __nv_bfloat16* out_base = dW + (long long)row0 * d_in + c0;
    for (int k = 0; k < n_alpha; ++k) {
      float s[CPT], is[CPT];
      if (AWQ_SPAN_OK((long long)k * d_in + c0, CPT, (long long)n_alpha * d_in, BS_FQ_S)) {
        load_f32<CPT>(s_all + (long long)k * d_in + c0, s);
        load_f32<CPT>(inv_all + (long long)k * d_in + c0, is);
      } else {
#pragma unroll
        for (int j = 0; j < CPT; ++j) s[j] = is[j] = 0.f;
      }
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        float v[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) v[j] = w[r][j] * s[j];
        FqGroup<CPT> fr;
        if constexpr (PT)
          fq_from_extremes<CPT>(v, bits, sym, fr, ext[2 * k], ext[2 * k + 1], clips.c[k]);
        else
          fq_group<CPT, GL>(v, bits, sym, fr, clips.c[k]);
#pragma unroll
        for (int q = 0; q < CPT / 8; ++q) {
          uint32_t out[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int j = 8 * q + 2 * h;
            __nv_bfloat162 p = __floats2bfloat162_rn(fq_dequant(fr, j) * is[j] - w[r][j],
                                                     fq_dequant(fr, j + 1) * is[j + 1] - w[r][j + 1]);
            out[h] = *reinterpret_cast<uint32_t*>(&p);
          }
          if (active && AWQ_SPAN_OK((long long)(row0 + r) * d_in + c0 + 8 * q + k * slice, 8, n_alpha * slice,
                                    BS_FQ_DW))
            __stcs(reinterpret_cast<uint4*>(out_base + k * slice + (long long)r * d_in) + q,
                   make_uint4(out[0], out[1], out[2], out[3]));
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// a6, first half: per-row losses l[k][r] = sum over column tiles of the
// contraction's partials (fp64, column tiles in order), optional fp32 copy,
// and per-block fp64 sums (fixed tree) per alpha.
// part layout: [n_blocks_n][M] with M = n_alpha * d_out_pad, row = k*d_out_pad + r.
// ---------------------------------------------------------------------------
constexpr int REDUCE_THREADS = 256;

__global__ void __launch_bounds__(REDUCE_THREADS) row_loss_reduce(const float* __restrict__ part, int n_blocks_n,
                                                                  long long M, int d_out, int d_out_pad,
                                                                  float* __restrict__ row_losses,
                                                                  double* __restrict__ block_sums) {
  __shared__ double red[REDUCE_THREADS];
  const int k = blockIdx.y;
  const int r = blockIdx.x * REDUCE_THREADS + threadIdx.x;
  double s = 0.0;
  if (r < d_out) {
    const long long m = (long long)k * d_out_pad + r;
    for (int nb = 0; nb < n_blocks_n; ++nb)
      if (AWQ_IDX_OK((long long)nb * M + m, (long long)n_blocks_n * M, BS_LOSS_PART))
        s += (double)part[(long long)nb * M + m];
    if (row_losses && AWQ_IDX_OK((long long)k * d_out + r, (long long)gridDim.y * d_out, BS_LOSS_ROW))
      row_losses[(long long)k * d_out + r] = (float)s;
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = REDUCE_THREADS / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) block_sums[(long long)k * gridDim.x + blockIdx.x] = red[0];
}

// a6, second half: losses, argmin (lowest index on ties), s_best. One block.
__global__ void loss_argmin(const double* __restrict__ block_sums, int n_chunks, int n_alpha,
                            const float* __restrict__ s_all, int d_in, float* __restrict__ losses,
                            double* __restrict__ losses64, int* __restrict__ best_out, float* __restrict__ s_best,
                            int* err) {
  __shared__ double L[MAX_ALPHA];
  __shared__ int best_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int k = warp; k < n_alpha; k += nw) {
    double s = 0.0;
    for (int c = lane; c < n_chunks; c += 32) s += block_sums[(long long)k * n_chunks + c];
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) L[k] = s;
  }
  __syncthreads();
  if (warp == 0) {
    // warp-shuffle argmin over (loss, index); ties go to the lower index
    double bv = INFINITY;
    int bi = MAX_ALPHA;
    bool finite = true;
    for (int k = lane; k < n_alpha; k += 32) {
      const double v = L[k];
      if (!isfinite(v)) finite = false;
      if (v < bv) {
        bv = v;
        bi = k;
      }
    }
    for (int off = 16; off > 0; off >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (ov < bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    finite = __all_sync(0xffffffffu, finite);
    if (lane == 0) {
      best_sh = finite ? bi : -1;
      *best_out = best_sh;
      if (!finite && err) atomicCAS(err, 0, ERR_NONFINITE);
    }
    for (int k = lane; k < n_alpha; k += 32) {
      losses[k] = (float)L[k];
      losses64[k] = L[k];
    }
  }
  __syncthreads();
  const int b = best_sh;
  for (int i = threadIdx.x; i < d_in; i += blockDim.x)
    s_best[i] = (b >= 0 && AWQ_IDX_OK((long long)b * d_in + i, (long long)n_alpha * d_in, BS_ARGMIN_S))
                    ? s_all[(long long)b * d_in + i]
                    : __int_as_float(0x7fc00000);
}

// ---------------------------------------------------------------------------
// a6 for several layers sharing X (rows of W split into segments, one layer
// each): fp64 loss per (segment, alpha) in a fixed order, then an argmin per
// segment. part layout as for row_loss_reduce.
// ---------------------------------------------------------------------------
// a6 for several layers sharing X (the segmented search): per-row fp64 losses
// (column tiles summed in order, one thread per row), then per segment and
// alpha a fixed-order sum of its rows, then the argmin per segment. part
// layout as for row_loss_reduce.
// ---------------------------------------------------------------------------
constexpr int MAX_SEG = 16;

struct SegTable {
  int start[MAX_SEG + 1];  // segment s holds rows [start[s], start[s+1])
};

__global__ void __launch_bounds__(REDUCE_THREADS) row_loss_rows(const float* __restrict__ part, int n_blocks_n,
                                                                long long M, int d_out, int d_out_pad,
                                                                float* __restrict__ row_losses,
                                                                double* __restrict__ rows64) {
  const int k = blockIdx.y;
  const int r = blockIdx.x * REDUCE_THREADS + threadIdx.x;
  if (r >= d_out) return;
  const long long m = (long long)k * d_out_pad + r;
  double s = 0.0;
  for (int nb = 0; nb < n_blocks_n; ++nb)
    if (AWQ_IDX_OK((long long)nb * M + m, (long long)n_blocks_n * M, BS_LOSS_PART))
      s += (double)part[(long long)nb * M + m];
  if (row_losses && AWQ_IDX_OK((long long)k * d_out + r, (long long)gridDim.y * d_out, BS_LOSS_ROW))
    row_losses[(long long)k * d_out + r] = (float)s;
  if (AWQ_IDX_OK(m, M, BS_LOSS_PART)) rows64[m] = s;
}

// seg_sums[k][sg] = sum of the row losses of segment sg at alpha k (thread-
// strided, then a fixed tree)
__global__ void __launch_bounds__(REDUCE_THREADS) segment_loss_reduce(const double* __restrict__ rows64, long long M,
                                                                      int d_out_pad, SegTable seg,
                                                                      double* __restrict__ seg_sums) {
  __shared__ double red[REDUCE_THREADS];
  const int sg = blockIdx.x, k = blockIdx.y;
  double acc = 0.0;
  for (int r = seg.start[sg] + threadIdx.x; r < seg.start[sg + 1]; r += REDUCE_THREADS) {
    const long long m = (long long)k * d_out_pad + r;
    if (AWQ_IDX_OK(m, M, BS_LOSS_PART)) acc += rows64[m];
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = REDUCE_THREADS / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) seg_sums[(long long)k * MAX_SEG + sg] = red[0];
}

// One block per segment: warp 0 takes losses[sg][k] and the warp-shuffle
// argmin (lowest k on ties); the block copies s_best[sg][:] = s(alpha_best).
__global__ void __launch_bounds__(256) segment_argmin(const double* __restrict__ seg_sums, int n_seg, int n_alpha,
                                                      const float* __restrict__ s_all, int d_in,
                                                      float* __restrict__ losses, int* __restrict__ best_out,
                                                      float* __restrict__ s_best, int* err) {
  __shared__ int b_shared;
  const int sg = blockIdx.x, lane = threadIdx.x & 31;
  if (sg >= n_seg) return;
  if (threadIdx.x < 32) {
    double bv = INFINITY;
    int bi = MAX_ALPHA;
    bool finite = true;
    for (int k = lane; k < n_alpha; k += 32) {
      const double v = seg_sums[(long long)k * MAX_SEG + sg];
      losses[(long long)sg * n_alpha + k] = (float)v;
      if (!isfinite(v)) finite = false;
      if (v < bv) {
        bv = v;
        bi = k;
      }
    }
    for (int off = 16; off > 0; off >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (ov < bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    finite = __all_sync(0xffffffffu, finite);
    const int b = finite ? bi : -1;
    if (lane == 0) {
      best_out[sg] = b;
      b_shared = b;
      if (!finite && err) atomicCAS(err, 0, ERR_NONFINITE);
    }
  }
  __syncthreads();
  const int b = b_shared;
  for (int i = threadIdx.x; i < d_in; i += blockDim.x)
    s_best[(long long)sg * d_in + i] =
        (b >= 0 && AWQ_IDX_OK((long long)b * d_in + i, (long long)n_alpha * d_in, BS_ARGMIN_S))
            ? s_all[(long long)b * d_in + i]
            : __int_as_float(0x7fc00000);
}

// ---------------------------------------------------------------------------
// Failure path of the bounded waits: one thread waits on an mbarrier that no
// one arrives at, through the same mbar_wait the GEMMs use; it gives up after
// AWQ_WAIT_LIMIT_NS and records ERR_WAIT_SELFTEST in *err.
// ---------------------------------------------------------------------------
constexpr int ERR_WAIT_SELFTEST = 0x401;

__global__ void bounded_wait_selftest(int* err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, err, ERR_WAIT_SELFTEST);
}

// ---------------------------------------------------------------------------
// Per-tensor quantisation: the layer-wide extremes of v = w s for each
// candidate. With every s_i > 0, max over (r, i) of fp32(w[r, i] s_i) is
// max over i of fp32(colmax_i s_i) (fp32 rounding is monotone), so one pass
// over W for column extremes serves every candidate.
// ---------------------------------------------------------------------------
// Order-preserving map of floats to unsigned keys (for atomicMax / atomicMin).
__device__ __forceinline__ uint32_t ord_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord_val(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// kmax[i] / kmin[i]: keys of max / min over rows of column i (kmax zeroed,
// kmin filled with 0xFF before the launch). Thread: 8 columns x a row block.
__global__ void col_minmax(const __nv_bfloat16* __restrict__ W, int d_out, int d_in, int rows_per_block,
                           uint32_t* __restrict__ kmax, uint32_t* __restrict__ kmin) {
  const int c8 = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (c8 >= d_in || !AWQ_SPAN_OK(c8, 8, d_in, BS_MINMAX_KEY)) return;
  const int r0 = blockIdx.y * rows_per_block;
  const int r1 = min(d_out, r0 + rows_per_block);
  float mx[8], mn[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    mx[j] = -INFINITY;
    mn[j] = INFINITY;
  }
  for (int r = r0; r < r1; ++r) {
    float f[8];
    if (!AWQ_SPAN_OK((long long)r * d_in + c8, 8, (long long)d_out * d_in, BS_MINMAX_W)) continue;
    unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(W + (long long)r * d_in + c8)), f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      mx[j] = fmaxf(mx[j], f[j]);
      mn[j] = fminf(mn[j], f[j]);
    }
  }
  if (r0 >= r1) return;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    atomicMax(&kmax[c8 + j], ord_key(mx[j]));
    atomicMin(&kmin[c8 + j], ord_key(mn[j]));
  }
}

// ext[2k] = max_i fp32(colmax_i s_k[i]), ext[2k + 1] = min_i fp32(colmin_i s_k[i]);
// one block per candidate.
__global__ void tensor_extremes(const uint32_t* __restrict__ kmax, const uint32_t* __restrict__ kmin,
                                const float* __restrict__ s_all, int d_in, float* __restrict__ ext) {
  const float* s = s_all + (long long)blockIdx.x * d_in;
  float mx = -INFINITY, mn = INFINITY;
  for (int i = threadIdx.x; i < d_in; i += blockDim.x) {
    mx = fmaxf(mx, ord_val(kmax[i]) * s[i]);
    mn = fminf(mn, ord_val(kmin[i]) * s[i]);
  }
  __shared__ float smx[32], smn[32];
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    smx[warp] = mx;
    smn[warp] = mn;
  }
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    mx = lane < nw ? smx[lane] : -INFINITY;
    mn = lane < nw ? smn[lane] : INFINITY;
    for (int o = 16; o > 0; o >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    if (lane == 0) {
      ext[2 * blockIdx.x] = mx;
      ext[2 * blockIdx.x + 1] = mn;
    }
  }
}

// ---------------------------------------------------------------------------
// Per-group clipping search. s_all[k] = s, inv_all[k] = 1/s for k < n.
// ---------------------------------------------------------------------------
__global__ void repeat_scales(const float* __restrict__ s, int d_in, int n, float* __restrict__ s_all,
                              float* __restrict__ inv_all, int* err) {
  const long long total = (long long)n * d_in;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const float v = s[i % d_in];
    if (!(v > 0.f) || !isfinite(v)) atomicCAS(err, 0, ERR_NONFINITE);
    s_all[i] = v;
    inv_all[i] = 1.0f / v;
  }
}

// err[c][r][j] = sum of the group's 32-column partials (fp64, in order) for
// clip candidate c; best[r][j] = argmin over c (lowest index on ties).
// part layout: part[chunk32 * part_ld + c * d_out_pad + r]. One thread per
// (group j, row r), rows fastest.
__global__ void group_clip_argmin(const float* __restrict__ part, long long part_ld, int d_out, int d_out_pad,
                                  int n_groups, int chunks_per_group, int n_clip, uint8_t* __restrict__ best,
                                  float* __restrict__ group_err, int* err) {
  const long long total = (long long)n_groups * d_out;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int j = (int)(i / d_out), r = (int)(i - (long long)j * d_out);
    double bv = INFINITY;
    int bi = 0;
    bool finite = true;
    for (int c = 0; c < n_clip; ++c) {
      double e = 0.0;
      for (int u = 0; u < chunks_per_group; ++u)
        if (AWQ_IDX_OK((long long)c * d_out_pad + r, part_ld, BS_CLIP_PART) &&
            AWQ_IDX_OK(j * chunks_per_group + u, (long long)n_groups * chunks_per_group, BS_CLIP_PART))
          e += (double)part[(long long)(j * chunks_per_group + u) * part_ld + (long long)c * d_out_pad + r];
      if (!isfinite(e)) finite = false;
      if (group_err && AWQ_IDX_OK(((long long)c * d_out + r) * n_groups + j, (long long)n_clip * d_out * n_groups,
                                  BS_CLIP_OUT))
        group_err[((long long)c * d_out + r) * n_groups + j] = (float)e;
      if (e < bv) {
        bv = e;
        bi = c;
      }
    }
    if (!finite) atomicCAS(err, 0, ERR_NONFINITE);
    if (AWQ_IDX_OK((long long)r * n_groups + j, (long long)d_out * n_groups, BS_CLIP_OUT))
      best[(long long)r * n_groups + j] = (uint8_t)bi;
  }
}

// ---------------------------------------------------------------------------
// a7: pack. Codes of Q(W S) (same quantiser as the search), 8 nibbles per
// uint32 (channel 8w+j in bits 4j..4j+3), fp16 step and zero per group.
// ([P2] §2.1 INT4 with fp16 scale, §4.2 packed 4-bit storage; [P4] §三.)
// ---------------------------------------------------------------------------
// One thread = CPT consecutive channels of PACK_ROWS consecutive rows (the
// scales are loaded once for all of them; PACK_ROWS independent loads of W are
// in flight per thread). Each row yields CPT/8 consecutive words.
constexpr int PACK_ROWS = 4;

// PT (per tensor): the step from the layer-wide extremes ext[0] = max v,
// ext[1] = min v; one step and zero point (scales[0], zeros[0]).
template <int CPT, int GL, bool PT = false>
__global__ void __launch_bounds__(256) quantize_pack(const __nv_bfloat16* __restrict__ W, const float* __restrict__ s,
                                                     int d_out, int d_in, int bits, int symmetric,
                                                     uint32_t* __restrict__ qweight, __half* __restrict__ scales,
                                                     __half* __restrict__ zeros, float clip,
                                                     const uint8_t* __restrict__ group_clip, ClipTable clips,
                                                     const float* __restrict__ ext) {
  const int chunks = d_in / CPT;
  const int row_groups = (d_out + PACK_ROWS - 1) / PACK_ROWS;
  // A warp task is 32 consecutive chunks (lanes) of one group of PACK_ROWS rows,
  // task t = (row group t / citers, chunk pass t % citers). Warps stride over
  // the tasks (the grid works on neighbouring rows at any time); the stride is
  // split into row groups and passes once, so stepping needs no division.
  const int citers = (chunks + 31) >> 5;
  const int n_warps = (int)((gridDim.x * blockDim.x) >> 5);
  const int warp_global = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int step_rg = n_warps / citers, step_ci = n_warps - step_rg * citers;
  int rg = warp_global / citers;
  int ci = warp_global - rg * citers;
  const int lane = threadIdx.x & 31;
  const bool sym = symmetric != 0;
  const int groups = d_in / (GL * CPT);
  const int words = d_in / 8;
  // W of the next task is loaded while this one is quantised (one task of
  // loads in flight per warp during the arithmetic)
  auto load_w = [&](int rg_, int ci_, uint4 (&dst)[PACK_ROWS][CPT / 8]) {
    const int ch = ci_ * 32 + lane;
    const bool act = rg_ < row_groups && ch < chunks;
    const int cc = act ? ch * CPT : 0;
#pragma unroll
    for (int r = 0; r < PACK_ROWS; ++r)
#pragma unroll
      for (int q = 0; q < CPT / 8; ++q)
        dst[r][q] = (act && rg_ * PACK_ROWS + r < d_out &&
                     AWQ_SPAN_OK((long long)(rg_ * PACK_ROWS + r) * d_in + cc + 8 * q, 8, (long long)d_out * d_in,
                                 BS_PACK_W))
                        ? __ldcs(reinterpret_cast<const uint4*>(W + (long long)(rg_ * PACK_ROWS + r) * d_in + cc) + q)
                        : make_uint4(0, 0, 0, 0);
  };
  uint4 wnext[PACK_ROWS][CPT / 8];
  load_w(rg, ci, wnext);
  for (; rg < row_groups; rg += step_rg, ci += step_ci, rg += (ci >= citers), ci -= (ci >= citers) ? citers : 0) {
    const int chunk = ci * 32 + lane;
    const bool active = chunk < chunks;
    const int c0 = active ? chunk * CPT : 0;
    const int row0 = rg * PACK_ROWS;
    uint4 wraw[PACK_ROWS][CPT / 8];
#pragma unroll
    for (int r = 0; r < PACK_ROWS; ++r)
#pragma unroll
      for (int q = 0; q < CPT / 8; ++q) wraw[r][q] = wnext[r][q];
    {
      int ci2 = ci + step_ci, rg2 = rg + step_rg;
      if (ci2 >= citers) {
        ci2 -= citers;
        ++rg2;
      }
      load_w(rg2, ci2, wnext);
    }
    float sc[CPT];
    if (AWQ_SPAN_OK(c0, CPT, d_in, BS_PACK_S)) {
      load_f32<CPT>(s + c0, sc);
    } else {
#pragma unroll
      for (int j = 0; j < CPT; ++j) sc[j] = 0.f;
    }
#pragma unroll
    for (int r = 0; r < PACK_ROWS; ++r) {
      float v[CPT];
#pragma unroll
      for (int q = 0; q < CPT / 8; ++q) {
        float f[8];
        unpack_bf16x8(wraw[r][q], f);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[8 * q + j] = f[j] * sc[8 * q + j];
      }
      // per-group clip ratio (index into clips) when given, else the scalar one
      float c = clip;
      if (group_clip && active && row0 + r < d_out &&
          AWQ_IDX_OK((long long)(row0 + r) * groups + chunk / GL, (long long)d_out * groups, BS_PACK_CLIP)) {
        const int idx = group_clip[(long long)(row0 + r) * groups + chunk / GL];
        c = idx < MAX_ALPHA ? clips.c[idx] : 1.0f;
      }
      FqGroup<CPT> fr;
      if constexpr (PT)
        fq_from_extremes<CPT>(v, bits, sym, fr, ext[0], ext[1], c);
      else
        fq_group<CPT, GL>(v, bits, sym, fr, c);
      if (active && row0 + r < d_out) {
        const int row = row0 + r;
        uint32_t* wp = qweight + (long long)row * words + c0 / 8;
        uint32_t wd[CPT / 8];
#pragma unroll
        for (int q = 0; q < CPT / 8; ++q) wd[q] = fq_word(fr, q);
        if (AWQ_SPAN_OK((long long)row * words + c0 / 8, CPT / 8, (long long)d_out * words, BS_PACK_Q)) {
          if constexpr (CPT == 16) {
            __stcs(reinterpret_cast<uint2*>(wp), make_uint2(wd[0], wd[1]));  // 8-byte aligned: c0 % 16 == 0
          } else {
#pragma unroll
            for (int q = 0; q < CPT / 8; ++q) __stcs(wp + q, wd[q]);
          }
        }
        if (PT ? (row == 0 && chunk == 0) : (chunk & (GL - 1)) == 0) {
          const long long gidx = PT ? 0 : (long long)row * groups + chunk / GL;
          if (AWQ_IDX_OK(gidx, PT ? 1 : (long long)d_out * groups, BS_PACK_SZ)) {
            scales[gidx] = __float2half_rn(fr.delta);
            zeros[gidx] = __float2half_rn(fr.zero);
          }
        }
      }
    }
  }
}

}  // namespace awq
