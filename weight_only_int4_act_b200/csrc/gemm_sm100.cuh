// Persistent tcgen05 GEMM for sm_100a with the AWQ loss epilogues.
//
// D[m, n] = sum_k A[m, k] * B[n, k]   (A [M, K], B [N, K], both bf16 row-major,
// i.e. K-major operands), fp32 accumulation in tensor memory. Tiles are
// 128 x 256 (one CTA per SM, cta_group::1, M=128 N=256 K=16 instructions),
// K is staged 64 at a time through a 4-deep shared-memory ring filled by TMA
// (128-byte swizzle, no multicast).
//
// Warp roles (192 threads):
//   warp 0      one thread takes tile indices from the global counter, publishes
//               them to the other warps and issues the TMA loads of A and B;
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators) and
//               one thread issues tcgen05.mma, committing each stage back to
//               the loader and each finished tile to the epilogue;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4)..+31, i.e. tile rows), then one of
//     EPI_SUMSQ  part[n_blk][m] = sum_{n in tile} D[m,n]^2         (||dW X^T||^2)
//     EPI_DOT    part[n_blk][m] = sum_{n in tile} D[m,n] E[m,n]    (trace(dW G dW^T))
//     EPI_STORE  C[m, n] = bf16(D[m, n])                            (G = X^T X)
//     EPI_DOT32  as EPI_DOT, one partial per 32-column chunk          (per-group errors)
// The accumulator is released before the partials are written, so the next
// tile's MMAs overlap this tile's epilogue.
//
// Tiles are handed out dynamically in the order of a tile index t (an atomic
// counter; each CTA takes the next index when it starts a tile), so CTAs that
// draw short tiles simply take more of them. Indices walk groups of `group_n`
// N-blocks (M-major inside a group) so that the CTAs running at one time share
// A panels and a B slice in L2.
//
// Block-triangular modes (the Gram form uses the symmetry of G = X^T X, with
// 256-wide channel blocks J): TRI_LOWER_STORE computes only the tiles of G
// whose column block is <= their row block and stores G' = 2G on strictly
// lower blocks, G on diagonal blocks; TRI_K then stops the contraction of
// column tile J at k < 256(J+1), so that sum over tiles of (dW G')[m, J] dW[m, J]
// = dW G dW^T (each off-diagonal block pair counted once, doubled).
// Every wait is bounded (ptx.cuh); on a timeout the CTA records an error in
// *err, drains its in-flight TMA loads and MMAs, frees TMEM and returns.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace awq {

enum EpiMode { EPI_SUMSQ = 0, EPI_DOT = 1, EPI_STORE = 2, EPI_DOT32 = 3 };

constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 256;
constexpr int GEMM_BK = 64;
constexpr int GEMM_STAGES = 4;
constexpr int GEMM_THREADS = 192;
constexpr int GEMM_A_STAGE = GEMM_BM * GEMM_BK * 2;  // 16 KB
constexpr int GEMM_B_STAGE = GEMM_BN * GEMM_BK * 2;  // 32 KB
constexpr int GEMM_TMEM_COLS = 512;
constexpr int GEMM_MN_CHUNK = 64 * GEMM_BK * 2;  // MN-major: one 64-wide chunk of 64 k-rows (8 KB)
constexpr int GEMM_SMEM_BYTES = 1024 /* alignment slack */ + GEMM_STAGES * (GEMM_A_STAGE + GEMM_B_STAGE) + 256;

// error codes written to *err by the GEMM (distinct per wait site)
constexpr int ERR_WAIT_EMPTY = 0x101, ERR_WAIT_FULL = 0x102, ERR_WAIT_TEMPTY = 0x103, ERR_WAIT_TFULL = 0x104,
              ERR_WAIT_SCHED = 0x105;
constexpr int GEMM_SCHED_SLOTS = 4;  // tile indices published ahead of the MMA and epilogue warps

// TRI_DIAG_STORE: only the diagonal 256-blocks of G, stored compactly as
// C[m, j] = G[m, 256*(m/256) + j] (ldC = 256) with the entries whose row and
// column fall in different quantisation groups set to 0; TRI_DIAG: column
// tile J contracts k in [256J, 256J+256) of A against that compact B.
enum TriMode { TRI_NONE = 0, TRI_LOWER_STORE = 1, TRI_K = 2, TRI_DIAG_STORE = 3, TRI_DIAG = 4 };

struct GemmArgs {
  int M, N, K;                 // problem size (rows of A, rows of B, contraction length)
  int tri;                     // TriMode
  int num_tiles;               // tiles visited (all, or the lower block triangle)
  int n_blocks_m, n_blocks_n;  // ceil(M/128), ceil(N/256)
  int group_n;                 // raster group width in N-blocks
  float* part;                 // SUMSQ / DOT: part[n_blk * part_ld + m], per-row partial sums
  long long part_ld;
  const __nv_bfloat16* E;      // DOT: E[M, ldE]; element (m, n) multiplies D[m, n]
  long long ldE;
  __nv_bfloat16* C;            // STORE: C[M, ldC]
  long long ldC;
  int* err;                    // device error word
  int* tile_counter;           // dynamic tile counter, zero at launch
  int group;                   // TRI_DIAG_STORE: quantisation group size (divides 256)
  int tail_first;              // pair G' only: tiles from here on are split in K (num_tiles: no split)
  int tail_split;              // K pieces per split tile (tail_first < num_tiles)
  float* tail_part;            // fp32 partial tiles [(num_tiles - tail_first) * tail_split][256 x 256]
};

// Number of tiles of the lower block triangle with n_blocks_m row tiles of
// 128: row tile mb holds column tiles 0..(mb>>1).
__host__ __device__ inline long long tri_lower_tiles(long long n_blocks_m) {
  const long long q = n_blocks_m >> 1;
  return (n_blocks_m & 1) ? (q + 1) * (q + 1) : q * (q + 1);
}

__device__ __forceinline__ void gemm_tile_coords(int t, const GemmArgs& a, int& mb, int& nb) {
  if (a.tri == TRI_DIAG_STORE) {
    mb = t;
    nb = t >> 1;
    return;
  }
  if (a.tri == TRI_LOWER_STORE) {
    // rows 2q and 2q+1 each hold q+1 tiles; tiles before row 2q: q(q+1)
    int q = (int)((sqrtf(4.0f * (float)t + 1.0f) - 1.0f) * 0.5f);
    while ((long long)(q + 1) * (q + 2) <= t) ++q;
    while ((long long)q * (q + 1) > t) --q;
    const int r = t - q * (q + 1);
    if (r <= q) {
      mb = 2 * q;
      nb = r;
    } else {
      mb = 2 * q + 1;
      nb = r - (q + 1);
    }
    return;
  }
  const int gn = a.group_n;
  const int per_group = a.n_blocks_m * gn;
  const int g = t / per_group;
  const int first = g * gn;
  const int width = min(gn, a.n_blocks_n - first);
  const int r = t - g * per_group;
  mb = r / width;
  nb = first + (r - mb * width);
  if (a.tri == TRI_K) {
    // interleave long and short contractions: positions 0, 1, 2, 3, ... take
    // column tiles n-1, 0, n-2, 1, ..., so every group of tiles (and every
    // CTA's run of them) mixes both and a short tile's epilogue overlaps a
    // long tile's MMAs
    nb = (nb & 1) ? (nb >> 1) : a.n_blocks_n - 1 - (nb >> 1);
  }
}

__device__ __forceinline__ int gemm_num_kb(const GemmArgs& a, int nb) {
  int k = a.K;
  if (a.tri == TRI_K) k = min(k, (nb + 1) * GEMM_BN);
  if (a.tri == TRI_DIAG) k = min(GEMM_BN, a.K - nb * GEMM_BN);
  return (k + GEMM_BK - 1) / GEMM_BK;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// MN = false: A [M, K] and B [N, K] row-major (K-major operands), one TMA box
// of 64 x 128 (A) and 64 x 256 (B) rows per stage.
// MN = true: A and B are the same row-major [K, M] matrix read transposed
// (MN-major operands; G = X^T X straight from X), boxes of 64 (M or N) x 64
// (K) loaded at 64-column offsets: 2 for A and 4 for B per stage.
template <int MODE, bool MN = false>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_bf16_tcgen05(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + GEMM_STAGES * GEMM_A_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + GEMM_STAGES * GEMM_B_STAGE);
  // bars: full[S], empty[S], tfull[2], tempty[2], drain, sched_full[R], sched_empty[R]
  constexpr int NB = 2 * GEMM_STAGES + 5 + 2 * GEMM_SCHED_SLOTS;
  volatile int* tile_ring = reinterpret_cast<volatile int*>(bars + NB);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NB) + GEMM_SCHED_SLOTS;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + GEMM_STAGES + s); };
  auto tfull_bar = [&](int a) { return smem_u32(bars + 2 * GEMM_STAGES + a); };
  auto tempty_bar = [&](int a) { return smem_u32(bars + 2 * GEMM_STAGES + 2 + a); };
  const uint32_t drain_bar = smem_u32(bars + 2 * GEMM_STAGES + 4);
  auto sfull_bar = [&](int r) { return smem_u32(bars + 2 * GEMM_STAGES + 5 + r); };
  auto sempty_bar = [&](int r) { return smem_u32(bars + 2 * GEMM_STAGES + 5 + GEMM_SCHED_SLOTS + r); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < GEMM_STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4);
    }
    mbar_init(drain_bar, 1);
    for (int r = 0; r < GEMM_SCHED_SLOTS; ++r) {
      mbar_init(sfull_bar(r), 1);
      mbar_init(sempty_bar(r), 5);  // the MMA thread and one lane of each epilogue warp
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), GEMM_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = args.num_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- tile scheduler + TMA producer
      // Tiles are handed out dynamically (a global counter, zeroed before the
      // launch) and published to the MMA and epilogue warps through a ring of
      // tile indices; -1 ends the sequence.
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_parity = 0;  // bit s: stage s has been loaded; parity of its last load
      int slot = 0;
      uint32_t sphase = 0;
      bool ok = true;
      while (ok) {
        if (!mbar_wait(sempty_bar(slot), sphase ^ 1u, abort_flag, args.err, ERR_WAIT_SCHED)) break;
        int t = atomicAdd(args.tile_counter, 1);
        if (t >= num_tiles) t = -1;
        tile_ring[slot] = t;
        mbar_arrive(sfull_bar(slot));
        if (++slot == GEMM_SCHED_SLOTS) {
          slot = 0;
          sphase ^= 1u;
        }
        if (t < 0) break;
        int mb, nb;
        gemm_tile_coords(t, args, mb, nb);
        const int num_kb = gemm_num_kb(args, nb);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, args.err, ERR_WAIT_EMPTY)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(stage), GEMM_A_STAGE + GEMM_B_STAGE);
          if constexpr (MN) {
#pragma unroll
            for (int c = 0; c < GEMM_BM / 64; ++c)
              tma_load_2d(smem_u32(sA + stage * GEMM_A_STAGE + c * GEMM_MN_CHUNK), &tmA, full_bar(stage),
                          mb * GEMM_BM + c * 64, kb * GEMM_BK);
#pragma unroll
            for (int c = 0; c < GEMM_BN / 64; ++c)
              tma_load_2d(smem_u32(sB + stage * GEMM_B_STAGE + c * GEMM_MN_CHUNK), &tmB, full_bar(stage),
                          nb * GEMM_BN + c * 64, kb * GEMM_BK);
          } else {
            const int ka = (args.tri == TRI_DIAG ? nb * GEMM_BN : 0) + kb * GEMM_BK;  // TRI_DIAG: B is compact
            tma_load_2d(smem_u32(sA + stage * GEMM_A_STAGE), &tmA, full_bar(stage), ka, mb * GEMM_BM);
            tma_load_2d(smem_u32(sB + stage * GEMM_B_STAGE), &tmB, full_bar(stage), kb * GEMM_BK, nb * GEMM_BN);
          }
          issued |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == GEMM_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every issued load must have landed before the CTA may exit
      for (int s = 0; s < GEMM_STAGES; ++s)
        if (issued & (1u << s)) mbar_wait_drain(full_bar(s), (last_parity >> s) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t IDESC = idesc_bf16_f32(GEMM_BM, GEMM_BN, MN);
      int stage = 0;
      uint32_t phase = 0;
      int slot = 0;
      uint32_t sphase = 0;
      bool ok = true;
      for (int local = 0; ok; ++local) {
        if (!mbar_wait(sfull_bar(slot), sphase, abort_flag, args.err, ERR_WAIT_SCHED)) break;
        const int t = tile_ring[slot];
        mbar_arrive(sempty_bar(slot));
        if (++slot == GEMM_SCHED_SLOTS) {
          slot = 0;
          sphase ^= 1u;
        }
        if (t < 0) break;
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, args.err, ERR_WAIT_TEMPTY)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * GEMM_BN;
        int mb, nb;
        gemm_tile_coords(t, args, mb, nb);
        const int num_kb = gemm_num_kb(args, nb);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, args.err, ERR_WAIT_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * GEMM_A_STAGE);
          const uint32_t b_base = smem_u32(sB + stage * GEMM_B_STAGE);
#pragma unroll
          for (int k = 0; k < GEMM_BK / 16; ++k) {
            // K-major: 16 elements = 32 B along the swizzled row; MN-major: 16 rows of 128 B
            const uint64_t ad = MN ? desc_mnmajor_sw128(a_base + k * 2048, GEMM_MN_CHUNK)
                                   : desc_kmajor_sw128(a_base + k * 32);
            const uint64_t bd = MN ? desc_mnmajor_sw128(b_base + k * 2048, GEMM_MN_CHUNK)
                                   : desc_kmajor_sw128(b_base + k * 32);
            mma_bf16(d_tmem, ad, bd, IDESC, (kb | k) != 0);
          }
          mma_commit(empty_bar(stage));
          if (++stage == GEMM_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) mma_commit(tfull_bar(acc));
      }
      // all MMAs of this thread must complete before TMEM is freed
      mma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else {
    // ---------------- epilogue (warps 2..5)
    const int quad = warp & 3;
    const int row_in_tile = quad * 32 + lane;
    int slot = 0;
    uint32_t sphase = 0;
    for (int local = 0;; ++local) {
      // warp-uniform decisions: the tcgen05.ld below is .sync.aligned
      const bool have = mbar_wait(sfull_bar(slot), sphase, abort_flag, args.err, ERR_WAIT_SCHED);
      if (!__all_sync(0xffffffffu, have)) break;
      const int t = tile_ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(sempty_bar(slot));
      if (++slot == GEMM_SCHED_SLOTS) {
        slot = 0;
        sphase ^= 1u;
      }
      if (t < 0) break;
      int mb, nb;
      gemm_tile_coords(t, args, mb, nb);
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const bool ready = mbar_wait(tfull_bar(acc), acc_phase, abort_flag, args.err, ERR_WAIT_TFULL);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * GEMM_BN;
      const int m = mb * GEMM_BM + row_in_tile;
      const int n0 = nb * GEMM_BN;
      float sum = 0.f;
#pragma unroll 1
      for (int c = 0; c < GEMM_BN / 32; ++c) {
        uint4 e[4];  // EPI_DOT(32): the 32 elements of E this chunk multiplies, fetched before the TMEM load
        if constexpr (MODE == EPI_DOT || MODE == EPI_DOT32) {
          const int col = n0 + c * 32;
          const __nv_bfloat16* erow = args.E + (long long)m * args.ldE + col;
#pragma unroll
          for (int v = 0; v < 4; ++v)
            e[v] = (m < args.M && col + v * 8 < args.N) ? __ldg(reinterpret_cast<const uint4*>(erow + v * 8))
                                                         : make_uint4(0, 0, 0, 0);
        }
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + c * 32, r);
        tmem_ld_wait();
        if constexpr (MODE == EPI_SUMSQ) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float d = __uint_as_float(r[j]);
            sum = fmaf(d, d, sum);
          }
        } else if constexpr (MODE == EPI_DOT || MODE == EPI_DOT32) {
          // columns past N hold D = 0 (zero-filled B rows) and e = 0
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint32_t ew[4] = {e[v].x, e[v].y, e[v].z, e[v].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              sum = fmaf(__uint_as_float(r[v * 8 + 2 * h]), bf16lo(ew[h]), sum);
              sum = fmaf(__uint_as_float(r[v * 8 + 2 * h + 1]), bf16hi(ew[h]), sum);
            }
          }
          if constexpr (MODE == EPI_DOT32) {  // one partial per 32-column chunk
            if (m < args.M) args.part[(long long)(nb * (GEMM_BN / 32) + c) * args.part_ld + m] = sum;
            sum = 0.f;
          }
        } else {
          const int col = n0 + c * 32;
          const bool diag = args.tri == TRI_DIAG_STORE;
          const float scale = (args.tri == TRI_LOWER_STORE && nb < (mb >> 1)) ? 2.0f : 1.0f;
          if (m < args.M) {
            __nv_bfloat16* crow = args.C + (long long)m * args.ldC + (diag ? col - n0 : col);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              if (col + v * 8 < args.N) {
                // TRI_DIAG_STORE keeps only entries of the row's own quantisation group
                const float keep = (!diag || (m / args.group) == ((col + v * 8) / args.group)) ? scale : 0.0f;
                uint32_t w[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                  __nv_bfloat162 p = __floats2bfloat162_rn(keep * __uint_as_float(r[v * 8 + 2 * h]),
                                                           keep * __uint_as_float(r[v * 8 + 2 * h + 1]));
                  w[h] = *reinterpret_cast<uint32_t*>(&p);
                }
                *reinterpret_cast<uint4*>(crow + v * 8) = make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      if constexpr (MODE == EPI_SUMSQ || MODE == EPI_DOT) {
        if (m < args.M) args.part[(long long)nb * args.part_ld + m] = sum;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, GEMM_TMEM_COLS);
  }
}

}  // namespace awq
