// The loss contraction and the Gram product on CTA pairs (tcgen05
// cta_group::2) for sm_100a.
//
// Same products and epilogues as gemm_sm100.cuh (EPI_SUMSQ, EPI_DOT with
// TRI_NONE or TRI_K; EPI_STORE with TRI_LOWER_STORE and MN-major operands for
// G' = the lower block triangle of X^T X), but each 256 x 256 tile is computed
// by a cluster of two CTAs on
// two SMs: CTA r of the pair loads rows [128 r, 128 r + 128) of the tile's A
// panel and of its B panel (64-wide K stages, TMA, no multicast), and one
// thread of the even CTA issues M=256 N=256 K=16 MMAs that read both CTAs'
// shared memory and accumulate 128 rows x 256 columns in each CTA's TMEM.
// Per SM and K step that is 32 KB of operand traffic instead of 48 KB for
// the same MMA work.
//
// Coordination inside the pair:
//   full[s]    even CTA only: armed by the even producer with both CTAs'
//              bytes; both CTAs' TMA loads complete on it (cta_group::2 form);
//   empty[s]   in each CTA, released by the MMA commit multicast to both;
//   tfull[a]   in each CTA, MMA commit multicast to both;
//   tempty[a]  even CTA only, 8 arrivals (the epilogue warps of both CTAs);
//   tile ring  the even producer takes tile indices from the global counter,
//              writes them into both CTAs' rings and arrives on both sfull;
//              sempty (even CTA) counts 10 readers (even MMA + 4 even
//              epilogue warps + odd producer + 4 odd epilogue warps).
// Last wave of the G' product: when the tiles leave a last wave of at most
// half the pairs, those R tiles are handed out as R x S pieces of K/S steps
// each (S = pairs / R), piece-major so that the pieces in flight together
// cover the same K range of every split tile (the pairs keep sweeping X in
// step, and each slice of X is still fetched once); each piece is written as
// fp32 partials and gram_tail_fixup adds the S pieces of a tile in K order.
// All waits are bounded (ptx.cuh); the CTAs meet at a cluster barrier before
// freeing TMEM (both CTAs, cta_group::2) and exiting.
#pragma once
#include "gemm_sm100.cuh"

namespace awq {

constexpr int PAIR_BM = 256;  // tile rows (128 per CTA)
constexpr int PAIR_BN = 256;  // tile columns (B rows, 128 per CTA)
constexpr int PAIR_BK = 64;
#ifndef AWQ_PAIR_STAGES
#define AWQ_PAIR_STAGES 6
#endif
constexpr int PAIR_STAGES = AWQ_PAIR_STAGES;
constexpr int PAIR_A_STAGE = 128 * PAIR_BK * 2;  // 16 KB per CTA
constexpr int PAIR_B_STAGE = 128 * PAIR_BK * 2;  // 16 KB per CTA
constexpr int PAIR_SLOTS = 4;
constexpr int PAIR_SMEM_BYTES = 1024 + PAIR_STAGES * (PAIR_A_STAGE + PAIR_B_STAGE) + 512;
static_assert(PAIR_SMEM_BYTES <= 232448, "shared memory per CTA");

// Tile t of the lower block triangle of 256 x 256 tiles: row block mb holds
// column blocks 0 .. mb (t = mb (mb + 1) / 2 + nb).
__device__ __forceinline__ void pair_tri_coords(int t, int& mb, int& nb) {
  int q = (int)((sqrtf(8.0f * (float)t + 1.0f) - 1.0f) * 0.5f);
  while ((long long)(q + 1) * (q + 2) / 2 <= t) ++q;
  while ((long long)q * (q + 1) / 2 > t) --q;
  mb = q;
  nb = t - q * (q + 1) / 2;
}

// Work item i of the counter: a whole tile, or piece (part q of split tile
// tail_first + r) when i >= tail_first, with its K steps [k0, k1) and slab.
struct PairWork {
  int t, k0, k1, slab;  // slab < 0: a whole tile
};
__device__ __forceinline__ PairWork pair_work(const GemmArgs& a, int i, int num_kb_tile) {
  PairWork w;
  if (i < a.tail_first) {
    w.t = i;
    w.k0 = 0;
    w.k1 = num_kb_tile;
    w.slab = -1;
    return w;
  }
  const int R = a.num_tiles - a.tail_first, j = i - a.tail_first;
  const int q = j / R, r = j - q * R;
  w.t = a.tail_first + r;
  w.k0 = q * num_kb_tile / a.tail_split;
  w.k1 = (q + 1) * num_kb_tile / a.tail_split;
  w.slab = j;  // = q R + r
  return w;
}

__device__ __forceinline__ void pair_tile_coords(int t, const GemmArgs& a, int& mb, int& nb) {
  if (a.tri == TRI_LOWER_STORE)
    pair_tri_coords(t, mb, nb);
  else
    gemm_tile_coords(t, a, mb, nb);
}

// MN = false: A [M, K] and B [N, K] row-major (K-major operands); each CTA loads
// one box of 64 (K) x 128 rows of each per stage.
// MN = true: A and B are the same row-major [K, M] matrix read transposed
// (G = X^T X straight from X): each CTA loads two boxes of 64 (M or N) x 64
// (K) per operand and stage, at 64-column offsets.
template <int MODE, bool MN = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GEMM_THREADS, 1)
    gemm_pair_bf16_tcgen05(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + PAIR_STAGES * PAIR_A_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + PAIR_STAGES * PAIR_B_STAGE);
  // full[S], empty[S], tfull[2], tempty[2], drain, sfull[R], sempty[R]
  constexpr int NB = 2 * PAIR_STAGES + 5 + 2 * PAIR_SLOTS;
  volatile int* tile_ring = reinterpret_cast<volatile int*>(bars + NB);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NB) + PAIR_SLOTS;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank() & 1u;
  const bool even = rank == 0;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + PAIR_STAGES + s); };
  auto tfull_bar = [&](int a) { return smem_u32(bars + 2 * PAIR_STAGES + a); };
  auto tempty_bar = [&](int a) { return smem_u32(bars + 2 * PAIR_STAGES + 2 + a); };
  const uint32_t drain_bar = smem_u32(bars + 2 * PAIR_STAGES + 4);
  auto sfull_bar = [&](int r) { return smem_u32(bars + 2 * PAIR_STAGES + 5 + r); };
  auto sempty_bar = [&](int r) { return smem_u32(bars + 2 * PAIR_STAGES + 5 + PAIR_SLOTS + r); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < PAIR_STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 8);
    }
    mbar_init(drain_bar, 1);
    for (int r = 0; r < PAIR_SLOTS; ++r) {
      mbar_init(sfull_bar(r), 1);
      mbar_init(sempty_bar(r), 10);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), GEMM_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // work items: whole tiles, then the pieces of the split last-wave tiles
  const int num_tiles = args.tail_first + (args.num_tiles - args.tail_first) * args.tail_split;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- tile scheduler (even CTA) + TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_parity = 0;
      int slot = 0;
      uint32_t sphase = 0;
      bool ok = true;
      while (ok) {
        int t;
        if (even) {
          if (!mbar_wait(sempty_bar(slot), sphase ^ 1u, abort_flag, args.err, ERR_WAIT_SCHED)) break;
          t = atomicAdd(args.tile_counter, 1);
          if (t >= num_tiles) t = -1;
          tile_ring[slot] = t;
          st_shared_remote(mapa_shared(smem_u32((const void*)(tile_ring + slot)), 1), t);
          mbar_arrive(sfull_bar(slot));
          mbar_arrive_remote(mapa_shared(sfull_bar(slot), 1));
        } else {
          if (!mbar_wait(sfull_bar(slot), sphase, abort_flag, args.err, ERR_WAIT_SCHED)) break;
          t = tile_ring[slot];
          mbar_arrive_remote(mapa_shared(sempty_bar(slot), 0));
        }
        if (++slot == PAIR_SLOTS) {
          slot = 0;
          sphase ^= 1u;
        }
        if (t < 0) break;
        int mb, nb;
        pair_tile_coords(t < args.tail_first ? t : args.tail_first + (t - args.tail_first) % max(1, args.num_tiles - args.tail_first),
                         args, mb, nb);
        const PairWork wk = pair_work(args, t, gemm_num_kb(args, nb));
        for (int kb = wk.k0; kb < wk.k1; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, args.err, ERR_WAIT_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t full_even = mapa_shared(full_bar(stage), 0);
          if (even) mbar_arrive_expect_tx(full_bar(stage), 2 * (PAIR_A_STAGE + PAIR_B_STAGE));
          if constexpr (MN) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              tma_load_2d_pair(smem_u32(sA + stage * PAIR_A_STAGE + c * GEMM_MN_CHUNK), &tmA, full_even,
                               mb * PAIR_BM + (int)rank * 128 + c * 64, kb * PAIR_BK);
              tma_load_2d_pair(smem_u32(sB + stage * PAIR_B_STAGE + c * GEMM_MN_CHUNK), &tmB, full_even,
                               nb * PAIR_BN + (int)rank * 128 + c * 64, kb * PAIR_BK);
            }
          } else {
            tma_load_2d_pair(smem_u32(sA + stage * PAIR_A_STAGE), &tmA, full_even, kb * PAIR_BK,
                             mb * PAIR_BM + (int)rank * 128);
            tma_load_2d_pair(smem_u32(sB + stage * PAIR_B_STAGE), &tmB, full_even, kb * PAIR_BK,
                             nb * PAIR_BN + (int)rank * 128);
          }
          issued |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == PAIR_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (even) {
        // loads land on the even CTA's full barriers: wait for every armed one
        for (int s = 0; s < PAIR_STAGES; ++s)
          if (issued & (1u << s)) mbar_wait_drain(full_bar(s), (last_parity >> s) & 1u);
      } else if (*abort_flag) {
        // on an aborted run, give this CTA's unconsumed loads time to land
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && even) {
      // ---------------- MMA issuer (even CTA)
      constexpr uint32_t IDESC = idesc_bf16_f32(PAIR_BM, PAIR_BN, MN);
      int stage = 0;
      uint32_t phase = 0;
      int slot = 0;
      uint32_t sphase = 0;
      bool ok = true;
      for (int local = 0; ok; ++local) {
        if (!mbar_wait(sfull_bar(slot), sphase, abort_flag, args.err, ERR_WAIT_SCHED)) break;
        const int t = tile_ring[slot];
        mbar_arrive(sempty_bar(slot));
        if (++slot == PAIR_SLOTS) {
          slot = 0;
          sphase ^= 1u;
        }
        if (t < 0) break;
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, args.err, ERR_WAIT_TEMPTY)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * PAIR_BN;
        int mb, nb;
        pair_tile_coords(t < args.tail_first ? t : args.tail_first + (t - args.tail_first) % max(1, args.num_tiles - args.tail_first),
                         args, mb, nb);
        const PairWork wk = pair_work(args, t, gemm_num_kb(args, nb));
        for (int kb = wk.k0; kb < wk.k1; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, args.err, ERR_WAIT_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * PAIR_A_STAGE);
          const uint32_t b_base = smem_u32(sB + stage * PAIR_B_STAGE);
#pragma unroll
          for (int k = 0; k < PAIR_BK / 16; ++k) {
            // K-major: 16 elements = 32 B along the swizzled row; MN-major: 16 rows of 128 B
            const uint64_t ad = MN ? desc_mnmajor_sw128(a_base + k * 2048, GEMM_MN_CHUNK)
                                   : desc_kmajor_sw128(a_base + k * 32);
            const uint64_t bd = MN ? desc_mnmajor_sw128(b_base + k * 2048, GEMM_MN_CHUNK)
                                   : desc_kmajor_sw128(b_base + k * 32);
            mma_bf16_pair(d_tmem, ad, bd, IDESC, (kb != wk.k0) || (k != 0));
          }
          mma_commit_pair(empty_bar(stage), 0x3);
          if (++stage == PAIR_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) mma_commit_pair(tfull_bar(acc), 0x3);
      }
      mma_commit_pair(drain_bar, 0x1);
      mbar_wait_drain(drain_bar, 0);
    }
  } else {
    // ---------------- epilogue (warps 2..5 of both CTAs)
    const int quad = warp & 3;
    const int row_in_tile = quad * 32 + lane;
    int slot = 0;
    uint32_t sphase = 0;
    for (int local = 0;; ++local) {
      const bool have = mbar_wait(sfull_bar(slot), sphase, abort_flag, args.err, ERR_WAIT_SCHED);
      if (!__all_sync(0xffffffffu, have)) break;
      const int t = tile_ring[slot];
      __syncwarp();
      if (lane == 0) {
        if (even)
          mbar_arrive(sempty_bar(slot));
        else
          mbar_arrive_remote(mapa_shared(sempty_bar(slot), 0));
      }
      if (++slot == PAIR_SLOTS) {
        slot = 0;
        sphase ^= 1u;
      }
      if (t < 0) break;
      int mb, nb;
      pair_tile_coords(t < args.tail_first ? t : args.tail_first + (t - args.tail_first) % max(1, args.num_tiles - args.tail_first),
                       args, mb, nb);
      const int slab = t < args.tail_first ? -1 : t - args.tail_first;
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const bool ready = mbar_wait(tfull_bar(acc), acc_phase, abort_flag, args.err, ERR_WAIT_TFULL);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * PAIR_BN;
      const int m = mb * PAIR_BM + (int)rank * 128 + row_in_tile;
      const int n0 = nb * PAIR_BN;
      float sum = 0.f;
#pragma unroll 1
      for (int c = 0; c < PAIR_BN / 32; ++c) {
        uint4 e[4];
        if constexpr (MODE == EPI_DOT) {
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
        } else if constexpr (MODE == EPI_STORE) {
          // G' = 2 G on strictly lower blocks, G on diagonal blocks (TRI_LOWER_STORE)
          const int col = n0 + c * 32;
          const float scale = nb < mb ? 2.0f : 1.0f;
          if (slab >= 0) {
            // a K piece of a split tile: fp32 partial, row 128 rank + row_in_tile of its slab
            float4* prow = reinterpret_cast<float4*>(
                args.tail_part + ((long long)slab * PAIR_BM + (int)rank * 128 + row_in_tile) * PAIR_BN + c * 32);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              prow[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                    __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
          } else if (m < args.M) {
            __nv_bfloat16* crow = args.C + (long long)m * args.ldC + col;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              if (col + v * 8 < args.N) {
                uint32_t w[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                  __nv_bfloat162 p = __floats2bfloat162_rn(scale * __uint_as_float(r[v * 8 + 2 * h]),
                                                           scale * __uint_as_float(r[v * 8 + 2 * h + 1]));
                  w[h] = *reinterpret_cast<uint32_t*>(&p);
                }
                *reinterpret_cast<uint4*>(crow + v * 8) = make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        } else {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint32_t ew[4] = {e[v].x, e[v].y, e[v].z, e[v].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              sum = fmaf(__uint_as_float(r[v * 8 + 2 * h]), bf16lo(ew[h]), sum);
              sum = fmaf(__uint_as_float(r[v * 8 + 2 * h + 1]), bf16hi(ew[h]), sum);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (even)
          mbar_arrive(tempty_bar(acc));
        else
          mbar_arrive_remote(mapa_shared(tempty_bar(acc), 0));
      }
      if constexpr (MODE != EPI_STORE) {
        if (m < args.M) args.part[(long long)nb * args.part_ld + m] = sum;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // all MMAs drained, all TMEM reads and remote arrivals done in both CTAs
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, GEMM_TMEM_COLS);
  }
}

// Block (r, y) finishes 1024 elements (4 per thread, 256 apart: coalesced)
// of split tile tail_first + r: its tail_split K pieces added in K order,
// times 2 off the diagonal blocks, rounded to bf16 into C.
__global__ void __launch_bounds__(256) gram_tail_fixup(const GemmArgs a) {
  const int R = a.num_tiles - a.tail_first, r = blockIdx.x;
  if (r >= R) return;
  int mb, nb;
  pair_tri_coords(a.tail_first + r, mb, nb);
  const float scale = nb < mb ? 2.0f : 1.0f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int e = blockIdx.y * 1024 + k * 256 + threadIdx.x;  // row-major in the 256 x 256 tile
    if (e >= PAIR_BM * PAIR_BN) continue;
    const int row = e / PAIR_BN, col = e - row * PAIR_BN;
    const long long m = (long long)mb * PAIR_BM + row, cn = (long long)nb * PAIR_BN + col;
    if (m >= a.M || cn >= a.N) continue;
    float acc = 0.0f;
    for (int q = 0; q < a.tail_split; ++q) {
      const long long i = ((long long)(q * R + r) * PAIR_BM + row) * PAIR_BN + col;
      if (AWQ_IDX_OK(i, (long long)R * a.tail_split * PAIR_BM * PAIR_BN, BS_GRAM_FIX)) acc += a.tail_part[i];
    }
    if (AWQ_IDX_OK(m * a.ldC + cn, (long long)a.M * a.ldC, BS_GRAM_FIX)) a.C[m * a.ldC + cn] = __float2bfloat16_rn(scale * acc);
  }
}

}  // namespace awq
