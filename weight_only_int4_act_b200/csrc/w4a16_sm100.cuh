// W4A16 product on sm_100a: Y[t, o] = sum_i X'[t, i] W_hat[o, i], where
// W_hat[o, i] = (code - z) * Delta is dequantised from the packed format
// (8 codes per uint32 word, lowest channel in the lowest nibble; fp16 step
// and zero point per (row, group)) inside the kernel, and X' is the bf16
// activation that already carries S^-1 (folded into its producer).
//
// Pages: "AWQ量化技术解析：激活感知的权重量化革命" (kwkr.cn) §1.2 (weights
// dequantised on the fly as W_int4 x scale_fp16) and §4.2 (dequantisation
// fused with the GEMM in one kernel, scales kept in shared memory);
// "大模型的开发应用（十八）：大模型量化：GPTQ与AWQ" (ewbang.com) AWQ 二.3 (INT4
// storage, dequantised for the product); "AWQ" (scholia-log) §2.1 and §4.3
// (W X = (W S)(S^-1 X), S^-1 folded into the adjacent operation).
//
// Tiles are 128 output channels x BN tokens (BN = 16 .. 256): the weights are
// the M = 128 operand of tcgen05.mma.cta_group::1.kind::f16 and the tokens
// the N operand, so a decode batch of a few tokens still fills a tile. One
// K step is 64 channels. Three shared-memory rings, each with its own
// full/empty mbarriers, so that each stream runs ahead as far as its ring
// allows: packed codes (4 KB a step, up to 24 steps deep: the weight bytes in
// flight that hide HBM latency), activations (BN x 64 bf16, 128-byte swizzle)
// and dequantised weights (128 x 64 bf16, 128-byte swizzle). Depths depend on
// BN (host plan). Warp roles (480 threads, one CTA per SM):
//   warp 0       TMA of the packed codes (128 rows x 8 words, no swizzle);
//   warp 1       allocates 512 TMEM columns (two accumulators at columns 0
//                and 256) and one thread issues the MMAs;
//   warp 2       TMA of the activation tiles;
//   warps 3..10  dequantise: thread (h, r) expands words 4h..4h+3 of row r
//                ((code - z) * Delta in fp32, exact, then one rounding to
//                bf16) into the K-major swizzled layout the MMA descriptor
//                reads; a proxy fence and one arrive per warp publish it;
//   warps 11..14 epilogue: tcgen05.ld of the accumulator (TMEM lane = output
//                channel, column = token), bf16 stores of Y (or fp32 split-K
//                partials), then release of the accumulator.
// K may be split across CTAs when there are fewer tiles than SMs; the
// partials are then summed in split order by a second kernel.
// Every wait is bounded; on a timeout the CTA records an error in *err,
// drains its in-flight copies and MMAs, frees TMEM and returns.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace awq {

constexpr int W4_BM = 128;
constexpr int W4_BK = 64;
constexpr int W4_MAX_BN = 256;
constexpr int W4_THREADS = 480;
constexpr int W4_A_STAGE = W4_BM * W4_BK * 2;  // dequantised weights, 16 KB
constexpr int W4_R_STAGE = W4_BM * W4_BK / 2;  // packed codes, 4 KB
constexpr int W4_MAX_RS = 32, W4_MAX_XS = 8, W4_MAX_AS = 4;
constexpr int W4_NBARS = 2 * (W4_MAX_RS + W4_MAX_XS + W4_MAX_AS) + 5;
constexpr int W4_TMEM_COLS = 512;
constexpr int W4_SMEM_LIMIT = 232448;

// Shared-memory bytes for ring depths (as, xs, rs) at BN tokens.
__host__ __device__ constexpr int w4_smem_bytes(int as, int xs, int rs, int bn) {
  return 1024 + as * W4_A_STAGE + xs * bn * W4_BK * 2 + rs * W4_R_STAGE + W4_NBARS * 8 + 64;
}

constexpr int ERR_W4_RFULL = 0x301, ERR_W4_REMPTY = 0x302, ERR_W4_XFULL = 0x303, ERR_W4_XEMPTY = 0x304,
              ERR_W4_AFULL = 0x305, ERR_W4_AEMPTY = 0x306, ERR_W4_TFULL = 0x307, ERR_W4_TEMPTY = 0x308;

struct W4Args {
  int N, d_out, d_in;
  int bn;            // tokens per tile
  int n_mb, n_nb;    // ceil(d_out / 128), ceil(N / bn)
  int splits;        // K splits (1: no split)
  int kb_per_split;  // K steps per split
  int n_kb;          // ceil(d_in / 64)
  int num_tiles;     // n_mb * n_nb * splits
  int ng;            // groups per row (d_in / group)
  int group_shift;   // log2(group)
  int as, xs, rs;    // ring depths: dequantised weights, activations, packed codes
  const __half* scales;  // [d_out, ng]
  const __half* zeros;   // [d_out, ng]
  __nv_bfloat16* Y;      // [N, d_out] (splits == 1)
  float* P;              // [splits][p_stride] with [N, d_out] in each slab (splits > 1)
  long long p_stride;    // N * d_out rounded up to a multiple of 4
  int* err;
};

__device__ __forceinline__ void w4_tile_coords(int t, const W4Args& a, int& mb, int& nb, int& split) {
  mb = t % a.n_mb;
  const int rest = t / a.n_mb;
  nb = rest % a.n_nb;
  split = rest / a.n_nb;
}

__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// (code - z) * Delta for the 8 codes of one word, as 8 bf16 in a uint4.
// 2^23 + code is built by OR-ing the code into the mantissa of 2^23, so
// subtracting 2^23 + z leaves code - z exactly; the product with the fp16
// step is exact in fp32 (at most 4 + 11 significant bits) and is rounded
// once, to nearest even, to bf16.
__device__ __forceinline__ uint4 dequant_word(uint32_t w, float zoff, float delta) {
  float f[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) f[j] = (__uint_as_float(((w >> (4 * j)) & 0xFu) | 0x4B000000u) - zoff) * delta;
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

// A ring position: stage index and the parity of its current phase.
struct Ring {
  int stage = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next(int depth) {
    if (++stage == depth) {
      stage = 0;
      phase ^= 1u;
    }
  }
};

// GPH = quantisation groups per half K step of 32 channels (1 for g >= 32).
template <int GPH>
__global__ void __launch_bounds__(W4_THREADS, 1)
    w4a16_gemm_tcgen05(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                       const W4Args args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bn = args.bn;
  const int AS = args.as, XS = args.xs, RS = args.rs;
  const uint32_t x_stage = (uint32_t)bn * W4_BK * 2;  // a multiple of 1024 (bn >= 16 in steps of 16)
  uint8_t* sA = smem;                        // [AS][128 rows][128 B], swizzled
  uint8_t* sX = sA + AS * W4_A_STAGE;        // [XS][BN rows][128 B], swizzled
  uint8_t* sR = sX + XS * x_stage;           // [RS][128 rows][32 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sR + RS * W4_R_STAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + W4_NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // bars: rfull[32] rempty[32] xfull[8] xempty[8] afull[4] aempty[4] tfull[2] tempty[2] drain
  auto rfull = [&](int s) { return smem_u32(bars + s); };
  auto rempty = [&](int s) { return smem_u32(bars + W4_MAX_RS + s); };
  auto xfull = [&](int s) { return smem_u32(bars + 2 * W4_MAX_RS + s); };
  auto xempty = [&](int s) { return smem_u32(bars + 2 * W4_MAX_RS + W4_MAX_XS + s); };
  auto afull = [&](int s) { return smem_u32(bars + 2 * W4_MAX_RS + 2 * W4_MAX_XS + s); };
  auto aempty = [&](int s) { return smem_u32(bars + 2 * W4_MAX_RS + 2 * W4_MAX_XS + W4_MAX_AS + s); };
  constexpr int T0 = 2 * (W4_MAX_RS + W4_MAX_XS + W4_MAX_AS);
  auto tfull = [&](int a) { return smem_u32(bars + T0 + a); };
  auto tempty = [&](int a) { return smem_u32(bars + T0 + 2 + a); };
  const uint32_t drain_bar = smem_u32(bars + T0 + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < RS; ++s) {
      mbar_init(rfull(s), 1);
      mbar_init(rempty(s), 8);  // one arrive per dequantising warp
    }
    for (int s = 0; s < XS; ++s) {
      mbar_init(xfull(s), 1);
      mbar_init(xempty(s), 1);
    }
    for (int s = 0; s < AS; ++s) {
      mbar_init(afull(s), 8);
      mbar_init(aempty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), 4);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tmW);
  if (warp == 2 && lane == 0) prefetch_tmap(&tmX);
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), W4_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 || warp == 2) {
    if (lane == 0) {
      // ---------------- TMA producers: packed codes (warp 0) or activations (warp 2)
      const bool codes = warp == 0;
      const int depth = codes ? RS : XS;
      Ring ring;
      uint32_t issued = 0, last_parity = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < args.num_tiles; t += gridDim.x) {
        int mb, nb, split;
        w4_tile_coords(t, args, mb, nb, split);
        const int kb0 = split * args.kb_per_split;
        const int kb1 = min(args.n_kb, kb0 + args.kb_per_split);
        for (int kb = kb0; kb < kb1; ++kb) {
          const uint32_t full = codes ? rfull(ring.stage) : xfull(ring.stage);
          const uint32_t empty = codes ? rempty(ring.stage) : xempty(ring.stage);
          if (!mbar_wait(empty, ring.phase ^ 1u, abort_flag, args.err, codes ? ERR_W4_REMPTY : ERR_W4_XEMPTY)) {
            ok = false;
            break;
          }
          if (codes) {
            mbar_arrive_expect_tx(full, W4_R_STAGE);
            tma_load_2d(smem_u32(sR + ring.stage * W4_R_STAGE), &tmW, full, kb * (W4_BK / 8), mb * W4_BM);
          } else {
            mbar_arrive_expect_tx(full, x_stage);
            tma_load_2d(smem_u32(sX + ring.stage * x_stage), &tmX, full, kb * W4_BK, nb * bn);
          }
          issued |= 1u << ring.stage;
          last_parity = (last_parity & ~(1u << ring.stage)) | (ring.phase << ring.stage);
          ring.next(depth);
        }
      }
      for (int s = 0; s < depth; ++s)
        if (issued & (1u << s)) mbar_wait_drain(codes ? rfull(s) : xfull(s), (last_parity >> s) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t idesc = idesc_bf16_f32(W4_BM, bn);
      Ring xr, ar;
      bool ok = true;
      int local = 0;
      for (int t = blockIdx.x; ok && t < args.num_tiles; t += gridDim.x, ++local) {
        int mb, nb, split;
        w4_tile_coords(t, args, mb, nb, split);
        const int kb0 = split * args.kb_per_split;
        const int kb1 = min(args.n_kb, kb0 + args.kb_per_split);
        const int acc = local & 1;
        if (!mbar_wait(tempty(acc), ((local >> 1) & 1) ^ 1u, abort_flag, args.err, ERR_W4_TEMPTY)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(xfull(xr.stage), xr.phase, abort_flag, args.err, ERR_W4_XFULL) ||
              !mbar_wait(afull(ar.stage), ar.phase, abort_flag, args.err, ERR_W4_AFULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + ar.stage * W4_A_STAGE);
          const uint32_t x_base = smem_u32(sX + xr.stage * x_stage);
#pragma unroll
          for (int k = 0; k < W4_BK / 16; ++k)
            mma_bf16(d_tmem, desc_kmajor_sw128(a_base + k * 32), desc_kmajor_sw128(x_base + k * 32), idesc,
                     (kb != kb0) || (k != 0));
          mma_commit(xempty(xr.stage));
          mma_commit(aempty(ar.stage));
          xr.next(XS);
          ar.next(AS);
        }
        if (ok) mma_commit(tfull(acc));
      }
      mma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else if (warp < 11) {
    // ---------------- dequantisation: thread (h, r) takes words 4h..4h+3 of row r
    const int d = threadIdx.x - 3 * 32;
    const int r = d & (W4_BM - 1);
    const int h = d >> 7;
    const uint32_t a_row_off = (uint32_t)r * 128;
    const int sw = r & 7;
    Ring rr, ar;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < args.num_tiles; t += gridDim.x) {
      int mb, nb, split;
      w4_tile_coords(t, args, mb, nb, split);
      const int kb0 = split * args.kb_per_split;
      const int kb1 = min(args.n_kb, kb0 + args.kb_per_split);
      const int row = mb * W4_BM + r;
      const bool valid = row < args.d_out;
      const __half* srow = args.scales + (long long)(valid ? row : 0) * args.ng;
      const __half* zrow = args.zeros + (long long)(valid ? row : 0) * args.ng;
      // step and zero point of the GPH groups of this thread's 32 channels, loaded one step ahead
      auto load_params = [&](int kb, float (&dq)[GPH], float (&zq)[GPH]) {
#pragma unroll
        for (int q = 0; q < GPH; ++q) {
          const int ch = kb * W4_BK + h * 32 + q * (32 / GPH);
          const int gi = min(ch >> args.group_shift, args.ng - 1);
          dq[q] = valid ? __half2float(srow[gi]) : 0.0f;
          zq[q] = 8388608.0f + (valid ? __half2float(zrow[gi]) : 0.0f);
        }
      };
      float dn[GPH], zn[GPH];
      load_params(kb0, dn, zn);
      for (int kb = kb0; kb < kb1; ++kb) {
        float dc[GPH], zc[GPH];
#pragma unroll
        for (int q = 0; q < GPH; ++q) {
          dc[q] = dn[q];
          zc[q] = zn[q];
        }
        if (kb + 1 < kb1) load_params(kb + 1, dn, zn);
        bool have = mbar_wait(rfull(rr.stage), rr.phase, abort_flag, args.err, ERR_W4_RFULL);
        if (!__all_sync(0xffffffffu, have)) {
          ok = false;
          break;
        }
        const uint4 w = *reinterpret_cast<const uint4*>(sR + rr.stage * W4_R_STAGE + r * 32 + h * 16);
        __syncwarp();
        if (lane == 0) mbar_arrive(rempty(rr.stage));
        rr.next(RS);
        have = mbar_wait(aempty(ar.stage), ar.phase ^ 1u, abort_flag, args.err, ERR_W4_AEMPTY);
        if (!__all_sync(0xffffffffu, have)) {
          ok = false;
          break;
        }
        const uint32_t words[4] = {w.x, w.y, w.z, w.w};
        uint8_t* arow = sA + ar.stage * W4_A_STAGE + a_row_off;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          constexpr int WPG = 4 / GPH;  // words per group inside the half step
          const uint4 v = dequant_word(words[c], zc[c / WPG], dc[c / WPG]);
          *reinterpret_cast<uint4*>(arow + (((4 * h + c) ^ sw) << 4)) = v;
        }
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) mbar_arrive(afull(ar.stage));
        ar.next(AS);
      }
    }
  } else {
    // ---------------- epilogue (warps 11..14; warp w reads TMEM lanes 32 (w % 4) ..)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    int local = 0;
    for (int t = blockIdx.x; t < args.num_tiles; t += gridDim.x, ++local) {
      int mb, nb, split;
      w4_tile_coords(t, args, mb, nb, split);
      const int acc = local & 1;
      const bool ready = mbar_wait(tfull(acc), (local >> 1) & 1, abort_flag, args.err, ERR_W4_TFULL);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const int o = mb * W4_BM + r;
      const int t0 = nb * bn;
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * 256;
      for (int c = 0; c * 32 < bn; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + c * 32, v);
        tmem_ld_wait();
        // tokens t0 + 32c + j for j < jn are inside both the tile and N
        const int jn = min(32, min(bn - c * 32, args.N - (t0 + c * 32)));
        if (o < args.d_out) {
          const long long e0 = (long long)(t0 + c * 32) * args.d_out + o;
          if (args.splits == 1) {
            __nv_bfloat16* y = args.Y + e0;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < jn) y[(long long)j * args.d_out] = __float2bfloat16_rn(__uint_as_float(v[j]));
          } else {
            float* P = args.P + (long long)split * args.p_stride + e0;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < jn) P[(long long)j * args.d_out] = __uint_as_float(v[j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty(acc));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, W4_TMEM_COLS);
  }
}

// Y = bf16(sum over splits of P[split]) in split order; 4 outputs per thread.
// Slabs are `stride` floats apart (a multiple of 4, so every float4 is aligned).
__global__ void w4a16_split_reduce(const float* __restrict__ P, int splits, long long n, long long stride,
                                   __nv_bfloat16* __restrict__ Y) {
  const long long n4 = n >> 2;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    float4 acc = reinterpret_cast<const float4*>(P)[i];
    for (int s = 1; s < splits; ++s) {
      const float4 p = reinterpret_cast<const float4*>(P + (long long)s * stride)[i];
      acc.x += p.x;
      acc.y += p.y;
      acc.z += p.z;
      acc.w += p.w;
    }
    uint2 out = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    reinterpret_cast<uint2*>(Y)[i] = out;
  }
  // tail (n not a multiple of 4)
  const long long tail0 = n4 << 2;
  const long long i = tail0 + (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (blockIdx.x == 0 && i < n) {
    float acc = P[i];
    for (int s = 1; s < splits; ++s) acc += P[(long long)s * stride + i];
    Y[i] = __float2bfloat16_rn(acc);
  }
}

// Fold S^-1 into the producer of X: row i of p [d_in, inner] (bf16) becomes
// p / s_i, the quotient in fp32 (correctly rounded division) rounded to
// nearest even bf16. VEC = 8: eight elements of one row per thread (inner a
// multiple of 8, p 16-byte aligned); VEC = 1: one element per thread.
template <int VEC>
__global__ void fold_inv_scales_kernel(const float* __restrict__ s, long long d_in, long long inner,
                                       __nv_bfloat16* __restrict__ p) {
  const long long units = d_in * inner / VEC;
  for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < units;
       u += (long long)gridDim.x * blockDim.x) {
    const long long e = u * VEC;
    const float si = s[e / inner];
    if constexpr (VEC == 8) {
      uint4 w = reinterpret_cast<const uint4*>(p)[u];
      uint32_t* h = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        h[q] = pack_bf16x2(__uint_as_float(h[q] << 16) / si, __uint_as_float(h[q] & 0xFFFF0000u) / si);
      reinterpret_cast<uint4*>(p)[u] = w;
    } else {
      p[e] = __float2bfloat16_rn(__bfloat162float(p[e]) / si);
    }
  }
}

}  // namespace awq
