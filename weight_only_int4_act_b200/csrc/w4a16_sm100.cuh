// W4A16 product on sm_100a: Y[t, o] = sum_i X'[t, i] W_hat[o, i], where
// W_hat[o, i] = (code - z) * Delta is dequantised from the packed format
// (8 codes per uint32 word, lowest channel in the lowest nibble; fp16 step
// and zero point per (row, group)) inside the kernel, and X' is the fp16 or
// bf16 activation that already carries S^-1 (folded into its producer). The
// dequantised weight enters the tensor cores in the activation type: in fp16
// (code - z) * Delta is rounded once; in bf16 Delta is first rounded to bf16,
// then the product.
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
// the N operand, so a decode batch of a few tokens still fills a tile. One K
// step is 128 channels (8 MMAs of K = 16). The dequantised weights never touch
// shared memory: the dequantising warps write them into tensor memory with
// tcgen05.st and the MMAs read A from there (lane = output channel, 32-bit
// column = two consecutive channels), so shared memory carries only the
// packed codes and the activations. Rings, each with full/empty mbarriers:
// packed codes in shared memory (two steps per TMA box, 128 rows x 128 B with
// the 128-byte swizzle: narrow boxes of one step's 32 B per row moved only
// ~7 GB/s per SM), activations in shared memory (BN x 128 as two 128-byte-
// swizzled 64-wide boxes), and dequantised weights in tensor memory (64
// columns a step, behind one or two accumulators). Depths depend on BN (host
// plan). Warp roles (480 threads, one CTA per SM):
//   warp 0       TMA of the packed codes;
//   warp 1       allocates the 512 TMEM columns and one thread issues the MMAs;
//   warp 2       TMA of the activation tiles;
//   warps 3..10  dequantise: warp w, lane l takes output channel
//                32 (w % 4) + l (its TMEM lane) and the half h = (w - 3) / 4 of
//                each step's channels, two codes per packed subtract and
//                multiply (dequant_word), 32 columns per tcgen05.st;
//   warps 11..14 epilogue: tcgen05.ld of the accumulator (TMEM lane = output
//                channel, column = token), stores of Y (or the fp32
//                partials), then release of the accumulator.
// The MMA issuer is the critical path: every other role waits with a short
// sleep between polls, so that waiting warps leave the issue slots of their
// scheduler (which the issuer shares with two dequantising warps) free.
// Work split: with many tiles, CTA c takes whole tiles c, c + G, ... (G
// CTAs). With few (decode widths, where 224 tiles on 148 SMs would leave a
// tail of half the CTAs idle), a static "stream-K" split: the (tile, K step)
// units, tile-major, are cut into G contiguous ranges of equal length and
// CTA c takes range c, cut at tile boundaries into segments. A tile that two
// or more CTAs touch is written by each as fp32 partials, CTA c into slab
// (c - first CTA of the tile), and w4a16_streamk_reduce adds the slabs in
// slab order. The split depends only on the shapes, so the result is
// deterministic. (Finishing a tile inside the kernel, by whichever CTA takes
// the last ticket of an atomic counter, measured slower: the fix-up lands on
// the critical path of the last CTAs.)
// Every wait is bounded; on a timeout the CTA records an error in *err,
// drains its in-flight copies and MMAs, frees TMEM and returns.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "check.cuh"
#include "ptx.cuh"

namespace awq {

// mbar_wait for long waits: sleeps `ns` between polls so that a waiting warp
// leaves the issue slots to the warps that do the work.
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* err,
                                                int code, uint32_t ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(ns);
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > AWQ_WAIT_LIMIT_NS) {
        *abort_flag = 1;
        if (err) atomicCAS(err, 0, code);
        return false;
      }
    }
  }
}

// Each thread of the warp writes 32 consecutive 32-bit columns of its TMEM lane.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16 (A in tensor memory: lane =
// row of A, 32-bit column = two consecutive K elements).
__device__ __forceinline__ void mma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

constexpr int W4_BM = 128;
constexpr int W4_SUB = 64;                      // channels per 128-byte-swizzled activation box
constexpr int W4_MAX_BN = 256;
constexpr int W4_THREADS = 480;
constexpr int W4_R_STAGE = W4_BM * 128;         // packed codes: one TMA box of 128 rows x 128 B (256 channels)

// A K step of BK channels (128 or 256): NSUB activation boxes, A_COLS TMEM
// columns of dequantised weights, RK steps per code box; a dequantising
// thread takes BK / 2 channels (CHUNKS 16-byte chunks of codes).
template <int BK>
struct W4Step {
  static constexpr int NSUB = BK / W4_SUB;
  static constexpr int A_COLS = BK / 2;
  static constexpr int RK = 256 / BK;
  static constexpr int CHUNKS = BK / 64;
};
constexpr int W4_MAX_RS = 32, W4_MAX_XS = 8, W4_MAX_AS = 8;
constexpr int W4_NBARS = 2 * (W4_MAX_RS + W4_MAX_XS + W4_MAX_AS) + 5;
constexpr int W4_TMEM_COLS = 512;
constexpr int W4_SMEM_LIMIT = 232448;

// Shared-memory bytes for ring depths (as, xs, rs) at BN tokens.
__host__ __device__ constexpr int w4_smem_bytes(int xs, int rs, int bn, int bk) {
  return 1024 + xs * bn * bk * 2 + rs * W4_R_STAGE + W4_NBARS * 8 + 64;
}
// TMEM columns: NACC accumulators of acc_stride columns, then the A ring.
__host__ __device__ constexpr int w4_nacc(int bn) { return bn == 256 ? 1 : 2; }
__host__ __device__ constexpr int w4_acc_stride(int bn) { return bn < 32 ? 32 : bn; }
__host__ __device__ constexpr int w4_max_as(int bn, int bk) {
  return (W4_TMEM_COLS - w4_nacc(bn) * w4_acc_stride(bn)) / (bk / 2);
}

constexpr int ERR_W4_RFULL = 0x301, ERR_W4_REMPTY = 0x302, ERR_W4_XFULL = 0x303, ERR_W4_XEMPTY = 0x304,
              ERR_W4_AFULL = 0x305, ERR_W4_AEMPTY = 0x306, ERR_W4_TFULL = 0x307, ERR_W4_TEMPTY = 0x308;

struct W4Args {
  int N, d_out, d_in;
  int bn;            // tokens per tile
  int n_mb, n_nb;    // ceil(d_out / 128), ceil(N / bn)
  int sk;            // 1: stream-K ranges of units, 0: whole tiles
  int n_kb;          // K steps per tile, ceil(d_in / BK)
  int num_tiles;     // n_mb * n_nb
  long long units;   // num_tiles * n_kb (stream-K)
  int ng;            // groups per row (d_in / group)
  int group_shift;   // log2(group)
  int as, xs, rs;    // ring depths: dequantised weights, activations, packed codes
  const __half* scales;  // [d_out, ng]
  const __half* zeros;   // [d_out, ng]
  void* Y;               // [N, d_out] in the activation type
  float* P;              // [slots][p_stride]: [N, d_out] fp32 partials in each slab (stream-K)
  long long p_stride;    // N * d_out rounded up to a multiple of 4
  int* err;
};

// First unit of stream-K range c of G over U units, and the range that holds unit u.
__host__ __device__ inline long long w4_sk_begin(long long c, long long G, long long U) { return c * U / G; }
__host__ __device__ inline long long w4_sk_cta(long long u, long long G, long long U) { return ((u + 1) * G - 1) / U; }

// One segment of a CTA's work: output tile (mb, nb), K steps [kb0, kb1);
// whole: no other CTA touches the tile (written to Y), else written to
// partial slab `slot`.
struct W4Seg {
  int mb, nb, kb0, kb1, slot, ns;  // ns: CTAs that touch the tile
  bool whole;
};

// The segments of this CTA, in order; every role walks the same sequence.
struct W4Sched {
  long long u, u1;
  __device__ explicit W4Sched(const W4Args& a) {
    if (a.sk) {
      u = w4_sk_begin(blockIdx.x, gridDim.x, a.units);
      u1 = w4_sk_begin(blockIdx.x + 1, gridDim.x, a.units);
    } else {
      u = blockIdx.x;
      u1 = a.num_tiles;
    }
  }
  __device__ bool next(const W4Args& a, W4Seg& g) {
    if (u >= u1) return false;
    long long tile;
    if (a.sk) {
      tile = u / a.n_kb;
      const long long t0 = tile * a.n_kb;
      g.kb0 = (int)(u - t0);
      g.kb1 = (int)min((long long)a.n_kb, (long long)g.kb0 + (u1 - u));
      const long long first = w4_sk_cta(t0, gridDim.x, a.units);
      g.ns = (int)(w4_sk_cta(t0 + a.n_kb - 1, gridDim.x, a.units) - first + 1);
      g.whole = g.ns == 1;
      g.slot = (int)(blockIdx.x - first);
      u += g.kb1 - g.kb0;
    } else {
      tile = u;
      g.kb0 = 0;
      g.kb1 = a.n_kb;
      g.whole = true;
      g.slot = 0;
      g.ns = 1;
      u += gridDim.x;
    }
    g.mb = (int)(tile % a.n_mb);
    g.nb = (int)(tile / a.n_mb);
    return true;
  }
};

__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// The 16-bit activation type: bf16 (F16 = false) or fp16 (F16 = true).
// kMagic: two copies of a value whose unit in the last place is 1 (128 in
// bf16, 1024 in fp16), so OR-ing a 4-bit code into its mantissa gives
// magic + code exactly.
template <bool F16>
struct W4Type {
  using T = __nv_bfloat16;
  using T2 = __nv_bfloat162;
  static constexpr uint32_t kMagic = 0x43004300u;
  static constexpr float kMagicF = 128.0f;
  static __device__ __forceinline__ T from_float(float x) { return __float2bfloat16_rn(x); }
  static __device__ __forceinline__ float to_float(T x) { return __bfloat162float(x); }
};
template <>
struct W4Type<true> {
  using T = __half;
  using T2 = __half2;
  static constexpr uint32_t kMagic = 0x64006400u;
  static constexpr float kMagicF = 1024.0f;
  static __device__ __forceinline__ T from_float(float x) { return __float2half_rn(x); }
  static __device__ __forceinline__ float to_float(T x) { return __half2float(x); }
};

template <bool F16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  using Ty = W4Type<F16>;
  typename Ty::T2 p;
  p.x = Ty::from_float(lo);
  p.y = Ty::from_float(hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// (code - z) * Delta for the 8 codes of one word, as 8 values of the
// activation type in a uint4 (channel order). Per pair of codes (byte i of
// the word): a byte permute puts code 2i in the low and code 2i+1 (from the
// word shifted by 4) in the high 16-bit half; masking and OR-ing the magic
// constant gives magic + code in each half, exactly; a packed subtract of
// magic + z leaves code - z exactly; a packed multiply by Delta rounds once.
// zz = (magic + z, magic + z) and dd = (Delta, Delta) in the activation type.
template <bool F16>
__device__ __forceinline__ uint4 dequant_word(uint32_t w, uint32_t zz, uint32_t dd) {
  using T2 = typename W4Type<F16>::T2;
  const uint32_t w4 = w >> 4;
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t t = __byte_perm(w, w4, (uint32_t)(i | (i << 4) | ((4 + i) << 8) | ((4 + i) << 12)));
    t = (t & 0x000F000Fu) | W4Type<F16>::kMagic;
    T2 h = *reinterpret_cast<const T2*>(&t);
    h = __hsub2(h, *reinterpret_cast<const T2*>(&zz));
    h = __hmul2(h, *reinterpret_cast<const T2*>(&dd));
    out[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
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

// GPH = quantisation groups per BK / 2 channels (one dequantising thread's
// share of a K step; 1 for g >= BK / 2); F16: fp16 activations and output
// (else bf16); BK: channels per K step (256 for decode-width tiles, so that
// each handshake carries 16 MMAs; 128 otherwise).
template <int GPH, bool F16, int BK>
__global__ void __launch_bounds__(W4_THREADS, 1)
    w4a16_gemm_tcgen05(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                       const W4Args args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bn = args.bn;
  const int AS = args.as, XS = args.xs, RS = args.rs;
  using St = W4Step<BK>;
  const uint32_t x_sub = (uint32_t)bn * W4_SUB * 2;  // one BN x 64 sub-tile; a multiple of 1024
  const uint32_t x_stage = St::NSUB * x_sub;
  uint8_t* sX = smem;                        // [XS][2][BN rows][128 B], swizzled
  uint8_t* sR = sX + XS * x_stage;           // [RS][128 rows][128 B], swizzled
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
  const int nacc = w4_nacc(bn), acc_stride = w4_acc_stride(bn);
  const uint32_t a_col0 = (uint32_t)(nacc * acc_stride);  // first TMEM column of the A ring

  if (warp == 0 || warp == 2) {
    if (lane == 0) {
      // ---------------- TMA producers: packed codes (warp 0, one box per RK
      // steps) or activations (warp 2, NSUB 64-wide boxes per step)
      const bool codes = warp == 0;
      const int depth = codes ? RS : XS;
      Ring ring;
      uint32_t issued = 0, last_parity = 0;
      bool ok = true;
      W4Sched sched(args);
      W4Seg g;
      while (ok && sched.next(args, g)) {
        const int mb = g.mb, nb = g.nb, kb0 = g.kb0, kb1 = g.kb1;
        for (int kb = kb0; kb < kb1; kb += codes ? St::RK : 1) {
          const uint32_t full = codes ? rfull(ring.stage) : xfull(ring.stage);
          const uint32_t empty = codes ? rempty(ring.stage) : xempty(ring.stage);
          if (!mbar_wait_sleep(empty, ring.phase ^ 1u, abort_flag, args.err, codes ? ERR_W4_REMPTY : ERR_W4_XEMPTY,
                               64)) {
            ok = false;
            break;
          }
          if (codes) {
            mbar_arrive_expect_tx(full, W4_R_STAGE);
            tma_load_2d(smem_u32(sR + ring.stage * W4_R_STAGE), &tmW, full, kb * (BK / 8), mb * W4_BM);
          } else {
            mbar_arrive_expect_tx(full, x_stage);
            uint8_t* dst = sX + ring.stage * x_stage;
#pragma unroll
            for (int sb = 0; sb < St::NSUB; ++sb)
              tma_load_2d(smem_u32(dst + sb * x_sub), &tmX, full, kb * BK + sb * W4_SUB, nb * bn);
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
      // ---------------- MMA issuer: BK / 16 MMAs (K = 16 each) per step
      // kind::f16 with both operands fp16 (format 0) or both bf16 (format 1)
      const uint32_t idesc = F16 ? ((1u << 4) | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(W4_BM >> 4) << 24))
                                 : idesc_bf16_f32(W4_BM, bn);
      // descriptor of activation stage 0; a stage, a sub-tile and a K offset
      // only move the start-address field (address >> 4; shared addresses are
      // below 256 KB)
      const uint64_t dx0 = desc_kmajor_sw128(smem_u32(sX));
      Ring xr, ar;
      bool ok = true;
      int local = 0;
      W4Sched sched(args);
      W4Seg g;
      for (; ok && sched.next(args, g); ++local) {
        const int kb0 = g.kb0, kb1 = g.kb1;
        const int acc = local % nacc;
        const uint32_t use = (uint32_t)(local / nacc);
        if (!mbar_wait(tempty(acc), (use & 1u) ^ 1u, abort_flag, args.err, ERR_W4_TEMPTY)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * acc_stride;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(xfull(xr.stage), xr.phase, abort_flag, args.err, ERR_W4_XFULL) ||
              !mbar_wait(afull(ar.stage), ar.phase, abort_flag, args.err, ERR_W4_AFULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_tmem = tmem_base + a_col0 + ar.stage * St::A_COLS;
          const uint64_t dx = dx0 + ((uint64_t)(xr.stage * x_stage) >> 4);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint32_t sub = (uint32_t)(k >> 2), kq = (uint32_t)(k & 3);
            mma_f16_tmem_a(d_tmem, a_tmem + k * 8, dx + ((sub * x_sub + kq * 32) >> 4), idesc,
                           (kb != kb0) || (k != 0));
          }
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
    // ---------------- dequantisation: warp w, lane l takes output channel
    // r = 32 (w % 4) + l (its TMEM lane) and channels h BK/2 .. (h+1) BK/2 - 1 of each step
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int h = (warp - 3) >> 2;
    const uint32_t a_lane = tmem_base + ((uint32_t)(quad * 32) << 16) + a_col0 + (uint32_t)(h * (BK / 4));
    const int sw = r & 7;
    Ring rr, ar;
    bool ok = true;
    W4Sched sched(args);
    W4Seg g;
    while (ok && sched.next(args, g)) {
      const int kb0 = g.kb0, kb1 = g.kb1;
      const int row = g.mb * W4_BM + r;
      const bool valid = row < args.d_out;
      const __half* srow = args.scales + (long long)(valid ? row : 0) * args.ng;
      const __half* zrow = args.zeros + (long long)(valid ? row : 0) * args.ng;
      // step and zero point of the GPH groups of this thread's BK / 2 channels. The
      // raw fp16 values of step kb + 2 are loaded while step kb is processed
      // and converted only when their step comes, so the loads stay in flight.
      using Ty = W4Type<F16>;
      auto load_params = [&](int kb, __half (&dq)[GPH], __half (&zq)[GPH]) {
#pragma unroll
        for (int q = 0; q < GPH; ++q) {
          const int ch = kb * BK + h * (BK / 2) + q * ((BK / 2) / GPH);
          const int gi = min(ch >> args.group_shift, args.ng - 1);
          const bool ld = valid && AWQ_IDX_OK((long long)row * args.ng + gi, (long long)args.d_out * args.ng,
                                              BS_W4_PARAMS);
          dq[q] = ld ? srow[gi] : __float2half_rn(0.0f);
          zq[q] = ld ? zrow[gi] : __float2half_rn(0.0f);
        }
      };
      __half d0[GPH], z0[GPH], d1[GPH], z1[GPH], d2[GPH], z2[GPH];  // steps kb, kb + 1, kb + 2
      load_params(kb0, d0, z0);
      if (kb0 + 1 < kb1) load_params(kb0 + 1, d1, z1);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (kb + 2 < kb1) load_params(kb + 2, d2, z2);
        uint32_t dc[GPH], zc[GPH];
#pragma unroll
        for (int q = 0; q < GPH; ++q) {
          const float dv = __half2float(d0[q]), zv = __half2float(z0[q]);
          dc[q] = pack2<F16>(dv, dv);                              // fp16 step: exact in fp16, rounded in bf16
          zc[q] = pack2<F16>(Ty::kMagicF + zv, Ty::kMagicF + zv);  // integer z <= 15: exact
          d0[q] = d1[q];
          z0[q] = z1[q];
          d1[q] = d2[q];
          z1[q] = z2[q];
        }
        // step kk of the code box: CHUNKS 16-byte chunks of row r from
        // 2 CHUNKS kk + CHUNKS h, swizzled
        const int kk = (kb - kb0) & (St::RK - 1);
        bool have = true;
        if (kk == 0) have = mbar_wait_sleep(rfull(rr.stage), rr.phase, abort_flag, args.err, ERR_W4_RFULL, 32);
        if (!__all_sync(0xffffffffu, have)) {
          ok = false;
          break;
        }
        const uint8_t* rrow = sR + rr.stage * W4_R_STAGE + r * 128;
        const int c0 = 2 * St::CHUNKS * kk + St::CHUNKS * h;
        uint32_t words[4 * St::CHUNKS];
#pragma unroll
        for (int c = 0; c < St::CHUNKS; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(rrow + (((c0 + c) ^ sw) << 4));
          words[4 * c] = w.x;
          words[4 * c + 1] = w.y;
          words[4 * c + 2] = w.z;
          words[4 * c + 3] = w.w;
        }
        if (kk == St::RK - 1 || kb == kb1 - 1) {
          __syncwarp();
          if (lane == 0) mbar_arrive(rempty(rr.stage));
          rr.next(RS);
        }
        have = mbar_wait_sleep(aempty(ar.stage), ar.phase ^ 1u, abort_flag, args.err, ERR_W4_AEMPTY, 32);
        if (!__all_sync(0xffffffffu, have)) {
          ok = false;
          break;
        }
        tc_fence_after();  // the MMAs that read this A stage have completed
        constexpr int NW = 4 * St::CHUNKS;  // words of the thread's BK / 2 channels
        constexpr int WPG = NW / GPH;       // words per group among them
#pragma unroll
        for (int half32 = 0; half32 < NW / 8; ++half32) {  // 32 TMEM columns per tcgen05.st
          uint32_t cols[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int wi = 8 * half32 + c;
            const uint4 v = dequant_word<F16>(words[wi], zc[wi / WPG], dc[wi / WPG]);
            cols[4 * c] = v.x;
            cols[4 * c + 1] = v.y;
            cols[4 * c + 2] = v.z;
            cols[4 * c + 3] = v.w;
          }
          tmem_st_32x32b_x32(a_lane + ar.stage * St::A_COLS + 32 * half32, cols);
        }
        tmem_st_wait();
        tc_fence_before();
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
    W4Sched sched(args);
    W4Seg g;
    for (; sched.next(args, g); ++local) {
      const int mb = g.mb, nb = g.nb;
      const int acc = local % nacc;
      const uint32_t use = (uint32_t)(local / nacc);
      // the accumulator takes a whole tile: wait without spinning
      const bool ready = mbar_wait_sleep(tfull(acc), use & 1u, abort_flag, args.err, ERR_W4_TFULL, 256);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const int o = mb * W4_BM + r;
      const int t0 = nb * bn;
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * acc_stride;
      for (int c = 0; c * 32 < bn; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + c * 32, v);
        tmem_ld_wait();
        // tokens t0 + 32c + j for j < jn are inside both the tile and N
        const int jn = min(32, min(bn - c * 32, args.N - (t0 + c * 32)));
        if (o < args.d_out) {
          const long long e0 = (long long)(t0 + c * 32) * args.d_out + o;
          if (g.whole) {
            typename W4Type<F16>::T* y = static_cast<typename W4Type<F16>::T*>(args.Y) + e0;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < jn && AWQ_IDX_OK(e0 + (long long)j * args.d_out, (long long)args.N * args.d_out, BS_W4_Y))
                y[(long long)j * args.d_out] = W4Type<F16>::from_float(__uint_as_float(v[j]));
          } else {
            float* P = args.P + (long long)g.slot * args.p_stride + e0;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < jn && AWQ_IDX_OK(e0 + (long long)j * args.d_out, (long long)args.N * args.d_out, BS_W4_P))
                P[(long long)j * args.d_out] = __uint_as_float(v[j]);
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

// Tiles that two or more CTAs touch, found on the host from the shapes: tile
// index and the number of partial slabs.
constexpr int W4_MAX_FIX = 160;
struct W4Fixups {
  int n;
  int tile[W4_MAX_FIX];
  int ns[W4_MAX_FIX];
};

// Stream-K fix-up: block (b, y) sums the partial slabs of split tile
// fx.tile[b] in slab order for 1024 of its elements (token-major, output
// channel fastest; 4 per thread, 256 apart, so that each load instruction is
// coalesced) and writes them rounded to the activation type.
template <bool F16>
__global__ void w4a16_streamk_reduce(const float* __restrict__ P, long long p_stride, int slots, int N, int d_out,
                                     int bn, int n_mb, const __grid_constant__ W4Fixups fx, void* __restrict__ Yv) {
  using T = typename W4Type<F16>::T;
  T* Y = static_cast<T*>(Yv);
  if (!AWQ_IDX_OK(blockIdx.x, fx.n, BS_W4_FIXUP)) return;
  const int tile = fx.tile[blockIdx.x], ns = min(fx.ns[blockIdx.x], slots);
  const int o0 = (tile % n_mb) * W4_BM, tok0 = (tile / n_mb) * bn;
  const int rows = min(W4_BM, d_out - o0), toks = min(bn, N - tok0);
  long long idx[4];
  bool in[4];
  float acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int e = blockIdx.y * 1024 + k * 256 + threadIdx.x;
    const int j = e / rows, r = e - j * rows;
    idx[k] = (long long)(tok0 + j) * d_out + o0 + r;
    in[k] = e < rows * toks && AWQ_IDX_OK(idx[k], (long long)N * d_out, BS_W4_FIXUP);
    acc[k] = 0.0f;
  }
  for (int sl = 0; sl < ns; ++sl) {
    const float* Ps = P + (long long)sl * p_stride;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (in[k]) acc[k] += Ps[idx[k]];
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (in[k]) Y[idx[k]] = W4Type<F16>::from_float(acc[k]);
}

// Fold S^-1 into the producer of X: row i of p [d_in, inner] (bf16 or fp16)
// becomes p / s_i, the quotient in fp32 (correctly rounded division) rounded
// to nearest even. VEC = 8: eight elements of one row per thread (inner a
// multiple of 8, p 16-byte aligned); VEC = 1: one element per thread.
template <int VEC, bool F16>
__global__ void fold_inv_scales_kernel(const float* __restrict__ s, long long d_in, long long inner, void* pv) {
  using Ty = W4Type<F16>;
  typename Ty::T* p = static_cast<typename Ty::T*>(pv);
  const long long units = d_in * inner / VEC;
  for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < units;
       u += (long long)gridDim.x * blockDim.x) {
    const long long e = u * VEC;
    if (!AWQ_IDX_OK(e / inner, d_in, BS_FOLD_S) || !AWQ_SPAN_OK(e, VEC, d_in * inner, BS_FOLD_P)) continue;
    const float si = s[e / inner];
    if constexpr (VEC == 8) {
      uint4 w = reinterpret_cast<const uint4*>(p)[u];
      uint32_t* hw = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const typename Ty::T2 v = *reinterpret_cast<const typename Ty::T2*>(&hw[q]);
        hw[q] = pack2<F16>(Ty::to_float(v.x) / si, Ty::to_float(v.y) / si);
      }
      reinterpret_cast<uint4*>(p)[u] = w;
    } else {
      p[e] = Ty::from_float(Ty::to_float(p[e]) / si);
    }
  }
}

}  // namespace awq
