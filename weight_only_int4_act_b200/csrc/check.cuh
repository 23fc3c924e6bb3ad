// Debug build (-DAWQ_BOUNDS_CHECK): explicit index checks on the global loads
// and stores that the kernels address by hand (the SIMT kernels, the W4A16
// kernel's step / zero loads and output stores, the stream-K fix-up and the
// fold). A check compares the span an access touches with the extent that the
// kernel's own arguments give the buffer. When it fails, the access is skipped
// (a load yields zero) and ERR_BOUNDS | site goes to the device word
// g_bounds_err (the first failure is kept); awq_bounds_error() reads and
// clears it on the host. No check traps or asserts, so the context stays usable.
//
// In the release build every check is the constant `true` and its arguments
// are not evaluated: the kernels compile to the same code as without them.
//
// The tensor-core GEMMs are not instrumented here: their operands come through
// TMA tensor maps (the hardware bounds each box; elements outside the map read
// as zero) and their epilogue stores sit behind m < M and col < N guards. In
// the debug build their launcher checks on the host that the furthest element
// those guards admit lies inside the buffer it was given.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace awq {

constexpr int ERR_BOUNDS = 0x800;  // recorded as ERR_BOUNDS | site

// The access whose check failed (low byte of the recorded code).
enum BoundsSite : int {
  BS_STATS_X = 1,   // act_absmean_partial: X rows
  BS_STATS_PART,    // act_absmean_partial: chunk sums
  BS_FQ_W,          // fake_quant_delta: W
  BS_FQ_S,          // fake_quant_delta: s_all / inv_all
  BS_FQ_DW,         // fake_quant_delta: dW stack
  BS_LOSS_PART,     // row_loss_reduce / segment_loss_reduce: partials
  BS_LOSS_ROW,      // row_loss_reduce / segment_loss_reduce: per-row losses
  BS_ARGMIN_S,      // loss_argmin / segment_argmin: s of the chosen alpha
  BS_MINMAX_W,      // col_minmax: W
  BS_MINMAX_KEY,    // col_minmax: column keys
  BS_CLIP_PART,     // group_clip_argmin: partials
  BS_CLIP_OUT,      // group_clip_argmin: errors and choices
  BS_PACK_W,        // quantize_pack: W
  BS_PACK_S,        // quantize_pack: s
  BS_PACK_CLIP,     // quantize_pack: per-group clip choices
  BS_PACK_Q,        // quantize_pack: qweight
  BS_PACK_SZ,       // quantize_pack: scales / zeros
  BS_W4_PARAMS,     // w4a16_gemm_tcgen05: step / zero loads
  BS_W4_Y,          // w4a16_gemm_tcgen05: Y stores
  BS_W4_P,          // w4a16_gemm_tcgen05: stream-K partial stores
  BS_W4_FIXUP,      // w4a16_streamk_reduce: split tiles, partials and Y
  BS_GRAM_FIX,      // gram_tail_fixup: partial pieces and G'
  BS_FOLD_S,        // fold_inv_scales_kernel: s
  BS_FOLD_P,        // fold_inv_scales_kernel: the folded tensor
  BS_SELFTEST = 0x7F,
};

// First failed check of this library's kernels on this device (0: none).
// Present in both builds; only the debug build writes it.
__device__ int g_bounds_err;

#ifdef AWQ_BOUNDS_CHECK
constexpr bool kBoundsCheck = true;

// Does [i, i + w) lie inside [0, n)? If not, record the site and say no.
__device__ __forceinline__ bool span_ok(long long i, long long w, long long n, int site) {
  if (i >= 0 && w >= 0 && i + w <= n) return true;
  atomicCAS(&g_bounds_err, 0, ERR_BOUNDS | site);
  return false;
}
#define AWQ_SPAN_OK(i, w, n, site) ::awq::span_ok((long long)(i), (long long)(w), (long long)(n), (site))
#else
constexpr bool kBoundsCheck = false;
#define AWQ_SPAN_OK(i, w, n, site) true
#endif
#define AWQ_IDX_OK(i, n, site) AWQ_SPAN_OK(i, 1, n, site)

// The failure path of the checks: one thread stores to element `n` of a
// buffer whose extent it declares as n. The check refuses the store and
// records BS_SELFTEST. The host gives the kernel a buffer of n + 1 elements,
// so the refused store would still have stayed inside the allocation.
__global__ void bounds_selftest(int* buf, int n) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    if (AWQ_IDX_OK(n, n, BS_SELFTEST)) buf[n] = 1;
  }
}

}  // namespace awq
