// C ABI of the AWQ search library (declared in include/awq.h): argument
// validation, workspace layout, TMA descriptor set-up and the launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "../../include/awq.h"
#include "awq_kernels.cuh"
#include "gemm_pair_sm100.cuh"
#include "gemm_sm100.cuh"
#include "w4a16_sm100.cuh"

using namespace awq;

namespace {

constexpr size_t kAlign = 1024;
// search workspace header: [0, 4) device error word, [256, 260) tile counter of the GEMMs
constexpr size_t kTileCounterOffset = 256;
constexpr long long kGramMaxPairs = 74;  // CTA pairs of the G' product (148 SMs)
constexpr int kStatsTargetBlocks = 148 * 4;  // one wave at 4 resident blocks per SM
constexpr int kGroupN = 8;
// raster width (column tiles) of the CTA-pair contraction: with 16, concurrent
// pairs share A panels over more column tiles (C5: 19.0 instead of 30.8 GB of
// DRAM reads per launch, 3 % faster; C2: the full width, 2 % faster); the
// full width at C5 was slower (the G' slice no longer stays in L2)
#ifndef AWQ_PAIR_GROUP_N
#define AWQ_PAIR_GROUP_N 16
#endif

inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }
inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline cudaStream_t as_stream(awq_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// ------------------------------------------------------------------ validation
awq_status check_cfg(const awq_qcfg* cfg) {
  if (!cfg) return AWQ_ERR_INVALID_ARG;
  if (cfg->bits < 2 || cfg->bits > 4) return AWQ_ERR_INVALID_ARG;
  const int g = cfg->group;  // 0: one step for the whole layer (per tensor)
  if (g != 0 && (g < 8 || g > 256 || (g & (g - 1)) != 0)) return AWQ_ERR_INVALID_ARG;
  if (cfg->symmetric != 0 && cfg->symmetric != 1) return AWQ_ERR_INVALID_ARG;
  if (cfg->n_alpha < 1 || cfg->n_alpha > MAX_ALPHA) return AWQ_ERR_INVALID_ARG;
  if (cfg->form < AWQ_FORM_AUTO || cfg->form > AWQ_FORM_GRAM) return AWQ_ERR_INVALID_ARG;
  if (!(cfg->eps_a <= 0.f || std::isfinite(cfg->eps_a))) return AWQ_ERR_INVALID_ARG;
  if (cfg->alphas) {
    for (int k = 0; k < cfg->n_alpha; ++k)
      if (!(cfg->alphas[k] >= 0.f && cfg->alphas[k] <= 1.f)) return AWQ_ERR_INVALID_ARG;
  }
  return AWQ_OK;
}

// sizes valid for the search / pack: d_in a multiple of g (hence of 8); bounds
// keep every index of the kernels and TMA coordinates inside int32.
awq_status check_layer_shape(int64_t d_out, int64_t d_in, const awq_qcfg* cfg) {
  if (d_out < 1 || d_in < 8 || d_in % 8 != 0) return AWQ_ERR_SHAPE;
  if (cfg->group == 0 ? d_in % FQ_CPT != 0 : d_in % cfg->group != 0) return AWQ_ERR_SHAPE;
  if (d_in > (1 << 20) || d_out > (1 << 24)) return AWQ_ERR_SHAPE;
  const long long M = (long long)cfg->n_alpha * cdiv(d_out, GEMM_BM) * GEMM_BM;
  if (M > (long long)INT32_MAX / 2) return AWQ_ERR_SHAPE;
  return AWQ_OK;
}

awq_status check_tokens(int64_t N) {
  if (N < 1 || N > (int64_t)INT32_MAX / 2) return AWQ_ERR_SHAPE;
  return AWQ_OK;
}

double alpha_value(const awq_qcfg* cfg, int k) {
  return cfg->alphas ? (double)cfg->alphas[k] : (double)k / (double)cfg->n_alpha;
}

float eps_value(const awq_qcfg* cfg) { return cfg->eps_a > 0.f ? cfg->eps_a : 1e-4f; }

// ------------------------------------------------------------------ device checks
awq_status check_device(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return AWQ_ERR_CUDA;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return AWQ_ERR_CUDA;
  if (major != 10 || minor != 0) return AWQ_ERR_UNSUPPORTED;
  if (num_sms && cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return AWQ_ERR_CUDA;
  return AWQ_OK;
}

awq_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

// ------------------------------------------------------------------ stats layout
struct StatsLayout {
  int col_blocks, rows_per_chunk, n_chunks;
  size_t off_part, total;
};

StatsLayout stats_layout(int64_t N, int64_t d_in) {
  StatsLayout L{};
  L.col_blocks = (int)cdiv(d_in, STATS_COLS);
  long long rpc = cdiv((long long)N * L.col_blocks, kStatsTargetBlocks);
  rpc = cdiv(rpc < 64 ? 64 : rpc, 64) * 64;
  L.rows_per_chunk = (int)rpc;
  L.n_chunks = (int)cdiv(N, rpc);
  L.off_part = kAlign;  // [0, 1024): error word
  L.total = L.off_part + align_up((size_t)L.n_chunks * d_in * sizeof(double));
  return L;
}

// ------------------------------------------------------------------ search layout
struct SearchLayout {
  int form;         // 1 direct, 2 Gram
  int n_alpha;
  int d_out_pad;
  long long M;      // rows of the dW stack
  int n_blocks_n;   // column tiles of the contraction
  int n_red_chunks; // blocks per alpha in the row reduction
  size_t off_s, off_inv, off_dw, off_part, off_blk, off_loss64, off_seg, off_rows64, off_ext, off_g, off_gpart, total;
};

// sum over 256-wide column blocks J of width(J) * min(d_in, 256 (J + 1)): the
// multiply-adds per row of the block-triangular Gram contraction
double tri_macs_per_row(int64_t d_in) {
  double t = 0.0;
  for (int64_t j0 = 0; j0 < d_in; j0 += GEMM_BN) {
    const int64_t w = d_in - j0 < GEMM_BN ? d_in - j0 : GEMM_BN;
    const int64_t k = j0 + GEMM_BN < d_in ? j0 + GEMM_BN : d_in;
    t += (double)w * (double)k;
  }
  return t;
}

int choose_form(int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg) {
  if (cfg->form == AWQ_FORM_DIRECT || cfg->form == AWQ_FORM_GRAM) return cfg->form;
  const double direct = (double)cfg->n_alpha * d_out * d_in * N;
  const double tri = tri_macs_per_row(d_in);
  const double gram = (double)N * tri + (double)cfg->n_alpha * d_out * tri;
  return direct <= gram ? AWQ_FORM_DIRECT : AWQ_FORM_GRAM;
}

// Per-tensor scratch: keys of the column max and min of W [d_in] each, then
// the extremes (max, min) of every candidate [MAX_ALPHA][2].
size_t ext_bytes(int64_t d_in) {
  return align_up((size_t)2 * d_in * sizeof(uint32_t)) + align_up((size_t)2 * MAX_ALPHA * sizeof(float));
}

SearchLayout search_layout(int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg) {
  SearchLayout L{};
  L.form = choose_form(d_out, d_in, N, cfg);
  L.n_alpha = cfg->n_alpha;
  L.d_out_pad = (int)(cdiv(d_out, GEMM_BM) * GEMM_BM);
  L.M = (long long)L.n_alpha * L.d_out_pad;
  L.n_blocks_n = (int)cdiv(L.form == AWQ_FORM_DIRECT ? N : d_in, GEMM_BN);
  L.n_red_chunks = (int)cdiv(d_out, REDUCE_THREADS);
  size_t off = kAlign;  // [0, 1024): error word and tile counter
  L.off_s = off;      off += align_up((size_t)L.n_alpha * d_in * sizeof(float));
  L.off_inv = off;    off += align_up((size_t)L.n_alpha * d_in * sizeof(float));
  L.off_dw = off;     off += align_up((size_t)L.M * d_in * 2);
  L.off_part = off;   off += align_up((size_t)L.n_blocks_n * L.M * sizeof(float));
  L.off_blk = off;    off += align_up((size_t)L.n_alpha * L.n_red_chunks * sizeof(double));
  L.off_loss64 = off; off += align_up((size_t)L.n_alpha * sizeof(double));
  L.off_seg = off;    off += align_up((size_t)MAX_ALPHA * MAX_SEG * sizeof(double));
  L.off_rows64 = off; off += align_up((size_t)L.M * sizeof(double));  // segmented search: fp64 row losses
  L.off_ext = off;    off += ext_bytes(d_in);  // per tensor: column extremes and candidate extremes
  if (L.form == AWQ_FORM_GRAM) {
    L.off_g = off;    off += align_up((size_t)d_in * d_in * 2);
    L.off_gpart = off;  // G' last wave split in K: at most one fp32 256 x 256 piece per pair
    off += align_up((size_t)kGramMaxPairs * PAIR_BM * PAIR_BN * sizeof(float));
  }
  L.total = off;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off); }

awq_status check_search_common(int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg, void* ws,
                               size_t ws_bytes, SearchLayout* L) {
  awq_status st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if ((st = check_layer_shape(d_out, d_in, cfg)) != AWQ_OK) return st;
  if ((st = check_tokens(N)) != AWQ_OK) return st;
  if (!ws || !aligned(ws, 256)) return AWQ_ERR_INVALID_ARG;
  *L = search_layout(d_out, d_in, N, cfg);
  if (ws_bytes < L->total) return AWQ_ERR_WORKSPACE;
  return AWQ_OK;
}

// ------------------------------------------------------------------ TMA
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D map of 16-bit elements (bf16 unless given) over a row-major [rows, cols]
// matrix with leading dimension ld (elements), box = box_rows x 64 columns,
// 128-byte swizzle, zero fill.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows,
              CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)GEMM_BK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D uint32 map over the packed codes [rows, words], box of box_words x
// box_rows (128-byte swizzle: box_words = 32).
bool make_map_u32(CUtensorMap* m, const void* base, uint64_t rows, uint64_t words, uint32_t box_words,
                  uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {words, rows};
  cuuint64_t strides[1] = {words * 4};
  cuuint32_t box[2] = {box_words, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Elements from each epilogue pointer of GemmArgs to the end of the buffer it
// points into (for the debug build's host-side index checks).
struct GemmExtents {
  long long part = 0, E = 0, C = 0;
};

// Debug build: does the furthest element the GEMM epilogue may touch lie inside
// each buffer? Every epilogue access sits behind m < M and col < N; partials
// take one row of part_ld per column tile (per 32-column chunk in EPI_DOT32),
// E is read and C written 8 elements at a time (TRI_DIAG_STORE: columns
// relative to the tile, at most bn of them).
template <int MODE>
bool gemm_extents_ok(const GemmArgs& a, int bn, const GemmExtents& x) {
  if (!kBoundsCheck) return true;
  const long long M = a.M, n8 = cdiv(a.N, 8) * 8;
  if (MODE == EPI_SUMSQ || MODE == EPI_DOT || MODE == EPI_DOT32) {
    const long long rows = MODE == EPI_DOT32 ? (long long)a.n_blocks_n * (bn / 32) : a.n_blocks_n;
    if (a.part_ld < M || (rows - 1) * a.part_ld + M > x.part) return false;
  }
  if (MODE == EPI_DOT || MODE == EPI_DOT32) {
    if (a.ldE < n8 || (M - 1) * a.ldE + n8 > x.E) return false;
  }
  if (MODE == EPI_STORE) {
    const long long w = a.tri == TRI_DIAG_STORE ? (n8 < bn ? n8 : bn) : n8;
    if (a.ldC < w || (M - 1) * a.ldC + w > x.C) return false;
  }
  return true;
}

// D = A[M, K] * B[Nr, K]^T with the given epilogue.
// MN = true: A and B are row-major [K, M] / [K, Nr] matrices read transposed.
template <int MODE, bool MN = false>
awq_status run_gemm(const void* A, long long M, long long lda, const void* B, long long Nr, long long ldb, long long K,
                    GemmArgs args, int tri, int num_sms, cudaStream_t st, const GemmExtents& ext) {
  CUtensorMap ta, tb;
  if (MN) {
    if (!make_map(&ta, A, K, M, lda, GEMM_BK)) return AWQ_ERR_CUDA;
    if (!make_map(&tb, B, K, Nr, ldb, GEMM_BK)) return AWQ_ERR_CUDA;
  } else {
    if (!make_map(&ta, A, M, K, lda, GEMM_BM)) return AWQ_ERR_CUDA;
    // TRI_DIAG: B is the compact [Nr, 256] diagonal-block matrix
    if (!make_map(&tb, B, Nr, tri == TRI_DIAG ? GEMM_BN : K, ldb, GEMM_BN)) return AWQ_ERR_CUDA;
  }
  args.M = (int)M;
  args.N = (int)Nr;
  args.K = (int)K;
  args.n_blocks_m = (int)cdiv(M, GEMM_BM);
  args.n_blocks_n = (int)cdiv(Nr, GEMM_BN);
  args.group_n = kGroupN < args.n_blocks_n ? kGroupN : args.n_blocks_n;
  args.tri = tri;
  const long long tiles = tri == TRI_LOWER_STORE ? tri_lower_tiles(args.n_blocks_m)
                          : tri == TRI_DIAG_STORE ? args.n_blocks_m
                                                  : (long long)args.n_blocks_m * args.n_blocks_n;
  if (tiles > INT32_MAX) return AWQ_ERR_SHAPE;
  args.num_tiles = (int)tiles;
  if (!gemm_extents_ok<MODE>(args, GEMM_BN, ext)) return AWQ_ERR_BOUNDS;
  if (cudaFuncSetAttribute(gemm_bf16_tcgen05<MODE, MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           GEMM_SMEM_BYTES) != cudaSuccess ||
      cudaFuncSetAttribute(gemm_bf16_tcgen05<MODE, MN>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared) != cudaSuccess)
    return AWQ_ERR_CUDA;
  if (cudaMemsetAsync(args.tile_counter, 0, sizeof(int), st) != cudaSuccess) return AWQ_ERR_CUDA;
  const int grid = (int)(tiles < num_sms ? tiles : num_sms);
  gemm_bf16_tcgen05<MODE, MN><<<grid, GEMM_THREADS, GEMM_SMEM_BYTES, st>>>(ta, tb, args);
  return launch_status();
}

// The contraction and the Gram product on CTA pairs (gemm_pair_sm100.cuh):
// 256 x 256 tiles. MN = true: A and B are row-major [K, M] / [K, Nr]
// matrices read transposed.
template <int MODE, bool MN = false>
awq_status run_gemm_pair(const void* A, long long M, long long lda, const void* B, long long Nr, long long ldb,
                         long long K, GemmArgs args, int tri, int num_sms, cudaStream_t st, const GemmExtents& ext) {
  CUtensorMap ta, tb;
  if (MN) {
    if (!make_map(&ta, A, K, M, lda, GEMM_BK)) return AWQ_ERR_CUDA;
    if (!make_map(&tb, B, K, Nr, ldb, GEMM_BK)) return AWQ_ERR_CUDA;
  } else {
    if (!make_map(&ta, A, M, K, lda, 128)) return AWQ_ERR_CUDA;
    if (!make_map(&tb, B, Nr, K, ldb, 128)) return AWQ_ERR_CUDA;
  }
  args.M = (int)M;
  args.N = (int)Nr;
  args.K = (int)K;
  args.n_blocks_m = (int)cdiv(M, PAIR_BM);
  args.n_blocks_n = (int)cdiv(Nr, PAIR_BN);
  args.group_n = AWQ_PAIR_GROUP_N < args.n_blocks_n ? AWQ_PAIR_GROUP_N : args.n_blocks_n;
  args.tri = tri;
  // TRI_LOWER_STORE: the tiles of the lower block triangle (row block mb, column blocks 0 .. mb)
  const long long tiles = tri == TRI_LOWER_STORE ? (long long)args.n_blocks_m * (args.n_blocks_m + 1) / 2
                                                 : (long long)args.n_blocks_m * args.n_blocks_n;
  if (tiles > INT32_MAX) return AWQ_ERR_SHAPE;
  args.num_tiles = (int)tiles;
  if (!gemm_extents_ok<MODE>(args, PAIR_BN, ext)) return AWQ_ERR_BOUNDS;
  if (cudaFuncSetAttribute(gemm_pair_bf16_tcgen05<MODE, MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           PAIR_SMEM_BYTES) != cudaSuccess)
    return AWQ_ERR_CUDA;
  if (cudaMemsetAsync(args.tile_counter, 0, sizeof(int), st) != cudaSuccess) return AWQ_ERR_CUDA;
  const long long pairs = tiles < num_sms / 2 ? tiles : num_sms / 2;
  // G' (tiles of equal K): a last wave of R <= pairs / 2 tiles runs as R x S
  // pieces of K / S steps (S = pairs / R, at least 2 steps a piece)
  args.tail_first = (int)tiles;
  args.tail_split = 1;
  long long R = 0;
  if (MODE == EPI_STORE && tri == TRI_LOWER_STORE && args.tail_part && tiles > pairs) {
    R = tiles % pairs;
    const long long n_kb = cdiv(K, GEMM_BK);
    long long S = R > 0 ? pairs / R : 0;
    if (S > n_kb / 2) S = n_kb / 2;
    if (R > 0 && S >= 2 && R * S <= kGramMaxPairs) {
      args.tail_first = (int)(tiles - R);
      args.tail_split = (int)S;
    } else {
      R = 0;
    }
  }
  gemm_pair_bf16_tcgen05<MODE, MN><<<(unsigned)(2 * pairs), GEMM_THREADS, PAIR_SMEM_BYTES, st>>>(ta, tb, args);
  awq_status rs = launch_status();
  if (rs != AWQ_OK || R == 0) return rs;
  gram_tail_fixup<<<dim3((unsigned)R, (unsigned)(PAIR_BM * PAIR_BN / 1024)), 256, 0, st>>>(args);
  return launch_status();
}

#ifndef AWQ_GEMM_PAIR
#define AWQ_GEMM_PAIR 1
#endif


// Grid of a grid-stride kernel with 256-thread blocks: enough blocks for the
// work, at most one wave of resident blocks.
template <typename K>
int elementwise_grid(K kernel, long long threads_needed, int num_sms) {
  long long blocks = cdiv(threads_needed, 256);
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, 0) != cudaSuccess || per_sm < 1) per_sm = 1;
  const long long cap = (long long)num_sms * per_sm;
  if (blocks > cap) blocks = cap;
  return (int)(blocks < 1 ? 1 : blocks);
}

}  // namespace

// =================================================================== C ABI
extern "C" {

const char* awq_status_str(awq_status s) {
  switch (s) {
    case AWQ_OK: return "AWQ_OK";
    case AWQ_ERR_INVALID_ARG: return "AWQ_ERR_INVALID_ARG: null or misaligned pointer, or bad config value";
    case AWQ_ERR_SHAPE: return "AWQ_ERR_SHAPE: unsupported or inconsistent sizes";
    case AWQ_ERR_WORKSPACE: return "AWQ_ERR_WORKSPACE: workspace smaller than required";
    case AWQ_ERR_NONFINITE: return "AWQ_ERR_NONFINITE: a candidate loss was NaN or infinite";
    case AWQ_ERR_CUDA: return "AWQ_ERR_CUDA: CUDA runtime call or launch failed";
    case AWQ_ERR_DEVICE: return "AWQ_ERR_DEVICE: a kernel gave up a bounded wait";
    case AWQ_ERR_UNSUPPORTED: return "AWQ_ERR_UNSUPPORTED: needs an sm_100 (B200) device";
    case AWQ_ERR_BOUNDS: return "AWQ_ERR_BOUNDS: an index check of the debug build failed";
  }
  return "AWQ_ERR_UNKNOWN";
}

size_t awq_stats_workspace_size(int64_t N, int64_t d_in) {
  if (N < 1 || d_in < 8) return 0;
  return stats_layout(N, d_in).total;
}

awq_status awq_act_stats(const void* X, int64_t N, int64_t d_in, float* a, void* ws, size_t ws_bytes,
                         awq_stream_t stream) {
  if (!X || !a || !ws) return AWQ_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(ws, 256)) return AWQ_ERR_INVALID_ARG;
  if (check_tokens(N) != AWQ_OK || d_in < 8 || d_in % 8 != 0 || d_in > (1 << 20)) return AWQ_ERR_SHAPE;
  const StatsLayout L = stats_layout(N, d_in);
  if (ws_bytes < L.total) return AWQ_ERR_WORKSPACE;
  awq_status st = check_device(nullptr);
  if (st != AWQ_OK) return st;
  cudaStream_t s = as_stream(stream);
  dim3 grid(L.col_blocks, L.n_chunks);
  act_absmean_partial<<<grid, STATS_THREADS, 0, s>>>(static_cast<const __nv_bfloat16*>(X), N, (int)d_in,
                                                     L.rows_per_chunk, at<double>(ws, L.off_part));
  if ((st = launch_status()) != AWQ_OK) return st;
  act_absmean_final<<<(unsigned)cdiv(d_in, FINAL_COLS), STATS_FINAL_THREADS, 0, s>>>(at<double>(ws, L.off_part),
                                                                                   L.n_chunks, N, (int)d_in, a);
  return launch_status();
}

size_t awq_search_workspace_size(int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg) {
  if (check_cfg(cfg) != AWQ_OK || check_layer_shape(d_out, d_in, cfg) != AWQ_OK || check_tokens(N) != AWQ_OK)
    return 0;
  return search_layout(d_out, d_in, N, cfg).total;
}

int32_t awq_search_form(int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg) {
  if (check_cfg(cfg) != AWQ_OK || check_layer_shape(d_out, d_in, cfg) != AWQ_OK || check_tokens(N) != AWQ_OK)
    return 0;
  return choose_form(d_out, d_in, N, cfg);
}

awq_status awq_step_scales(const float* a, int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg, void* ws,
                           size_t ws_bytes, awq_stream_t stream) {
  SearchLayout L;
  awq_status st = check_search_common(d_out, d_in, N, cfg, ws, ws_bytes, &L);
  if (st != AWQ_OK) return st;
  if (!a) return AWQ_ERR_INVALID_ARG;
  if ((st = check_device(nullptr)) != AWQ_OK) return st;
  AlphaGrid grid{};
  for (int k = 0; k < cfg->n_alpha; ++k) grid.v[k] = alpha_value(cfg, k);
  cudaStream_t s = as_stream(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return AWQ_ERR_CUDA;
  const dim3 sgrid((unsigned)cdiv(d_in, SCALES_THREADS), (unsigned)cfg->n_alpha);
  candidate_scales<<<sgrid, SCALES_THREADS, 0, s>>>(a, (int)d_in, grid, eps_value(cfg), at<float>(ws, L.off_s),
                                                   at<float>(ws, L.off_inv));
  return launch_status();
}

// Per-tensor extremes into the scratch at `ext_ws` (ext_bytes(d_in)): column
// max / min of W, then (max, min) of v = w s for each of the n scale vectors
// s_all[n][d_in], at ext_table(ext_ws, d_in).
float* ext_table(void* ext_ws, int64_t d_in) {
  return reinterpret_cast<float*>(static_cast<uint8_t*>(ext_ws) + align_up((size_t)2 * d_in * sizeof(uint32_t)));
}

awq_status launch_tensor_extremes(const void* W, int64_t d_out, int64_t d_in, const float* s_all, int n,
                                  void* ext_ws, int sms, cudaStream_t st) {
  uint32_t* kmax = static_cast<uint32_t*>(ext_ws);
  uint32_t* kmin = kmax + d_in;
  if (cudaMemsetAsync(kmax, 0, (size_t)d_in * sizeof(uint32_t), st) != cudaSuccess ||
      cudaMemsetAsync(kmin, 0xFF, (size_t)d_in * sizeof(uint32_t), st) != cudaSuccess)
    return AWQ_ERR_CUDA;
  const int xb = (int)cdiv(d_in / 8, 256);
  long long yb = (4LL * sms + xb - 1) / xb;
  if (yb > d_out) yb = d_out;
  if (yb < 1) yb = 1;
  const int rows_per_block = (int)cdiv(d_out, yb);
  yb = cdiv(d_out, rows_per_block);
  col_minmax<<<dim3(xb, (unsigned)yb), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(W), (int)d_out, (int)d_in,
                                                     rows_per_block, kmax, kmin);
  tensor_extremes<<<n, 256, 0, st>>>(kmax, kmin, s_all, (int)d_in, ext_table(ext_ws, d_in));
  return launch_status();
}

// Fake quantisation of grid points [k0, k1) into their slices of the dW stack.
// max_per_sm > 0 caps the grid at that many blocks per SM.
awq_status launch_fake_quant(const void* W, int64_t d_out, int64_t d_in, const awq_qcfg* cfg, const SearchLayout& L,
                             void* ws, int k0, int k1, int sms, int max_per_sm, cudaStream_t st,
                             const ClipTable* clip_table = nullptr) {
  ClipTable clips;
  for (int k = 0; k < MAX_ALPHA; ++k) clips.c[k] = 1.0f;
  if (clip_table)
    for (int k = k0; k < k1; ++k) clips.c[k - k0] = clip_table->c[k];
  const long long slice = (long long)L.d_out_pad * d_in;
  float* ext = nullptr;
  if (cfg->group == 0) {
    // per tensor: the layer-wide extremes of every candidate first
    awq_status es = launch_tensor_extremes(W, d_out, d_in, at<float>(ws, L.off_s) + (long long)k0 * d_in, k1 - k0,
                                           at<void>(ws, L.off_ext), sms, st);
    if (es != AWQ_OK) return es;
    ext = ext_table(at<void>(ws, L.off_ext), d_in);
  }
  auto launch = [&](auto kernel, int cpt) {
    const long long units = (long long)(L.d_out_pad / FQ_ROWS) * (d_in / cpt);
    int grid = elementwise_grid(kernel, units, sms);
    if (max_per_sm > 0 && grid > sms * max_per_sm) grid = sms * max_per_sm;
    kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(W), (int)d_out, (int)d_in, L.d_out_pad,
                                 at<float>(ws, L.off_s) + (long long)k0 * d_in,
                                 at<float>(ws, L.off_inv) + (long long)k0 * d_in, k1 - k0, cfg->bits,
                                 cfg->symmetric, at<__nv_bfloat16>(ws, L.off_dw) + k0 * slice, clips, ext);
  };
  constexpr int C = FQ_CPT;
  switch (cfg->group) {
    case 0: launch(fake_quant_delta<C, FQ_ROWS, 1, true>, C); break;
    case 8: launch(fake_quant_delta<8, FQ_ROWS, 1>, 8); break;
    case 16: launch(fake_quant_delta<(C < 16 ? C : 16), FQ_ROWS, 16 / (C < 16 ? C : 16)>, (C < 16 ? C : 16)); break;
    case 32: launch(fake_quant_delta<(C < 32 ? C : 32), FQ_ROWS, 32 / (C < 32 ? C : 32)>, (C < 32 ? C : 32)); break;
    case 64: launch(fake_quant_delta<C, FQ_ROWS, 64 / C>, C); break;
    case 128: launch(fake_quant_delta<C, FQ_ROWS, 128 / C>, C); break;
    case 256: launch(fake_quant_delta<C, FQ_ROWS, 256 / C>, C); break;
    default: return AWQ_ERR_INVALID_ARG;
  }
  return launch_status();
}

// The error contraction for grid points [k0, k1): rows [k0, k1) * d_out_pad of
// the dW stack.
awq_status launch_contract(const void* X, int64_t d_in, int64_t N, const SearchLayout& L, void* ws, int k0, int k1,
                           int sms, cudaStream_t st) {
  GemmArgs ga{};
  const long long row0 = (long long)k0 * L.d_out_pad;
  const long long rows = (long long)(k1 - k0) * L.d_out_pad;
  ga.part = at<float>(ws, L.off_part) + row0;
  ga.part_ld = L.M;
  ga.err = at<int>(ws, 0);
  ga.tile_counter = at<int>(ws, kTileCounterOffset);
  const __nv_bfloat16* dw = at<__nv_bfloat16>(ws, L.off_dw) + row0 * d_in;
  GemmExtents ext;
  ext.part = (long long)L.n_blocks_n * L.M - row0;
  ext.E = (L.M - row0) * d_in;
  if (L.form == AWQ_FORM_DIRECT) {
    if (AWQ_GEMM_PAIR) return run_gemm_pair<EPI_SUMSQ>(dw, rows, d_in, X, N, d_in, d_in, ga, TRI_NONE, sms, st, ext);
    return run_gemm<EPI_SUMSQ>(dw, rows, d_in, X, N, d_in, d_in, ga, TRI_NONE, sms, st, ext);
  }
  ga.E = dw;
  ga.ldE = d_in;
  if (AWQ_GEMM_PAIR)
    return run_gemm_pair<EPI_DOT>(dw, rows, d_in, at<void>(ws, L.off_g), d_in, d_in, d_in, ga, TRI_K, sms, st, ext);
  return run_gemm<EPI_DOT>(dw, rows, d_in, at<void>(ws, L.off_g), d_in, d_in, d_in, ga, TRI_K, sms, st, ext);
}

awq_status awq_step_fake_quant(const void* W, int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg, void* ws,
                               size_t ws_bytes, awq_stream_t stream) {
  SearchLayout L;
  awq_status st = check_search_common(d_out, d_in, N, cfg, ws, ws_bytes, &L);
  if (st != AWQ_OK) return st;
  if (!W || !aligned(W, 16)) return AWQ_ERR_INVALID_ARG;
  int sms = 0;
  if ((st = check_device(&sms)) != AWQ_OK) return st;
  return launch_fake_quant(W, d_out, d_in, cfg, L, ws, 0, cfg->n_alpha, sms, 0, as_stream(stream));
}

awq_status awq_step_gram(const void* X, int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg, void* ws,
                         size_t ws_bytes, awq_stream_t stream) {
  SearchLayout L;
  awq_status st = check_search_common(d_out, d_in, N, cfg, ws, ws_bytes, &L);
  if (st != AWQ_OK) return st;
  if (L.form != AWQ_FORM_GRAM) return AWQ_OK;
  if (!X || !aligned(X, 16)) return AWQ_ERR_INVALID_ARG;
  int sms = 0;
  if ((st = check_device(&sms)) != AWQ_OK) return st;
  GemmArgs ga{};
  ga.C = at<__nv_bfloat16>(ws, L.off_g);
  ga.ldC = d_in;
  ga.err = at<int>(ws, 0);
  ga.tile_counter = at<int>(ws, kTileCounterOffset);
  ga.tail_part = at<float>(ws, L.off_gpart);
  GemmExtents ext;
  ext.C = (long long)d_in * d_in;
  // G = X^T X with both operands read transposed from X [N, d_in] (MN-major)
  return run_gemm_pair<EPI_STORE, true>(X, d_in, d_in, X, d_in, d_in, N, ga, TRI_LOWER_STORE, sms,
                                        as_stream(stream), ext);
}

awq_status awq_step_contract(const void* X, int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg, void* ws,
                             size_t ws_bytes, awq_stream_t stream) {
  SearchLayout L;
  awq_status st = check_search_common(d_out, d_in, N, cfg, ws, ws_bytes, &L);
  if (st != AWQ_OK) return st;
  if (L.form == AWQ_FORM_DIRECT && (!X || !aligned(X, 16))) return AWQ_ERR_INVALID_ARG;
  int sms = 0;
  if ((st = check_device(&sms)) != AWQ_OK) return st;
  return launch_contract(X, d_in, N, L, ws, 0, cfg->n_alpha, sms, as_stream(stream));
}

awq_status awq_step_reduce(int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg, void* ws, size_t ws_bytes,
                           float* losses, int32_t* best, float* s_best, float* row_losses, awq_stream_t stream) {
  SearchLayout L;
  awq_status st = check_search_common(d_out, d_in, N, cfg, ws, ws_bytes, &L);
  if (st != AWQ_OK) return st;
  if (!losses || !best || !s_best) return AWQ_ERR_INVALID_ARG;
  if ((st = check_device(nullptr)) != AWQ_OK) return st;
  cudaStream_t s = as_stream(stream);
  dim3 rgrid(L.n_red_chunks, L.n_alpha);
  row_loss_reduce<<<rgrid, REDUCE_THREADS, 0, s>>>(at<float>(ws, L.off_part), L.n_blocks_n, L.M, (int)d_out,
                                                  L.d_out_pad, row_losses, at<double>(ws, L.off_blk));
  if ((st = launch_status()) != AWQ_OK) return st;
  loss_argmin<<<1, 256, 0, s>>>(at<double>(ws, L.off_blk), L.n_red_chunks, L.n_alpha, at<float>(ws, L.off_s),
                                (int)d_in, losses, at<double>(ws, L.off_loss64), best, s_best, at<int>(ws, 0));
  return launch_status();
}

awq_status awq_search_scales(const void* W, const void* X, const float* a, int64_t d_out, int64_t d_in, int64_t N,
                             const awq_qcfg* cfg, void* ws, size_t ws_bytes, float* losses, int32_t* best,
                             float* s_best, float* row_losses, awq_stream_t stream) {
  SearchLayout L;
  awq_status st = check_search_common(d_out, d_in, N, cfg, ws, ws_bytes, &L);
  if (st != AWQ_OK) return st;
  if (!W || !X || !a || !losses || !best || !s_best) return AWQ_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(X, 16)) return AWQ_ERR_INVALID_ARG;
  if ((st = awq_step_scales(a, d_out, d_in, N, cfg, ws, ws_bytes, stream)) != AWQ_OK) return st;
  if ((st = awq_step_fake_quant(W, d_out, d_in, N, cfg, ws, ws_bytes, stream)) != AWQ_OK) return st;
  if ((st = awq_step_gram(X, d_out, d_in, N, cfg, ws, ws_bytes, stream)) != AWQ_OK) return st;
  if ((st = awq_step_contract(X, d_out, d_in, N, cfg, ws, ws_bytes, stream)) != AWQ_OK) return st;
  return awq_step_reduce(d_out, d_in, N, cfg, ws, ws_bytes, losses, best, s_best, row_losses, stream);
}

awq_status awq_search_scales_segmented(const void* W, const void* X, const float* a, int64_t d_out, int64_t d_in,
                                       int64_t N, const awq_qcfg* cfg, int32_t n_seg, const int64_t* seg_rows,
                                       void* ws, size_t ws_bytes, float* losses, int32_t* best, float* s_best,
                                       float* row_losses, awq_stream_t stream) {
  SearchLayout L;
  awq_status st = check_search_common(d_out, d_in, N, cfg, ws, ws_bytes, &L);
  if (st != AWQ_OK) return st;
  if (!W || !X || !a || !losses || !best || !s_best || !seg_rows) return AWQ_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(X, 16)) return AWQ_ERR_INVALID_ARG;
  if (n_seg < 1 || n_seg > MAX_SEG) return AWQ_ERR_INVALID_ARG;
  if (cfg->group == 0) return AWQ_ERR_UNSUPPORTED;  // one step per layer would span the segments
  SegTable seg{};
  int64_t acc = 0;
  for (int i = 0; i < n_seg; ++i) {
    if (seg_rows[i] < 1) return AWQ_ERR_SHAPE;
    seg.start[i] = (int)acc;
    acc += seg_rows[i];
    if (acc > d_out) return AWQ_ERR_SHAPE;
  }
  if (acc != d_out) return AWQ_ERR_SHAPE;
  seg.start[n_seg] = (int)acc;
  if ((st = awq_step_scales(a, d_out, d_in, N, cfg, ws, ws_bytes, stream)) != AWQ_OK) return st;
  if ((st = awq_step_fake_quant(W, d_out, d_in, N, cfg, ws, ws_bytes, stream)) != AWQ_OK) return st;
  if ((st = awq_step_gram(X, d_out, d_in, N, cfg, ws, ws_bytes, stream)) != AWQ_OK) return st;
  if ((st = awq_step_contract(X, d_out, d_in, N, cfg, ws, ws_bytes, stream)) != AWQ_OK) return st;
  cudaStream_t s = as_stream(stream);
  row_loss_rows<<<dim3((unsigned)cdiv(d_out, REDUCE_THREADS), L.n_alpha), REDUCE_THREADS, 0, s>>>(
      at<float>(ws, L.off_part), L.n_blocks_n, L.M, (int)d_out, L.d_out_pad, row_losses, at<double>(ws, L.off_rows64));
  if ((st = launch_status()) != AWQ_OK) return st;
  segment_loss_reduce<<<dim3(n_seg, L.n_alpha), REDUCE_THREADS, 0, s>>>(at<double>(ws, L.off_rows64), L.M,
                                                                        L.d_out_pad, seg, at<double>(ws, L.off_seg));
  if ((st = launch_status()) != AWQ_OK) return st;
  segment_argmin<<<n_seg, 256, 0, s>>>(at<double>(ws, L.off_seg), n_seg, L.n_alpha, at<float>(ws, L.off_s),
                                       (int)d_in, losses, best, s_best, at<int>(ws, 0));
  return launch_status();
}

namespace {
// Workspace of the per-group clipping search (cfg->n_alpha = number of clip ratios).
struct ClipLayout {
  int n, d_out_pad, n_chunks;  // candidates, padded rows, 32-column chunks of the partials
  long long M;
  size_t off_s, off_inv, off_dw, off_part, off_g, total;
};

ClipLayout clip_layout(int64_t d_out, int64_t d_in, const awq_qcfg* cfg) {
  ClipLayout L{};
  L.n = cfg->n_alpha;
  L.d_out_pad = (int)(cdiv(d_out, GEMM_BM) * GEMM_BM);
  L.M = (long long)L.n * L.d_out_pad;
  L.n_chunks = (int)cdiv(d_in, GEMM_BN) * (GEMM_BN / 32);
  size_t off = kAlign;
  L.off_s = off;    off += align_up((size_t)L.n * d_in * sizeof(float));
  L.off_inv = off;  off += align_up((size_t)L.n * d_in * sizeof(float));
  L.off_dw = off;   off += align_up((size_t)L.M * d_in * 2);
  L.off_part = off; off += align_up((size_t)L.n_chunks * L.M * sizeof(float));
  L.off_g = off;    off += align_up((size_t)d_in * GEMM_BN * 2);
  L.total = off;
  return L;
}

awq_status check_clip_common(int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg, const void* ws,
                             size_t ws_bytes, ClipLayout* L) {
  awq_status st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if ((st = check_layer_shape(d_out, d_in, cfg)) != AWQ_OK) return st;
  if ((st = check_tokens(N)) != AWQ_OK) return st;
  if (cfg->group < 32) return AWQ_ERR_UNSUPPORTED;  // errors are gathered per 32-column chunk
  if (!ws || !aligned(ws, 256)) return AWQ_ERR_INVALID_ARG;
  *L = clip_layout(d_out, d_in, cfg);
  if (ws_bytes < L->total) return AWQ_ERR_WORKSPACE;
  return AWQ_OK;
}
}  // namespace

size_t awq_group_clip_workspace_size(int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg) {
  ClipLayout L;
  if (check_clip_common(d_out, d_in, N, cfg, reinterpret_cast<void*>(256), SIZE_MAX, &L) != AWQ_OK) return 0;
  return L.total;
}

awq_status awq_search_group_clip(const void* W, const void* X, const float* s, const float* clips, int64_t d_out,
                                 int64_t d_in, int64_t N, const awq_qcfg* cfg, void* ws, size_t ws_bytes,
                                 uint8_t* best_clip, float* group_err, awq_stream_t stream) {
  ClipLayout L;
  awq_status st = check_clip_common(d_out, d_in, N, cfg, ws, ws_bytes, &L);
  if (st != AWQ_OK) return st;
  if (!W || !X || !s || !clips || !best_clip) return AWQ_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(X, 16)) return AWQ_ERR_INVALID_ARG;
  ClipTable table{};
  for (int k = 0; k < L.n; ++k) {
    if (!(clips[k] > 0.f && clips[k] <= 1.f)) return AWQ_ERR_INVALID_ARG;
    table.c[k] = clips[k];
  }
  int sms = 0;
  if ((st = check_device(&sms)) != AWQ_OK) return st;
  cudaStream_t cs = as_stream(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(int), cs) != cudaSuccess) return AWQ_ERR_CUDA;
  repeat_scales<<<2 * sms, 256, 0, cs>>>(s, (int)d_in, L.n, at<float>(ws, L.off_s), at<float>(ws, L.off_inv),
                                         at<int>(ws, 0));
  if ((st = launch_status()) != AWQ_OK) return st;
  // candidates: the same scales, one clip ratio each
  SearchLayout SL{};
  SL.d_out_pad = L.d_out_pad;
  SL.off_s = L.off_s;
  SL.off_inv = L.off_inv;
  SL.off_dw = L.off_dw;
  if ((st = launch_fake_quant(W, d_out, d_in, cfg, SL, ws, 0, L.n, sms, 0, cs, &table)) != AWQ_OK) return st;
  // diagonal 256-blocks of G = X^T X, masked to each quantisation group, compact [d_in, 256]
  GemmArgs gs{};
  gs.C = at<__nv_bfloat16>(ws, L.off_g);
  gs.ldC = GEMM_BN;
  gs.err = at<int>(ws, 0);
  gs.tile_counter = at<int>(ws, kTileCounterOffset);
  gs.group = cfg->group;
  // entries outside the stored diagonal (columns past d_in) must read as 0
  if (cudaMemsetAsync(gs.C, 0, (size_t)d_in * GEMM_BN * 2, cs) != cudaSuccess) return AWQ_ERR_CUDA;
  GemmExtents gext;
  gext.C = (long long)d_in * GEMM_BN;
  if ((st = run_gemm<EPI_STORE, true>(X, d_in, d_in, X, d_in, d_in, N, gs, TRI_DIAG_STORE, sms, cs, gext)) !=
      AWQ_OK)
    return st;
  // per (row, 32-column chunk) errors of every candidate: dW[:, J] G_J dW[:, J]^T restricted to the groups
  GemmArgs ga{};
  ga.part = at<float>(ws, L.off_part);
  ga.part_ld = L.M;
  ga.err = at<int>(ws, 0);
  ga.tile_counter = at<int>(ws, kTileCounterOffset);
  ga.E = at<__nv_bfloat16>(ws, L.off_dw);
  ga.ldE = d_in;
  GemmExtents cext;
  cext.part = (long long)L.n_chunks * L.M;
  cext.E = L.M * d_in;
  if ((st = run_gemm<EPI_DOT32>(at<void>(ws, L.off_dw), L.M, d_in, at<void>(ws, L.off_g), d_in, GEMM_BN, d_in, ga,
                                TRI_DIAG, sms, cs, cext)) != AWQ_OK)
    return st;
  const int ng = (int)(d_in / cfg->group);
  const long long units = (long long)ng * d_out;
  group_clip_argmin<<<(unsigned)(cdiv(units, 256) < 8 * sms ? cdiv(units, 256) : 8 * sms), 256, 0, cs>>>(
      at<float>(ws, L.off_part), L.M, (int)d_out, L.d_out_pad, ng, cfg->group / 32, L.n, best_clip, group_err,
      at<int>(ws, 0));
  return launch_status();
}

awq_status awq_workspace_error(void* ws, awq_stream_t stream) {
  if (!ws) return AWQ_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  int word = 0;
  if (cudaMemcpyAsync(&word, ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return AWQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return AWQ_ERR_CUDA;
  if (word == 0) return AWQ_OK;
  if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return AWQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return AWQ_ERR_CUDA;
  return word == ERR_NONFINITE ? AWQ_ERR_NONFINITE : AWQ_ERR_DEVICE;
}

awq_status pack_impl(const void* W, const float* s, int64_t d_out, int64_t d_in, const awq_qcfg* cfg, float clip,
                     const uint8_t* group_clip, const ClipTable& gtable, uint32_t* qweight, void* scales, void* zeros,
                     awq_stream_t stream, void* ws = nullptr, size_t ws_bytes = 0) {
  awq_status st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if ((st = check_layer_shape(d_out, d_in, cfg)) != AWQ_OK) return st;
  if (cfg->group == 0) {  // per tensor: the extremes need scratch
    if (!ws || !aligned(ws, 256)) return ws ? AWQ_ERR_INVALID_ARG : AWQ_ERR_WORKSPACE;
    if (ws_bytes < ext_bytes(d_in)) return AWQ_ERR_WORKSPACE;
    if (group_clip) return AWQ_ERR_UNSUPPORTED;
  }
  if (!(clip > 0.f && clip <= 1.f)) return AWQ_ERR_INVALID_ARG;
  if (!W || !s || !qweight || !scales || !zeros) return AWQ_ERR_INVALID_ARG;
  // qweight: the kernel stores 8-byte pairs of words
  if (!aligned(W, 16) || !aligned(s, 16) || !aligned(qweight, 8) || !aligned(scales, 2) || !aligned(zeros, 2))
    return AWQ_ERR_INVALID_ARG;
  int sms = 0;
  if ((st = check_device(&sms)) != AWQ_OK) return st;
  const float* ext = nullptr;
  if (cfg->group == 0) {
    if ((st = launch_tensor_extremes(W, d_out, d_in, s, 1, ws, sms, as_stream(stream))) != AWQ_OK) return st;
    ext = ext_table(ws, d_in);
  }
  auto launch = [&](auto kernel, int cpt) {
    const long long units = cdiv(d_out, PACK_ROWS) * (d_in / cpt);
    const int grid = elementwise_grid(kernel, units, sms);
    kernel<<<grid, 256, 0, as_stream(stream)>>>(static_cast<const __nv_bfloat16*>(W), s, (int)d_out, (int)d_in,
                                                cfg->bits, cfg->symmetric, qweight, static_cast<__half*>(scales),
                                                static_cast<__half*>(zeros), clip, group_clip, gtable, ext);
  };
  constexpr int C = FQ_CPT;
  switch (cfg->group) {
    case 0: launch(quantize_pack<C, 1, true>, C); break;
    case 8: launch(quantize_pack<8, 1>, 8); break;
    case 16: launch(quantize_pack<(C < 16 ? C : 16), 16 / (C < 16 ? C : 16)>, (C < 16 ? C : 16)); break;
    case 32: launch(quantize_pack<(C < 32 ? C : 32), 32 / (C < 32 ? C : 32)>, (C < 32 ? C : 32)); break;
    case 64: launch(quantize_pack<C, 64 / C>, C); break;
    case 128: launch(quantize_pack<C, 128 / C>, C); break;
    case 256: launch(quantize_pack<C, 256 / C>, C); break;
    default: return AWQ_ERR_INVALID_ARG;
  }
  return launch_status();
}

awq_status awq_quantize_pack_clipped(const void* W, const float* s, int64_t d_out, int64_t d_in, const awq_qcfg* cfg,
                                     float clip, uint32_t* qweight, void* scales, void* zeros, awq_stream_t stream) {
  ClipTable none{};
  return pack_impl(W, s, d_out, d_in, cfg, clip, nullptr, none, qweight, scales, zeros, stream);
}

awq_status awq_quantize_pack(const void* W, const float* s, int64_t d_out, int64_t d_in, const awq_qcfg* cfg,
                             uint32_t* qweight, void* scales, void* zeros, awq_stream_t stream) {
  return awq_quantize_pack_clipped(W, s, d_out, d_in, cfg, 1.0f, qweight, scales, zeros, stream);
}

size_t awq_pack_workspace_size(int64_t d_out, int64_t d_in, const awq_qcfg* cfg) {
  if (check_cfg(cfg) != AWQ_OK || check_layer_shape(d_out, d_in, cfg) != AWQ_OK) return 0;
  return cfg->group == 0 ? ext_bytes(d_in) : 256;
}

awq_status awq_quantize_pack_ws(const void* W, const float* s, int64_t d_out, int64_t d_in, const awq_qcfg* cfg,
                                float clip, void* ws, size_t ws_bytes, uint32_t* qweight, void* scales, void* zeros,
                                awq_stream_t stream) {
  ClipTable none{};
  return pack_impl(W, s, d_out, d_in, cfg, clip, nullptr, none, qweight, scales, zeros, stream, ws, ws_bytes);
}

awq_status awq_quantize_pack_group_clip(const void* W, const float* s, const float* clips, int32_t n_clips,
                                        const uint8_t* best_clip, int64_t d_out, int64_t d_in, const awq_qcfg* cfg,
                                        uint32_t* qweight, void* scales, void* zeros, awq_stream_t stream) {
  if (!clips || !best_clip || n_clips < 1 || n_clips > MAX_ALPHA) return AWQ_ERR_INVALID_ARG;
  ClipTable table;
  for (int k = 0; k < MAX_ALPHA; ++k) table.c[k] = 1.0f;  // indices past n_clips: no clipping
  for (int k = 0; k < n_clips; ++k) {
    if (!(clips[k] > 0.f && clips[k] <= 1.f)) return AWQ_ERR_INVALID_ARG;
    table.c[k] = clips[k];
  }
  return pack_impl(W, s, d_out, d_in, cfg, 1.0f, best_clip, table, qweight, scales, zeros, stream);
}

awq_status awq_search_candidates(const void* W, const void* X, const float* s_cand, const float* clips,
                                 int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg, void* ws,
                                 size_t ws_bytes, float* losses, int32_t* best, float* s_best, float* row_losses,
                                 awq_stream_t stream) {
  SearchLayout L;
  awq_status st = check_search_common(d_out, d_in, N, cfg, ws, ws_bytes, &L);
  if (st != AWQ_OK) return st;
  if (!W || !X || !s_cand || !losses || !best || !s_best) return AWQ_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(X, 16)) return AWQ_ERR_INVALID_ARG;
  ClipTable table;
  for (int k = 0; k < MAX_ALPHA; ++k) table.c[k] = 1.0f;
  if (clips)
    for (int k = 0; k < cfg->n_alpha; ++k) {
      if (!(clips[k] > 0.f && clips[k] <= 1.f)) return AWQ_ERR_INVALID_ARG;
      table.c[k] = clips[k];
    }
  int sms = 0;
  if ((st = check_device(&sms)) != AWQ_OK) return st;
  cudaStream_t s = as_stream(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return AWQ_ERR_CUDA;
  const long long n = (long long)cfg->n_alpha * d_in;
  set_candidate_scales<<<(unsigned)(cdiv(n, 256) < 4 * sms ? cdiv(n, 256) : 4 * sms), 256, 0, s>>>(
      s_cand, n, at<float>(ws, L.off_s), at<float>(ws, L.off_inv), at<int>(ws, 0));
  if ((st = launch_status()) != AWQ_OK) return st;
  if ((st = launch_fake_quant(W, d_out, d_in, cfg, L, ws, 0, cfg->n_alpha, sms, 0, s, &table)) != AWQ_OK) return st;
  if ((st = awq_step_gram(X, d_out, d_in, N, cfg, ws, ws_bytes, stream)) != AWQ_OK) return st;
  if ((st = awq_step_contract(X, d_out, d_in, N, cfg, ws, ws_bytes, stream)) != AWQ_OK) return st;
  return awq_step_reduce(d_out, d_in, N, cfg, ws, ws_bytes, losses, best, s_best, row_losses, stream);
}

awq_status awq_debug_copy_dw(const void* ws, int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg, int32_t k,
                             void* dst, awq_stream_t stream) {
  SearchLayout L;
  awq_status st = check_search_common(d_out, d_in, N, cfg, const_cast<void*>(ws), SIZE_MAX, &L);
  if (st != AWQ_OK) return st;
  if (!dst || k < 0 || k >= cfg->n_alpha) return AWQ_ERR_INVALID_ARG;
  const void* src = static_cast<const uint8_t*>(ws) + L.off_dw + (size_t)k * L.d_out_pad * d_in * 2;
  if (cudaMemcpyAsync(dst, src, (size_t)d_out * d_in * 2, cudaMemcpyDeviceToDevice, as_stream(stream)) != cudaSuccess)
    return AWQ_ERR_CUDA;
  return AWQ_OK;
}

}  // extern "C"

// =================================================================== statistics without allocation
// Some callers cannot allocate device memory at the point where they need the
// activation statistics: code that runs inside a memory pool or arena they do
// not own, a plugin host that hands out only its own tensors, or a region where
// a cudaMalloc would synchronise the device. For them awq_act_stats_noalloc
// takes its scratch from a fixed array that lives in this library's device
// image instead of from a caller workspace.
namespace {

constexpr long long kNoallocScratchDoubles = 1ll << 19;  // 4 MiB of fp64 partial sums
constexpr int kNoallocMaxDevices = 64;

// Loaded on every device that loads the library and held until the process exits.
static __device__ __align__(256) double g_noalloc_stats_scratch[kNoallocScratchDoubles];

// One call's partial sums are n_chunks * d_in doubles. stats_layout gives a
// single chunk when a row of column blocks already fills its target grid, and
// otherwise at most target / col_blocks + 1 chunks, so the partials never
// exceed (2 * target) * STATS_COLS doubles for any d_in the array admits.
static_assert(2ll * kStatsTargetBlocks * STATS_COLS <= kNoallocScratchDoubles,
              "the statistics' partial sums must fit the scratch array for every admitted d_in");

std::mutex g_noalloc_mu;
struct NoallocSlot {
  unsigned long long ctx_id;  // context the address belongs to (0: none yet)
  void* ptr;
};
NoallocSlot g_noalloc_slot[kNoallocMaxDevices] = {};

// Process-unique id of the current context, or 0 when the runtime has not made
// one current yet (cuCtxGetId ids are never reused within a process).
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array on the current device. In host code the
// array's name is only a host-side stand-in, so its address is looked up with
// the device current and cached per device, together with the id of the
// context it was found in. If that context is destroyed and another one takes
// its place (cudaDeviceReset), the library's module, and the array with it, is
// loaded anew at another address: the changed context id makes the next call
// look the address up again instead of using the stale one.
awq_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
  if (dev < 0 || dev >= kNoallocMaxDevices) return AWQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc_slot[dev];
  const unsigned long long id = current_context_id();
  if (!slot.ptr || id == 0 || id != slot.ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_stats_scratch) != cudaSuccess || !p) return AWQ_ERR_CUDA;
    slot.ptr = p;
    slot.ctx_id = current_context_id();  // the lookup made the device's context current
  }
  *out = slot.ptr;
  return AWQ_OK;
}

}  // namespace

extern "C" awq_status awq_act_stats_noalloc(const void* X, int64_t N, int64_t d_in, float* a, awq_stream_t stream) {
  if (!X || !a) return AWQ_ERR_INVALID_ARG;
  if (!aligned(X, 16)) return AWQ_ERR_INVALID_ARG;
  if (check_tokens(N) != AWQ_OK || d_in < 8 || d_in % 8 != 0 || d_in > kNoallocScratchDoubles) return AWQ_ERR_SHAPE;
  // same chunking as awq_act_stats; its partial sums always fit the array (see
  // the static_assert above), checked again here before anything is enqueued
  const StatsLayout L = stats_layout(N, d_in);
  if ((long long)L.n_chunks * d_in > kNoallocScratchDoubles) return AWQ_ERR_SHAPE;
  awq_status st = check_device(nullptr);
  if (st != AWQ_OK) return st;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != AWQ_OK) return st;
  double* part = static_cast<double*>(scratch);
  cudaStream_t s = as_stream(stream);
  // every partial the second kernel reads is written by the first one in this
  // call, so nothing needs clearing between calls
  act_absmean_partial<<<dim3(L.col_blocks, L.n_chunks), STATS_THREADS, 0, s>>>(
      static_cast<const __nv_bfloat16*>(X), N, (int)d_in, L.rows_per_chunk, part);
  if ((st = launch_status()) != AWQ_OK) return st;
  act_absmean_final<<<(unsigned)cdiv(d_in, FINAL_COLS), STATS_FINAL_THREADS, 0, s>>>(part, L.n_chunks, N, (int)d_in, a);
  return launch_status();
}

// ===================================================================== inference side
namespace {
constexpr int kW4TargetCtas = 148;  // CTAs of the W4A16 grid: one per SM

struct W4Plan {
  int bn, bk, n_mb, n_nb, n_kb;
  int as, xs, rs;  // ring depths
  bool sk;         // stream-K ranges (few tiles) or whole tiles
  int grid, slots;
  long long tiles, units, p_stride;
  int smem;
  size_t ws;
};
static_assert(kW4TargetCtas - 1 <= W4_MAX_FIX, "split tiles per launch");

// The tiles of a stream-K plan that two or more ranges touch (each found at
// its first inner range boundary), with their slab counts.
void w4_fixups(const W4Plan& p, W4Fixups& fx) {
  fx.n = 0;
  for (long long c = 1; c < p.grid; ++c) {
    const long long b = w4_sk_begin(c, p.grid, p.units), tile = b / p.n_kb, t0 = tile * p.n_kb;
    if (b == t0 || w4_sk_cta(t0, p.grid, p.units) != c - 1) continue;
    fx.tile[fx.n] = (int)tile;
    fx.ns[fx.n] = (int)(w4_sk_cta(t0 + p.n_kb - 1, p.grid, p.units) - (c - 1) + 1);
    ++fx.n;
  }
}

W4Plan w4_plan(int64_t N, int64_t d_out, int64_t d_in, int group) {
  W4Plan p{};
  p.bn = N <= 16 ? 16 : N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
  // ring depths: deep packed-code rings for narrow (weight-streaming) tiles
  // K steps of 256 channels for decode-width tiles (16 MMAs per handshake),
  // 128 otherwise (a 256-wide activation stage of 256 tokens would take
  // 128 KB). Ring depths: codes and activations in shared memory, dequantised
  // weights in the tensor-memory columns the accumulators leave (an MMA's
  // commit lands about a microsecond after issue and holds its stages).
  p.bk = p.bn <= 64 && group > 8 ? 256 : 128;  // g = 8 keeps 128 (sixteen groups a thread would spill)
  if (p.bn <= 32) { p.xs = p.bn == 16 ? 8 : 6; p.rs = 6; }
  else if (p.bn == 64) { p.xs = 4; p.rs = 4; }
  else if (p.bn == 128) { p.xs = 4; p.rs = 4; }
  else { p.xs = 3; p.rs = 2; }
  p.as = w4_max_as(p.bn, p.bk) < W4_MAX_AS ? w4_max_as(p.bn, p.bk) : W4_MAX_AS;
  p.smem = w4_smem_bytes(p.xs, p.rs, p.bn, p.bk);
  p.n_mb = (int)cdiv(d_out, W4_BM);
  p.n_nb = (int)cdiv(N, p.bn);
  p.n_kb = (int)cdiv(d_in, p.bk);
  p.tiles = (long long)p.n_mb * p.n_nb;
  p.units = p.tiles * p.n_kb;
  // Fewer than two waves of whole tiles: stream-K over equal ranges of
  // (tile, K step) units, at least 4 K steps per CTA (the rings' fill and
  // drain is paid per CTA). The grid is fixed by the shapes alone, so that
  // the workspace can be sized without a device.
  p.sk = p.tiles < 2 * kW4TargetCtas && p.n_kb > 1;
  if (p.sk) {
    const long long g = p.units / 4 < kW4TargetCtas ? p.units / 4 : kW4TargetCtas;
    p.grid = (int)(g > 1 ? g : 1);
    p.slots = 1;
    for (long long t = 0; t < p.tiles; ++t) {
      const long long n = w4_sk_cta(t * p.n_kb + p.n_kb - 1, p.grid, p.units) - w4_sk_cta(t * p.n_kb, p.grid, p.units) + 1;
      if (n > p.slots) p.slots = (int)n;
    }
  } else {
    p.grid = (int)(p.tiles < kW4TargetCtas ? p.tiles : kW4TargetCtas);
    p.slots = 1;
  }
  p.p_stride = (N * d_out + 3) / 4 * 4;
  p.ws = kAlign + (p.slots > 1 ? align_up((size_t)p.slots * p.p_stride * sizeof(float)) : 0);
  return p;
}

awq_status check_w4(int64_t N, int64_t d_out, int64_t d_in, const awq_qcfg* cfg) {
  if (!cfg) return AWQ_ERR_INVALID_ARG;
  if (cfg->bits < 2 || cfg->bits > 4) return AWQ_ERR_INVALID_ARG;
  const int g = cfg->group;
  if (g < 8 || g > 256 || (g & (g - 1)) != 0) return AWQ_ERR_INVALID_ARG;
  if (N < 1 || d_out < 1 || d_in < 32) return AWQ_ERR_SHAPE;
  if (d_in % 32 != 0 || d_in % g != 0) return AWQ_ERR_SHAPE;  // packed rows: a multiple of 16 bytes
  if (d_in > (1 << 20) || d_out > (1 << 24) || N > (1 << 24)) return AWQ_ERR_SHAPE;
  if ((long long)N * d_out > (long long)INT32_MAX * 4) return AWQ_ERR_SHAPE;
  if (w4_plan(N, d_out, d_in, cfg->group).tiles > INT32_MAX) return AWQ_ERR_SHAPE;
  return AWQ_OK;
}
}  // namespace

extern "C" size_t awq_w4a16_workspace_size(int64_t N, int64_t d_out, int64_t d_in, const awq_qcfg* cfg) {
  if (check_w4(N, d_out, d_in, cfg) != AWQ_OK) return 0;
  return w4_plan(N, d_out, d_in, cfg->group).ws;
}

extern "C" awq_status awq_w4a16_gemm(const void* X, awq_dtype dtype, const uint32_t* qweight, const void* scales,
                                     const void* zeros, int64_t N, int64_t d_out, int64_t d_in, const awq_qcfg* cfg,
                                     void* Y, void* ws, size_t ws_bytes, awq_stream_t stream) {
  awq_status st = check_w4(N, d_out, d_in, cfg);
  if (st != AWQ_OK) return st;
  if (dtype != AWQ_DTYPE_BF16 && dtype != AWQ_DTYPE_F16) return AWQ_ERR_INVALID_ARG;
  const bool f16 = dtype == AWQ_DTYPE_F16;
  if (!X || !qweight || !scales || !zeros || !Y || !ws) return AWQ_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(qweight, 16) || !aligned(scales, 2) || !aligned(zeros, 2) || !aligned(Y, 16) ||
      !aligned(ws, 256))
    return AWQ_ERR_INVALID_ARG;
  const W4Plan p = w4_plan(N, d_out, d_in, cfg->group);
  if (ws_bytes < p.ws) return AWQ_ERR_WORKSPACE;
  int sms = 0;
  if ((st = check_device(&sms)) != AWQ_OK) return st;
  cudaStream_t cs = as_stream(stream);
  CUtensorMap tx, tw;
  if (!make_map(&tx, X, N, d_in, d_in, p.bn, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
    return AWQ_ERR_CUDA;
  if (!make_map_u32(&tw, qweight, d_out, d_in / 8, 32, W4_BM, CU_TENSOR_MAP_SWIZZLE_128B))
    return AWQ_ERR_CUDA;
  W4Args a{};
  a.N = (int)N;
  a.d_out = (int)d_out;
  a.d_in = (int)d_in;
  a.bn = p.bn;
  a.n_mb = p.n_mb;
  a.n_nb = p.n_nb;
  a.sk = p.sk ? 1 : 0;
  a.n_kb = p.n_kb;
  a.num_tiles = (int)p.tiles;
  a.units = p.units;
  a.ng = (int)(d_in / cfg->group);
  int sh = 0;
  while ((1 << sh) < cfg->group) ++sh;
  a.group_shift = sh;
  a.as = p.as;
  a.xs = p.xs;
  a.rs = p.rs;
  if (p.smem > W4_SMEM_LIMIT) return AWQ_ERR_UNSUPPORTED;
  a.scales = static_cast<const __half*>(scales);
  a.zeros = static_cast<const __half*>(zeros);
  a.Y = Y;
  a.P = p.slots > 1 ? at<float>(ws, kAlign) : nullptr;
  a.p_stride = p.p_stride;
  a.err = at<int>(ws, 0);
  if (cudaMemsetAsync(ws, 0, sizeof(int), cs) != cudaSuccess) return AWQ_ERR_CUDA;
  const int grid = p.grid;
  auto launch = [&](auto kernel) -> awq_status {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem) != cudaSuccess)
      return AWQ_ERR_CUDA;
    kernel<<<grid, W4_THREADS, p.smem, cs>>>(tx, tw, a);
    return launch_status();
  };
  // template arguments: quantisation groups per BK / 2 channels, activation type, K step
  auto dispatch = [&](auto f16_tag, auto bk_tag) -> awq_status {
    constexpr bool F = decltype(f16_tag)::value;
    constexpr int K = decltype(bk_tag)::value;
    constexpr int H = K / 2;  // channels per dequantising thread and step
    switch (cfg->group) {
      case 8:
        if constexpr (K == 128) return launch(w4a16_gemm_tcgen05<H / 8, F, K>);
        return AWQ_ERR_UNSUPPORTED;  // the plan keeps g = 8 on 128-channel steps
      case 16: return launch(w4a16_gemm_tcgen05<H / 16, F, K>);
      case 32: return launch(w4a16_gemm_tcgen05<H / 32, F, K>);
      case 64: return launch(w4a16_gemm_tcgen05<(H / 64 > 0 ? H / 64 : 1), F, K>);
      default: return launch(w4a16_gemm_tcgen05<(H / 128 > 0 ? H / 128 : 1), F, K>);  // 128 and 256
    }
  };
  using T = std::true_type;
  using Fa = std::false_type;
  using K128 = std::integral_constant<int, 128>;
  using K256 = std::integral_constant<int, 256>;
  if (f16)
    st = p.bk == 256 ? dispatch(T{}, K256{}) : dispatch(T{}, K128{});
  else
    st = p.bk == 256 ? dispatch(Fa{}, K256{}) : dispatch(Fa{}, K128{});
  if (st != AWQ_OK || p.slots == 1) return st;
  W4Fixups fx;
  w4_fixups(p, fx);
  if (fx.n == 0) return AWQ_OK;
  const dim3 rgrid((unsigned)fx.n, (unsigned)cdiv((long long)W4_BM * p.bn, 1024));
  if (f16)
    w4a16_streamk_reduce<true><<<rgrid, 256, 0, cs>>>(a.P, p.p_stride, p.slots, (int)N, (int)d_out, p.bn, p.n_mb, fx, Y);
  else
    w4a16_streamk_reduce<false><<<rgrid, 256, 0, cs>>>(a.P, p.p_stride, p.slots, (int)N, (int)d_out, p.bn, p.n_mb, fx,
                                                       Y);
  return launch_status();
}

extern "C" awq_status awq_fold_inv_scales(const float* s, int64_t d_in, void* p, awq_dtype dtype, int64_t inner,
                                          awq_stream_t stream) {
  if (!s || !p) return AWQ_ERR_INVALID_ARG;
  if (dtype != AWQ_DTYPE_BF16 && dtype != AWQ_DTYPE_F16) return AWQ_ERR_INVALID_ARG;
  if (d_in < 1 || inner < 1 || d_in > (1 << 24) || inner > (1 << 24)) return AWQ_ERR_SHAPE;
  if (!aligned(p, 2) || !aligned(s, 4)) return AWQ_ERR_INVALID_ARG;
  int sms = 0;
  awq_status st = check_device(&sms);
  if (st != AWQ_OK) return st;
  cudaStream_t cs = as_stream(stream);
  const bool vec = inner % 8 == 0 && aligned(p, 16);
  const long long units = d_in * inner / (vec ? 8 : 1);
  const long long blocks = cdiv(units, 256);
  const unsigned grid = (unsigned)(blocks < 8LL * sms ? blocks : 8LL * sms);
  const bool f16 = dtype == AWQ_DTYPE_F16;
  if (vec && f16)
    fold_inv_scales_kernel<8, true><<<grid, 256, 0, cs>>>(s, d_in, inner, p);
  else if (vec)
    fold_inv_scales_kernel<8, false><<<grid, 256, 0, cs>>>(s, d_in, inner, p);
  else if (f16)
    fold_inv_scales_kernel<1, true><<<grid, 256, 0, cs>>>(s, d_in, inner, p);
  else
    fold_inv_scales_kernel<1, false><<<grid, 256, 0, cs>>>(s, d_in, inner, p);
  return launch_status();
}

extern "C" awq_status awq_selftest_bounded_wait(void* ws, awq_stream_t stream) {
  if (!ws || !aligned(ws, 256)) return AWQ_ERR_INVALID_ARG;
  awq_status st = check_device(nullptr);
  if (st != AWQ_OK) return st;
  cudaStream_t cs = as_stream(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(int), cs) != cudaSuccess) return AWQ_ERR_CUDA;
  bounded_wait_selftest<<<1, 32, 0, cs>>>(at<int>(ws, 0));
  return launch_status();
}

extern "C" int32_t awq_bounds_checks_enabled(void) { return kBoundsCheck ? 1 : 0; }

extern "C" awq_status awq_bounds_error(int32_t* site, awq_stream_t stream) {
  if (site) *site = 0;
  if (!kBoundsCheck) return AWQ_OK;
  cudaStream_t cs = as_stream(stream);
  int word = 0;
  if (cudaMemcpyFromSymbolAsync(&word, g_bounds_err, sizeof(int), 0, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return AWQ_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return AWQ_ERR_CUDA;
  if (word == 0) return AWQ_OK;
  const int zero = 0;
  if (cudaMemcpyToSymbolAsync(g_bounds_err, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, cs) != cudaSuccess)
    return AWQ_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return AWQ_ERR_CUDA;
  if (site) *site = word & 0xFF;
  return AWQ_ERR_BOUNDS;
}

extern "C" awq_status awq_selftest_bounds(void* ws, size_t ws_bytes, awq_stream_t stream) {
  if (!ws || !aligned(ws, 256)) return AWQ_ERR_INVALID_ARG;
  if (ws_bytes < 256) return AWQ_ERR_WORKSPACE;
  if (!kBoundsCheck) return AWQ_ERR_UNSUPPORTED;
  awq_status st = check_device(nullptr);
  if (st != AWQ_OK) return st;
  // ws holds 64 ints; the kernel declares an extent of 63 and stores to element 63
  bounds_selftest<<<1, 32, 0, as_stream(stream)>>>(at<int>(ws, 0), 63);
  return launch_status();
}
