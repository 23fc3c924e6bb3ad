/*
 * awq.h - C ABI of the B200 (sm_100a) library for the AWQ calibration and
 * scale-search path of one linear layer.
 *
 * The operations follow these pages (cited by title and section):
 *   [P1] "AWQ量化" tutorial (aiqz.cc): 量化基础, 激活感知, 缩放保护, GPTQ对比.
 *   [P2] "AWQ量化技术解析：激活感知的权重量化革命" (kwkr.cn): §2.1, §4.2.
 *   [P3] "大模型的开发应用（十八）：大模型量化：GPTQ与AWQ" (ewbang.com): AWQ 二.2.
 *   [P4] "AWQ 量化全流程拆解：将 70B 大模型塞进单张消费级 GPU" (lnrq.cn): §三.
 *   [P5] "AWQ" (scholia-log, inference-quantization/2_AWQ): §1.1, §1.2, §2.1-2.3,
 *        §3.1-3.3, §4.1.
 *
 * Conventions for every entry point:
 *   - W is bf16 [d_out, d_in], row-major (rows are output channels).
 *   - X is bf16 [N, d_in], row-major (N calibration tokens x input channels).
 *   - Groups are g consecutive input channels within one row of W.
 *   - Every pointer argument is DEVICE memory owned by the caller, unless the
 *     comment says "host". The library allocates no device memory and keeps
 *     no state of its own beyond what awq_act_stats_noalloc documents;
 *     scratch memory is the caller's workspace.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream). A returned AWQ_OK means the work was
 *     validated and enqueued. Errors the device finds (a wait that timed out,
 *     non-finite losses) are written to a word in the workspace and read back
 *     by awq_workspace_error().
 *   - Argument and shape errors are returned before anything is enqueued; no
 *     entry point aborts the process.
 *   - Device pointers must be 16-byte aligned; workspaces 256-byte aligned.
 */
#ifndef AWQ_B200_H
#define AWQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* awq_stream_t; /* identical to cudaStream_t */

typedef enum {
  AWQ_OK = 0,
  AWQ_ERR_INVALID_ARG = 1, /* null pointer, misaligned pointer, bad config value */
  AWQ_ERR_SHAPE = 2,       /* d_in % g, d_in % 8, empty or oversized dimensions */
  AWQ_ERR_WORKSPACE = 3,   /* workspace smaller than the matching *_workspace_size() */
  AWQ_ERR_NONFINITE = 4,   /* a candidate loss was NaN or infinite (device-side) */
  AWQ_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
  AWQ_ERR_DEVICE = 6,      /* a kernel gave up a bounded wait (device-side) */
  AWQ_ERR_UNSUPPORTED = 7, /* no sm_100 device, or a configuration not built */
  AWQ_ERR_BOUNDS = 8       /* debug build: an index check failed (awq_bounds_error) */
} awq_status;

typedef enum { AWQ_FORM_AUTO = 0, AWQ_FORM_DIRECT = 1, AWQ_FORM_GRAM = 2 } awq_form;

/* Quantiser and search settings ([P4] §三 quant_config: w_bit, q_group_size,
 * zero_point). */
typedef struct {
  int32_t bits;         /* 2, 3 or 4; codes are stored one per 4-bit nibble */
  int32_t group;        /* g in {8, 16, 32, 64, 128, 256}, d_in % g == 0; or 0: per tensor
                           (one step for the whole layer, as in [P1] 量化基础; d_in % 16
                           == 0; not for the segmented or group-clip searches nor the
                           W4A16 product, and the pack needs awq_quantize_pack_ws) */
  int32_t symmetric;    /* 0: min/max affine with zero point; 1: symmetric */
  int32_t n_alpha;      /* grid size, 1..64 */
  int32_t form;         /* awq_form: how the loss contraction is evaluated */
  float eps_a;          /* floor on a_i before the power; <= 0 selects 1e-4 */
  const float* alphas;  /* HOST array [n_alpha] of grid points in [0, 1], or
                           NULL for alpha_k = k / n_alpha ([P3] AWQ 二.2) */
} awq_qcfg;

/* Human-readable name of a status; never NULL. */
const char* awq_status_str(awq_status s);

/* ---------------------------------------------------------------------------
 * Step a1: activation statistics.
 * a[i] = (1/N) sum_t |X[t, i]|  ([P1] 激活感知, importance Omega_i; [P5] §1.2,
 * a_i = E|x_i|). X: bf16 [N, d_in]; a: float [d_in]. Partial sums are kept in
 * float64 and combined in a fixed order (bitwise repeatable).
 * ws: scratch of awq_stats_workspace_size(N, d_in) bytes.
 * Errors: AWQ_ERR_INVALID_ARG (null/misaligned), AWQ_ERR_SHAPE (N < 1,
 * d_in < 8 or d_in % 8), AWQ_ERR_WORKSPACE, AWQ_ERR_CUDA.
 * ------------------------------------------------------------------------- */
size_t awq_stats_workspace_size(int64_t N, int64_t d_in);
awq_status awq_act_stats(const void* X_bf16, int64_t N, int64_t d_in, float* a, void* ws,
                         size_t ws_bytes, awq_stream_t stream);

/* ---------------------------------------------------------------------------
 * Step a1 for callers that cannot allocate device memory (no counterpart on
 * the pages; it exists for the library's users). Same result as
 * awq_act_stats, but the fp64 partial sums go to a fixed scratch array of
 * 4 MiB (524288 doubles) compiled into the library, which every GPU that
 * loads the library holds until the process exits. No cudaMalloc, cudaFree or
 * other allocating call is made.
 *   - Limits: N >= 1, d_in a multiple of 8 and at most 524288; larger d_in
 *     returns AWQ_ERR_SHAPE. Any N within those limits fits the array.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it with the
 *     id of the device's current context; make that first call before any
 *     stream capture. After the context is destroyed and rebuilt
 *     (cudaDeviceReset), the next call sees a new context id and looks the
 *     address up again (so that call, too, belongs before any capture).
 *   - All calls in the process share the one array: calls whose work overlaps
 *     on the GPU (different streams or threads) race and give wrong results.
 *     Calls ordered on one stream are safe; nothing needs clearing between
 *     them because every partial read is first written by the same call.
 * Other errors as awq_act_stats.
 * ------------------------------------------------------------------------- */
awq_status awq_act_stats_noalloc(const void* X_bf16, int64_t N, int64_t d_in, float* a, awq_stream_t stream);

/* ---------------------------------------------------------------------------
 * Steps a2-a6: the scale search.
 * For each alpha_k of the grid:
 *   s_i = max(a_i, eps_a)^alpha_k / sqrt(max_j s_j * min_j s_j)      ([P5] §4.1)
 *   dW  = Q(W S) S^-1 - W, group-wise along d_in                       ([P1] 缩放保护)
 *         symmetric: Delta = max|v| / (2^(b-1)-1), q = clamp(rne(v/Delta), -2^(b-1), 2^(b-1)-1)
 *         asymmetric: Delta = (max v - min v) / (2^b-1), z = clamp(rne(-min v/Delta), 0, 2^b-1),
 *                     q = clamp(rne(v/Delta) + z, 0, 2^b-1), v_hat = (q - z) Delta
 *   L_k = ||dW X^T||_F^2                                               ([P5] §1.1, §4.1)
 * then best = argmin_k L_k (lowest k on ties) and s_best = s(alpha_best).
 * The contraction runs on tcgen05 tensor cores with bf16 operands and fp32
 * accumulation, either directly (dW X^T) or through G = X^T X.
 * Outputs (device): losses float [n_alpha]; best int32 [1]; s_best float
 * [d_in]; row_losses float [n_alpha, d_out] (per-row losses) or NULL.
 * On non-finite losses the device sets best = -1, fills s_best with NaN and
 * records AWQ_ERR_NONFINITE in the workspace.
 * ws: scratch of awq_search_workspace_size(...) bytes (dominated by the
 * n_alpha x d_out x d_in bf16 stack of candidate dW).
 * ------------------------------------------------------------------------- */
size_t awq_search_workspace_size(int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg);
awq_status awq_search_scales(const void* W_bf16, const void* X_bf16, const float* a, int64_t d_out,
                             int64_t d_in, int64_t N, const awq_qcfg* cfg, void* ws, size_t ws_bytes,
                             float* losses, int32_t* best, float* s_best, float* row_losses,
                             awq_stream_t stream);

/* ---------------------------------------------------------------------------
 * The search for several linear layers that read the same activations X
 * (for example the q/k/v projections, or gate/up): W is their row
 * concatenation [d_out, d_in] with layer i holding seg_rows[i] consecutive
 * rows (HOST array, n_seg in 1..16, sum = d_out). The statistics, the Gram
 * product and one fake-quant and contraction launch serve all layers; each
 * layer gets its own losses and choice:
 *   losses float [n_seg, n_alpha], best int32 [n_seg], s_best float
 *   [n_seg, d_in], row_losses as in awq_search_scales (or NULL).
 * Layers whose scales are folded into one shared preceding operation need a
 * single shared choice: that is awq_search_scales on the same concatenated W
 * (its loss is the sum over the layers). Workspace: awq_search_workspace_size
 * with the total d_out. Errors as awq_search_scales, plus
 * AWQ_ERR_INVALID_ARG for n_seg out of range and AWQ_ERR_SHAPE when the
 * segment sizes do not sum to d_out.
 * ------------------------------------------------------------------------- */
awq_status awq_search_scales_segmented(const void* W_bf16, const void* X_bf16, const float* a, int64_t d_out,
                                       int64_t d_in, int64_t N, const awq_qcfg* cfg, int32_t n_seg,
                                       const int64_t* seg_rows, void* ws, size_t ws_bytes, float* losses,
                                       int32_t* best, float* s_best, float* row_losses, awq_stream_t stream);

/* The contraction form awq_search_scales will use for these sizes (1 direct,
 * 2 Gram): AUTO picks the one with fewer multiply-adds, n_alpha*d_out*d_in*N
 * versus (N + n_alpha*d_out) * T(d_in), where T(d_in) ~ d_in^2/2 counts the
 * lower block triangle of the symmetric G = X^T X (256-wide blocks) that the
 * Gram form evaluates: sum_{i,j} dW_i G_ij dW_j over j's block <= i's block,
 * off-diagonal blocks doubled. */
int32_t awq_search_form(int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg);

/* Read back (synchronising `stream`) the device error word of a search or
 * stats workspace and clear it: AWQ_OK, AWQ_ERR_NONFINITE or AWQ_ERR_DEVICE. */
awq_status awq_workspace_error(void* ws, awq_stream_t stream);

/* ---------------------------------------------------------------------------
 * Step a7: quantise at the chosen scales and pack.
 * codes of Q(W S) with the quantiser above ([P2] §2.1 INT4 clip and fp16
 * scale; [P4] §三 zero point), stored one per nibble, eight per uint32 word:
 *   qweight uint32 [d_out, d_in/8], code of channel 8w+j in bits 4j..4j+3;
 *   scales  fp16   [d_out, d_in/g] = Delta (rounded to nearest even);
 *   zeros   fp16   [d_out, d_in/g] = z (asymmetric) or 2^(b-1) (symmetric,
 *                                    whose codes are stored as q + 2^(b-1)).
 * s: float [d_in] (typically s_best).
 * ------------------------------------------------------------------------- */
awq_status awq_quantize_pack(const void* W_bf16, const float* s, int64_t d_out, int64_t d_in,
                             const awq_qcfg* cfg, uint32_t* qweight, void* scales_f16, void* zeros_f16,
                             awq_stream_t stream);

/* Pack with a clip ratio clip in (0, 1]: each group's range is shrunk by clip
 * before the step is taken (symmetric: c max|v|; asymmetric: c max v and
 * c min v) and values beyond it take the extreme codes. clip = 1 is
 * awq_quantize_pack. AWQ_ERR_INVALID_ARG for clip outside (0, 1]. */
awq_status awq_quantize_pack_clipped(const void* W_bf16, const float* s, int64_t d_out, int64_t d_in,
                                     const awq_qcfg* cfg, float clip, uint32_t* qweight, void* scales_f16,
                                     void* zeros_f16, awq_stream_t stream);

/* The clipped pack with a workspace (DEVICE, 256-byte aligned, at least
 * awq_pack_workspace_size bytes): any cfg->group, including 0 (per tensor:
 * the layer-wide max and min of W S are taken first, and scales / zeros are
 * [1] each). awq_quantize_pack* without a workspace return AWQ_ERR_WORKSPACE
 * for group 0. */
size_t awq_pack_workspace_size(int64_t d_out, int64_t d_in, const awq_qcfg* cfg);
awq_status awq_quantize_pack_ws(const void* W_bf16, const float* s, int64_t d_out, int64_t d_in,
                                const awq_qcfg* cfg, float clip, void* ws, size_t ws_bytes, uint32_t* qweight,
                                void* scales_f16, void* zeros_f16, awq_stream_t stream);

/* ---------------------------------------------------------------------------
 * The search over caller-given candidates instead of the a^alpha grid
 * ([P5] 参考资料: the practical algorithm searches a restricted
 * parameterisation of the scales, possibly combined with clipping).
 * Candidate k uses the scale vector s_cand[k] (DEVICE float [n, d_in], every
 * entry > 0) and the clip ratio clips[k] (HOST float [n] in (0, 1], or NULL
 * for no clipping), n = cfg->n_alpha (cfg->alphas is ignored). For example:
 * the clipping search is n copies of s_best with a grid of clip ratios; a
 * salience mask ([P1] 显著识别) is s_i = factor on the channels above a
 * percentile of a and 1 elsewhere. Outputs as in awq_search_scales, with
 * s_best = the chosen candidate's scales; a non-positive scale is recorded as
 * AWQ_ERR_NONFINITE. Workspace: awq_search_workspace_size.
 * ------------------------------------------------------------------------- */
awq_status awq_search_candidates(const void* W_bf16, const void* X_bf16, const float* s_cand, const float* clips,
                                 int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg, void* ws,
                                 size_t ws_bytes, float* losses, int32_t* best, float* s_best, float* row_losses,
                                 awq_stream_t stream);

/* ---------------------------------------------------------------------------
 * Per-group clipping search ([P5] 参考资料 note: the clipping search, read per
 * quantisation group). With the scales s fixed (DEVICE float [d_in], every
 * entry > 0, e.g. s_best of the scale search), clip candidate c (ratio
 * clips[c], HOST float [n] in (0, 1], n = cfg->n_alpha <= 64; cfg->alphas is
 * ignored) gives dW_c = Q(W S; clips[c]) S^-1 - W. For row r and group j
 * (columns j*g .. j*g+g-1) its error is the group's own output error
 *   err[c, r, j] = sum_t (sum_{i in j} dW_c[r, i] X[t, i])^2
 *               = dW_c[r, j] G_jj dW_c[r, j]^T,    G = X^T X,
 * i.e. the block-diagonal part of the layer error dW G dW^T. Computed as:
 * the diagonal 256-blocks of G on the tensor cores (masked to the groups),
 * every candidate's dW stack, one contraction of dW against those blocks with
 * per-32-column partials, then a float64 sum per group and the argmin.
 *   best_clip   DEVICE uint8 [d_out, d_in/g]: index of the smallest error,
 *               the lowest index on exact ties.
 *   group_err   DEVICE float [n, d_out, d_in/g] or NULL: the errors.
 * Requires g >= 32 (AWQ_ERR_UNSUPPORTED otherwise). Workspace:
 * awq_group_clip_workspace_size; non-finite errors or a non-positive scale
 * are recorded as AWQ_ERR_NONFINITE (awq_workspace_error). Asynchronous.
 * ------------------------------------------------------------------------- */
size_t awq_group_clip_workspace_size(int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg);
awq_status awq_search_group_clip(const void* W_bf16, const void* X_bf16, const float* s, const float* clips,
                                 int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg, void* ws,
                                 size_t ws_bytes, uint8_t* best_clip, float* group_err, awq_stream_t stream);

/* awq_quantize_pack with a clip ratio per (row, group): group j of row r uses
 * clips[best_clip[r * (d_in/g) + j]] (clips HOST float [n_clips] in (0, 1],
 * n_clips <= 64; best_clip DEVICE uint8 [d_out, d_in/g], entries < n_clips,
 * e.g. the output of awq_search_group_clip; an entry >= n_clips means no
 * clipping). Outputs as in awq_quantize_pack. AWQ_ERR_INVALID_ARG for a ratio
 * outside (0, 1], n_clips outside [1, 64] or a NULL table. */
awq_status awq_quantize_pack_group_clip(const void* W_bf16, const float* s, const float* clips, int32_t n_clips,
                                        const uint8_t* best_clip, int64_t d_out, int64_t d_in, const awq_qcfg* cfg,
                                        uint32_t* qweight, void* scales_f16, void* zeros_f16, awq_stream_t stream);

/* ---------------------------------------------------------------------------
 * Inference side: the quantised layer as it runs after calibration.
 * ------------------------------------------------------------------------- */
/* 16-bit floating-point types of the inference-side calls. */
typedef enum awq_dtype { AWQ_DTYPE_BF16 = 0, AWQ_DTYPE_F16 = 1 } awq_dtype;

/* Fold S^-1 into the operation that produces X ("AWQ" (scholia-log) §4.3: a
 * diagonal S^-1 is absorbed by the adjacent LayerNorm or Linear, so the
 * layer computes Q(W S)(S^-1 X) at no extra cost). p is that operation's bf16
 * parameter block with the channel on the first axis, DEVICE [d_in, inner]
 * row-major, bf16 or fp16 (dtype), updated in place: p[i, j] <- p[i, j] /
 * s[i], the quotient in fp32 (correctly rounded) and rounded to nearest even
 * in the same type. inner = 1 for a
 * norm's weight or bias, d_prev for the previous linear layer's weight
 * [d_in, d_prev]. s is DEVICE float [d_in]; a non-positive or non-finite s_i
 * gives the IEEE quotient (no check). Asynchronous. */
awq_status awq_fold_inv_scales(const float* s, int64_t d_in, void* p, awq_dtype dtype, int64_t inner,
                               awq_stream_t stream);

/* W4A16 product reading the packed format ("AWQ量化技术解析" (kwkr.cn) §1.2,
 * §4.2: weights dequantised on the fly as W_int4 x scale_fp16, fused with the
 * GEMM; ewbang.com AWQ 二.3: dequantised to FP16 for the product):
 *   Y[t, o] = sum_i X'[t, i] * (code[o, i] - z[o, i/g]) * Delta[o, i/g]
 * X'      DEVICE [N, d_in] row-major, fp16 or bf16 (dtype), 16-byte aligned:
 *         activations that already carry S^-1 (awq_fold_inv_scales on their
 *         producer).
 * qweight, scales, zeros: the output of awq_quantize_pack* for this layer
 *         (DEVICE uint32 [d_out, d_in/8], fp16 [d_out, d_in/g] twice);
 *         cfg->bits and cfg->group describe them (cfg->n_alpha, form, eps_a
 *         and alphas are ignored; symmetric codes carry their zero point).
 * Y       DEVICE [N, d_out] row-major in the same type, 16-byte aligned.
 * The dequantised weights enter the tensor cores in that type: fp16 rounds
 * (code - z) * Delta once; bf16 rounds Delta to bf16 and then the product.
 * Accumulation is fp32; Y is rounded once. Requires d_in a multiple of 32
 * and of g (AWQ_ERR_SHAPE). cfg->group must be a group size (8 ... 256): the
 * per-tensor layout (group 0, one step for the layer) is not read by this
 * kernel and gives AWQ_ERR_INVALID_ARG.
 * Workspace: awq_w4a16_workspace_size (error word, and fp32 partials of the
 * tiles that are split between CTAs when there are fewer than two waves of
 * output tiles); AWQ_ERR_WORKSPACE if smaller.
 * Asynchronous; device-side errors land in the workspace (awq_workspace_error). */
size_t awq_w4a16_workspace_size(int64_t N, int64_t d_out, int64_t d_in, const awq_qcfg* cfg);
awq_status awq_w4a16_gemm(const void* X, awq_dtype dtype, const uint32_t* qweight, const void* scales_f16,
                          const void* zeros_f16, int64_t N, int64_t d_out, int64_t d_in, const awq_qcfg* cfg,
                          void* Y, void* ws, size_t ws_bytes, awq_stream_t stream);

/* ---------------------------------------------------------------------------
 * The search, one step at a time (awq_search_scales is exactly these calls
 * in this order). They share the search workspace; offsets are internal.
 * ------------------------------------------------------------------------- */
/* a2: candidate scales s and 1/s of every alpha into the workspace. */
awq_status awq_step_scales(const float* a, int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg,
                           void* ws, size_t ws_bytes, awq_stream_t stream);
/* a3: the bf16 stack dW[k] = Q(W S_k) S_k^-1 - W for every alpha into the
 * workspace (rows padded to a multiple of 128 with zeros). */
awq_status awq_step_fake_quant(const void* W_bf16, int64_t d_out, int64_t d_in, int64_t N,
                               const awq_qcfg* cfg, void* ws, size_t ws_bytes, awq_stream_t stream);
/* a4 (Gram form only): the lower block triangle of G = X^T X (bf16, strictly
 * lower 256-blocks doubled) into the workspace. */
awq_status awq_step_gram(const void* X_bf16, int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg,
                         void* ws, size_t ws_bytes, awq_stream_t stream);
/* a5: the tensor-core contraction with the fused squared-sum epilogue, per
 * (row, column-tile) partials into the workspace. X_bf16 is read by the
 * direct form only. */
awq_status awq_step_contract(const void* X_bf16, int64_t d_out, int64_t d_in, int64_t N,
                             const awq_qcfg* cfg, void* ws, size_t ws_bytes, awq_stream_t stream);
/* a6: fixed-order float64 reduction, argmin, s_best (outputs as in
 * awq_search_scales). */
awq_status awq_step_reduce(int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg, void* ws,
                           size_t ws_bytes, float* losses, int32_t* best, float* s_best, float* row_losses,
                           awq_stream_t stream);

/* Copy of the candidate dW stack for inspection: dW for grid index k, rows
 * [0, d_out), as bf16 [d_out, d_in] into dst (device). */
awq_status awq_debug_copy_dw(const void* ws, int64_t d_out, int64_t d_in, int64_t N, const awq_qcfg* cfg,
                             int32_t k, void* dst_bf16, awq_stream_t stream);

/* Failure path of the bounded waits, for tests: one block waits on an
 * mbarrier that nothing arrives at, through the wait every GEMM of this
 * library uses; after the wall-clock limit (2 s) the wait gives up, sets the
 * workspace error word and the kernel returns, so that awq_workspace_error
 * then reports AWQ_ERR_DEVICE and the context stays usable. ws: DEVICE,
 * 256-byte aligned, at least 256 bytes. Asynchronous. */
awq_status awq_selftest_bounded_wait(void* ws, awq_stream_t stream);

/* Debug build (compiled with -DAWQ_BOUNDS_CHECK). Every global load and store
 * that a kernel addresses by hand (everything but the TMA tensor-map copies)
 * first checks the span it touches against the extent the kernel's arguments
 * give that buffer; a failed check skips the access (a load reads zero) and
 * records the site in a device word of the library, the first failure kept.
 * The GEMM launchers also check on the host that the furthest element their
 * epilogue may store or read lies inside the buffer, and return
 * AWQ_ERR_BOUNDS without launching if not. In the release build the checks
 * compile to nothing. */

/* 1 if this library was built with the index checks, else 0. */
int32_t awq_bounds_checks_enabled(void);

/* Read back (synchronising `stream`) and clear the device word of the index
 * checks: AWQ_OK if no check failed since the last call, else AWQ_ERR_BOUNDS
 * with *site (host, may be NULL) set to the failing access's site code (the
 * low byte of the word; 0x7F: awq_selftest_bounds). Always AWQ_OK in the
 * release build. */
awq_status awq_bounds_error(int32_t* site, awq_stream_t stream);

/* Failure path of the index checks, for tests: one thread stores to element n
 * of an int buffer whose extent it declares as n; the check refuses the store
 * and records site 0x7F. The buffer is ws, which holds n + 1 ints, so even the
 * refused store would have stayed inside it. ws: DEVICE, 256-byte aligned, at
 * least 256 bytes. Asynchronous. Returns AWQ_ERR_UNSUPPORTED (and launches
 * nothing) in the release build. */
awq_status awq_selftest_bounds(void* ws, size_t ws_bytes, awq_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* AWQ_B200_H */
