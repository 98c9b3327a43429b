/*
 * gptq.h — C ABI of the B200 (sm_100a) GPTQ layer-wise weight quantization library
 * (libgptq_b200.so).
 *
 * The method (GPTQ; group min-max RTN as its baseline) as the source pages state it:
 *   - "大模型量化技术原理：GPTQ、AWQ、GGUF核心机制与部署选型指南" (0539edu.com/news/6111416):
 *     §2.1 the affine quantizer q = round(x/scale) + zero_point and its min-max scale,
 *     §3.1 the layer objective ||WX - W_qX||^2 and the quantize config (bits, group_size,
 *     desc_act), §4.2 one fp16 scale and one fp16 zero point per group.
 *   - GPTQ deep-dive (hncyxsy.com/news/243429): §2.2 OBS compensation with the inverse
 *     Hessian, §2.4 fixed order + lazy batch updates + Cholesky, §3.1 the four per-layer steps
 *     (H = 2XX^T + lambda*I; Cholesky; per 128-column block: scale, round, accumulate the
 *     error, then update the later columns; store codes, scales, zeros), §3.3 group_size,
 *     desc_act, damp_percent.
 *   - "AWQ、MinMax、GPTQ 三大校准算法原理与选型指南" (gtnt.cn/news/115337) §4: Hessian collection,
 *     block_size 128 a multiple of group_size, perc_damp 0.01.
 *   - Calibration-methods page (bhfrc.com/news/5741) §2.2 group min-max, §2.3 GPTQ order by
 *     descending Hessian diagonal.
 *
 * Conventions for every call
 *   - Matrices are dense and row-major. W is [d_out x d_in] (PyTorch Linear layout); X is
 *     [n_tokens x d_in]; H is [d_in x d_in].
 *   - Pointers marked "device" are CUDA device memory of the current device; the caller owns
 *     them. No call allocates device memory except gptq_hessian_create.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Work is
 *     ordered on it. Calls are not thread-safe on the same handle or workspace.
 *   - gptq_quantize_layer and gptq_inverse_factor also run part of the factorisation (and
 *     gptq_quantize_layer part of its far lazy updates) on a second stream that the library
 *     owns (one per device). It is forked from `stream` and joined back to it by events inside
 *     the call, so the call stays ordered on `stream`.
 *   - One process drives one GPU. The library sets its kernels' shared-memory limits once per
 *     process, on the device current at the first call; a process that switches devices
 *     between calls is not supported (launches on the second device fail with CUDA).
 *   - Argument errors are detected on the host before any launch and return GPTQ_ERR_ARG.
 *   - fp16 values are passed as their 16-bit patterns (uint16_t).
 *   - The library runs only on sm_100 devices; elsewhere calls return GPTQ_ERR_UNSUPPORTED.
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gptq_status {
    GPTQ_OK = 0,
    GPTQ_ERR_ARG = -1,          /* invalid argument; nothing was launched */
    GPTQ_ERR_NOT_PD = -2,       /* damped Hessian not positive definite (a Cholesky pivot <= 0,
                                   or lambda = percdamp*mean(diag H) <= 0) */
    GPTQ_ERR_NONFINITE = -3,    /* NaN or Inf found in H or W */
    GPTQ_ERR_CUDA = -4,         /* a CUDA runtime/driver call failed */
    GPTQ_ERR_OOM = -5,          /* gptq_hessian_create could not allocate */
    GPTQ_ERR_TIMEOUT = -6,      /* a bounded device-side wait gave up (kernel returned early) */
    GPTQ_ERR_WORKSPACE = -7,    /* workspace smaller than gptq_quantize_layer_workspace() */
    GPTQ_ERR_UNSUPPORTED = -8   /* current device is not compute capability 10.0 */
} gptq_status;

enum { GPTQ_DTYPE_F16 = 0, GPTQ_DTYPE_F32 = 1 };

/* Human-readable name of a status code (static string). */
const char* gptq_status_string(int status);

/* ------------------------------------------------------------------------------------------
 * Stage 1: calibration Hessian H = 2 * X^T X  (GPTQ deep-dive §3.1 step 1; gtnt.cn §4).
 * Accumulated over any number of calls (H grows by 2*X^T X each call; no 1/n normalisation:
 * GPTQ's result does not change when H is scaled). Runs on the tensor cores (tcgen05, fp16
 * inputs, fp32 accumulation). Only the upper triangle (j >= i) of the stored H is maintained.
 * ------------------------------------------------------------------------------------------ */
typedef struct gptq_hessian gptq_hessian;

/* Allocate a handle owning a zeroed fp32 [d_in x d_in] H on the current device.
 * d_in: 8 <= d_in <= 65536, multiple of 8. *out receives the handle. Errors: ARG, OOM, CUDA,
 * UNSUPPORTED. */
gptq_status gptq_hessian_create(int d_in, gptq_hessian** out);

/* H += 2 * X^T X.  X: device, fp16 [n_tokens x d_in] row-major, 16-byte aligned; n_tokens >= 0
 * (0 is a no-op). Asynchronous on `stream`; X must stay valid until the work completes.
 * Errors: ARG (null/misaligned X, n_tokens < 0), CUDA. */
gptq_status gptq_hessian_accumulate(gptq_hessian* h, const void* X, int64_t n_tokens,
                                    void* stream);

/* Write the full symmetric H (upper triangle mirrored) into H_out: device fp32
 * [d_in x d_in]. Synchronises `stream` to report a device-side TIMEOUT from earlier
 * accumulations. Errors: ARG, CUDA, TIMEOUT. */
gptq_status gptq_hessian_get(const gptq_hessian* h, float* H_out, void* stream);

/* Device pointer to the handle's H storage (upper triangle valid; lower triangle
 * unspecified), usable directly as the H argument of gptq_quantize_layer. */
const float* gptq_hessian_data(const gptq_hessian* h);

/* Tokens accumulated so far; d_in of the handle. */
int64_t gptq_hessian_tokens(const gptq_hessian* h);
int gptq_hessian_dim(const gptq_hessian* h);

/* Reset H to zero (asynchronous on `stream`). */
gptq_status gptq_hessian_reset(gptq_hessian* h, void* stream);

/* Free the handle and its H. Safe on NULL. */
gptq_status gptq_hessian_destroy(gptq_hessian* h);

/* Handle-free form: H (device fp32 [d_in x d_in], caller-owned, 16-byte aligned, row stride
 * d_in) += 2 * X^T X on its upper triangle (tiles that straddle the diagonal also update some
 * entries below it). The tensor cores accumulate at most 512 tokens at a time; those partial
 * sums are added in fp32 with round-to-nearest, and each work unit adds its sum into H with
 * atomic fp32 adds (so the low bits of H depend on the order units finish). `unit_tokens`
 * sets the tokens per work unit (0 = chosen to balance the SMs; otherwise a multiple of 64).
 * status_dev: device int, or NULL; set to GPTQ_ERR_TIMEOUT if a bounded wait gave up. */
gptq_status gptq_hessian_accumulate_into(float* H, int d_in, const void* X, int64_t n_tokens,
                                         int unit_tokens, int* status_dev, void* stream);

/* ------------------------------------------------------------------------------------------
 * Stages 2-4: GPTQ quantization of one linear layer (GPTQ deep-dive §2.2, §2.4, §3.1, §3.3;
 * gtnt.cn §4).
 *   lambda = percdamp * mean(diag H);  H_d = H + lambda*I
 *   processing order: identity, or (act_order != 0) diag(H) descending, ties by lower index
 *   U upper triangular with U^T U = H_d^-1 (fp32 blocked Cholesky + triangular inverse)
 *   for each block of `block_size` columns: for each column q (in order):
 *       at a group's first column: per row, scale/zero from min/max of the group's current
 *       (compensated) weights: scale = (max-min)/(2^bits-1) rounded up to fp16, zero =
 *       rint(-min/scale);  code = clamp(rint(w/scale) + zero, 0, 2^bits-1);
 *       e = (w - scale*(code-zero)) / U[q][q];  later columns of the block -= e * U[q][.]
 *   after the block: all later columns -= Err_block * U[block rows][later columns]
 *
 * Arguments
 *   W        device, [d_out x d_in], fp16 (w_dtype = GPTQ_DTYPE_F16) or fp32; not modified.
 *   d_out    >= 1.   d_in: >= 8, multiple of 8 and of group_size, <= 65536.
 *   H        device fp32 [d_in x d_in]; only the upper triangle (j >= i) is read; not modified.
 *   bits     2..8.  group_size: >= 1, divides d_in and block_size.
 *   block_size  8..128, a multiple of 8 and of group_size (gtnt.cn §4: block_size is a
 *            multiple of group_size); the last block may be narrower.
 *   percdamp >= 0; lambda <= 0 (percdamp 0, or an all-zero diagonal) gives GPTQ_ERR_NOT_PD.
 *   act_order 0 or 1.
 *   codes    device uint8 [d_out x d_in], codes in ORIGINAL column order, in [0, 2^bits-1].
 *   scales, zeros  device fp16 [d_out x d_in/group_size], indexed by processing-order group.
 *   g_idx    device int32 [d_in]: processing-order group of each original column.
 *   perm     device int32 [d_in] or NULL: perm[p] = original column processed at position p.
 *   loss     host float or NULL: if given, tr(D H D^T)/tr(W H W^T) with D = W - What and the
 *            undamped H (the layer's relative output error ||(W - What) X^T||^2/||W X^T||^2).
 *   workspace device, >= gptq_quantize_layer_workspace(d_out, d_in, block_size) bytes,
 *            256-byte aligned; contents are scratch.
 * The call synchronises `stream` once at its end to read the device status word.
 * Errors: ARG, WORKSPACE, NOT_PD, NONFINITE, CUDA, UNSUPPORTED. On NOT_PD/NONFINITE the outputs
 * are unspecified.
 * ------------------------------------------------------------------------------------------ */
size_t gptq_quantize_layer_workspace(int d_out, int d_in, int block_size);

gptq_status gptq_quantize_layer(const void* W, int w_dtype, int d_out, int d_in,
                                const float* H, int bits, int group_size, int block_size,
                                float percdamp, int act_order,
                                uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                                int32_t* g_idx, int32_t* perm, float* loss,
                                void* workspace, size_t workspace_bytes, void* stream);

/* gptq_quantize_layer with the quantizer variants (same arguments, plus two switches, same
 * workspace size). gptq_quantize_layer is this call with sym = 0 and static_groups = 0.
 *   sym            1: the symmetric quantizer of 0539edu.com §2.3 (zero point fixed at 0,
 *                  q = round(x/scale)): scale = 2*max|w|/(2^bits-1) rounded up to fp16 over the
 *                  group, and the signed zero stored as the code offset 2^(bits-1), so
 *                  code = clamp(rint(w/scale) + 2^(bits-1), 0, 2^bits-1) and zeros hold
 *                  2^(bits-1).
 *   static_groups  1: every group's scale and zero are fixed from the ORIGINAL weights, groups
 *                  of group_size consecutive original columns, before any column is quantized;
 *                  each column uses the group of its original position, whatever order
 *                  act_order processes it in: g_idx[c] = c / group_size and scales/zeros are
 *                  indexed by that group (the inference-time gather of GPTQ deep-dive §3.3
 *                  then reads contiguous groups).
 *   group_size == d_in  one group per row (per-channel): its scale and zero come from the
 *                  whole original row before its first column is quantized; block_size is then
 *                  free (any multiple of 8 up to 128).
 * Errors: as gptq_quantize_layer; ARG also for sym or static_groups outside {0, 1}. */
gptq_status gptq_quantize_layer_ex(const void* W, int w_dtype, int d_out, int d_in,
                                   const float* H, int bits, int group_size, int block_size,
                                   float percdamp, int act_order, int sym, int static_groups,
                                   uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                                   int32_t* g_idx, int32_t* perm, float* loss,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* No-allocation form of gptq_quantize_layer, with the same arguments except the workspace.
 * The pages have no counterpart; this is an integration aid. It is for callers that may not
 * allocate device memory when they quantize: runtimes that reserved almost all of the GPU for
 * their own pools at start-up, and deployments that forbid device allocation after
 * initialisation. Such callers cannot supply a workspace either. The scratch is a fixed
 * 32 MiB device array inside the library, held until the process exits. It takes device
 * memory when the library's device code is loaded onto a GPU; under CUDA's lazy module loading
 * (the default) that happens at this entry point's first call on each device, so a caller
 * that reserves its memory pools at start-up should make one call before reserving them.
 *   - Layers whose gptq_quantize_layer_workspace(d_out, d_in, block_size) exceeds 32 MiB are
 *     rejected with GPTQ_ERR_WORKSPACE before anything is launched. For example, d_in = 1024
 *     fits up to d_out = 1653 and d_in = 512 up to d_out = 2779; d_in = 4096 does not fit.
 *   - No cudaMalloc, cudaFree or other allocating call is made.
 *   - The first call on each device looks up the array's device address (cudaGetSymbolAddress
 *     with that device current). Make that first call before any stream capture on the device.
 *   - All calls share the one array, and it keeps the previous call's contents. The status
 *     block at its head is cleared by every call, and everything else is written before it is
 *     read. Calls that overlap on the GPU (concurrent streams, or several host threads) race on
 *     the array and must be serialised by the caller.
 * Synchronises `stream` once at its end, like gptq_quantize_layer. Errors: as
 * gptq_quantize_layer, plus WORKSPACE for layers that do not fit. */
gptq_status gptq_quantize_layer_noalloc(const void* W, int w_dtype, int d_out, int d_in,
                                        const float* H, int bits, int group_size, int block_size,
                                        float percdamp, int act_order,
                                        uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                                        int32_t* g_idx, int32_t* perm, float* loss,
                                        void* stream);

/* Stage 2 on its own: the processing order and U (upper triangular, zero below the diagonal,
 * U^T U = (P H P + lambda*I)^-1 in the processing order P) that gptq_quantize_layer uses.
 *   H        device fp32 [d_in x d_in], upper triangle read.  d_in: >= 8, multiple of 8.
 *   U        device fp32 [d_in x d_in] (written).   perm: device int32 [d_in] or NULL.
 *   workspace >= gptq_inverse_factor_workspace(d_in) bytes, 256-byte aligned.
 * Synchronises `stream` once. Errors: ARG, WORKSPACE, NOT_PD, NONFINITE, CUDA, UNSUPPORTED. */
size_t gptq_inverse_factor_workspace(int d_in);
gptq_status gptq_inverse_factor(const float* H, int d_in, float percdamp, int act_order,
                                float* U, int32_t* perm, void* workspace,
                                size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------------
 * Baseline: group min-max round-to-nearest (bhfrc.com §2.2; 0539edu.com §2.1, §4.2; GPTQ
 * deep-dive §1.2). The quantizer above applied to the original W with no compensation.
 *   W       device [d_out x d_in], fp16 or fp32, 16-byte aligned.
 *   d_in    multiple of group_size and of 8.  group_size >= 1 (fast path: 8..256, power of 2).
 *   packed  device uint8: bits == 4 -> [d_out x d_in/2], two codes per byte, even column in
 *           the low nibble; otherwise [d_out x d_in], one code per byte.
 *   scales, zeros  device fp16 [d_out x d_in/group_size].
 * Asynchronous; bit-exact with the fp64 definition (scale/zero computed in fp64, the rounding
 * decision made exactly). Errors: ARG, CUDA, UNSUPPORTED.
 * ------------------------------------------------------------------------------------------ */
gptq_status rtn_minmax_quantize(const void* W, int w_dtype, int d_out, int d_in, int bits,
                                int group_size, uint8_t* packed, uint16_t* scales,
                                uint16_t* zeros, void* stream);

/* Group RTN with a clip search per group (gtnt.cn §3, awq_clip: each quantization block's clip
 * bound c is searched in [amax * min_ratio, amax], amax = max |w| of the block, truncating the
 * weights to [-c, c] before their min-max scale is taken).
 *   For ratios rho_i = 1 - i*step, i = 0 .. round((1 - min_ratio)/step) (the pages' defaults
 *   min_ratio = 0.5, step = 0.05: 11 ratios), c = rho_i * amax; the group's weights are clamped
 *   to [-c, c] and quantized with the scale and zero of the clamped group (sym selects the
 *   symmetric quantizer). The criterion is the group's share of the layer output error,
 *   d * H_gg * d with d = w - What (original weights minus the reconstruction) and H_gg the
 *   group's diagonal block of H = 2 X^T X; with H = NULL it is the weight error d.d. The smallest
 *   criterion wins, ties to the larger ratio. For the chosen ratio the codes, scales and zeros
 *   equal the fp64 definition bit for bit; the criterion is accumulated in fp32.
 *   W        device [d_out x d_in], fp16 or fp32.  d_in: a multiple of group_size.
 *   group_size  16, 32, 64 or 128.
 *   H        device fp32 [d_in x d_in], upper triangle read, 16-byte aligned; or NULL.
 *   min_ratio in (0, 1], step > 0, at most 64 grid points.
 *   packed, scales, zeros  as rtn_minmax_quantize.
 *   ratio_idx device uint8 [d_out x d_in/group_size] (index i of the chosen ratio), or NULL.
 * Asynchronous. Errors: ARG, CUDA, UNSUPPORTED. */
gptq_status rtn_clip_search(const void* W, int w_dtype, int d_out, int d_in, int bits,
                            int group_size, int sym, const float* H, double min_ratio,
                            double step, uint8_t* packed, uint16_t* scales, uint16_t* zeros,
                            uint8_t* ratio_idx, void* stream);

/* Group RTN of clipped weights (bhfrc.com §4.3: instead of the extreme values, take a
 * percentile of the values, such as 99.99 %, or a fixed absolute range, such as [-10, 10], and
 * truncate what lies outside before the min-max range is formed).
 *   Per group: hi = the p-quantile and lo = the (1 - p)-quantile of its weights,
 *   p = percentile / 100; a q-quantile is v[k] + t * (v[k+1] - v[k]) with v the group sorted
 *   ascending, h = q * (group_size - 1), k = floor(h), t = h - k (v[group_size-1] when k is the
 *   last position), every operation rounded on its own in fp64. With abs_range > 0, lo and hi
 *   are further limited to [-abs_range, abs_range]. The weights are clamped to [lo, hi] and
 *   quantized with the quantizer of the range [lo, hi] (asymmetric: widened to contain 0;
 *   symmetric with sym = 1: m = max(|lo|, |hi|)). percentile = 100 and abs_range = 0 give
 *   rtn_quantize_ex. Codes, scales and zeros equal that fp64 definition bit for bit.
 *   W        device [d_out x d_in], fp16 or fp32, finite.  d_in: a multiple of group_size.
 *   group_size  16, 32, 64 or 128.   percentile in [50, 100].   abs_range >= 0 (0: none).
 *   packed, scales, zeros  as rtn_minmax_quantize.
 * Asynchronous. Errors: ARG, CUDA, UNSUPPORTED. */
gptq_status rtn_range_clip(const void* W, int w_dtype, int d_out, int d_in, int bits,
                           int group_size, int sym, double percentile, double abs_range,
                           uint8_t* packed, uint16_t* scales, uint16_t* zeros, void* stream);

/* rtn_minmax_quantize with the symmetric quantizer as an option (sym = 1: zero point fixed,
 * see gptq_quantize_layer_ex; sym = 0 is rtn_minmax_quantize). Same layouts and errors. */
gptq_status rtn_quantize_ex(const void* W, int w_dtype, int d_out, int d_in, int bits,
                            int group_size, int sym, uint8_t* packed, uint16_t* scales,
                            uint16_t* zeros, void* stream);

/* ------------------------------------------------------------------------------------------
 * The W4A16 layer that serves the quantized weights (0539edu.com §3.2, §5.2: 4-bit weights,
 * fp16 activations; GPTQ deep-dive §3.3: with desc_act the groups of the columns are scattered
 * and inference gathers them):
 *   Y = fp16(X * What^T + R),  What[r][c] = fp16(scale[r][k] * (code[r][c] - zero[r][k])),
 * fp32 accumulation on the tensor cores (tcgen05 kind::f16), k the group of column c.
 * The act_order gather is done on both sides of the contraction: w4a16_pack stores the codes in
 * the processing order of `perm` (so every group is again a run of group_size consecutive
 * columns, as the scales of gptq_quantize_layer are indexed), and w4a16_linear with the same
 * perm gathers the columns of X into the workspace before the GEMM. Without act_order (or with
 * static groups, whose g_idx is c / group_size) pass perm = NULL to both.
 * ------------------------------------------------------------------------------------------ */

/* packed[r][p/2] = codes[r][perm[p]] (codes[r][p] if perm is NULL), even p in the low nibble.
 *   codes   device uint8 [d_out x d_in] (gptq_quantize_layer's output, original order).
 *   perm    device int32 [d_in] or NULL.   packed: device uint8 [d_out x d_in/2].
 * Asynchronous. Errors: ARG (d_in odd), CUDA, UNSUPPORTED. */
gptq_status w4a16_pack(const uint8_t* codes, int d_out, int d_in, const int32_t* perm,
                       uint8_t* packed, void* stream);

/* Workspace bytes of w4a16_linear: n_tokens * d_in * 2 with a perm (the gathered X), else 0. */
size_t w4a16_linear_workspace(int64_t n_tokens, int d_in, int has_perm);

/* Y = fp16(X * What^T + R).
 *   X        device fp16 [n_tokens x d_in], 16-byte aligned; 1 <= n_tokens < 2^31.
 *   d_in     a multiple of 64, <= 65536.   d_out: a multiple of 8.
 *   packed   device uint8 [d_out x d_in/2] from w4a16_pack (same perm), 16-byte aligned.
 *   scales, zeros  device fp16 [d_out x d_in/group_size]: group p / group_size of processing
 *            position p.   group_size: a multiple of 8 dividing d_in.
 *   perm     device int32 [d_in] or NULL (see w4a16_pack).
 *   R        device fp16 [n_tokens x d_out] or NULL (a residual added before the rounding; may
 *            be the same buffer as Y).
 *   Y        device fp16 [n_tokens x d_out], 16-byte aligned.
 *   workspace device, >= w4a16_linear_workspace(n_tokens, d_in, perm != NULL) bytes (may be
 *            NULL without perm).
 *   status_dev device int or NULL: set to GPTQ_ERR_TIMEOUT if a bounded wait gave up.
 * Asynchronous. Errors: ARG, WORKSPACE, CUDA, UNSUPPORTED. */
gptq_status w4a16_linear(const void* X, int64_t n_tokens, int d_in, const uint8_t* packed,
                         const uint16_t* scales, const uint16_t* zeros, int group_size,
                         int d_out, const int32_t* perm, const void* R, void* Y,
                         void* workspace, size_t workspace_bytes, int* status_dev,
                         void* stream);

/* ------------------------------------------------------------------------------------------
 * AWQ-lite (gtnt.cn §3, awq_lite; 0539edu.com §3.2): per-input-channel scales
 * s = x_mean^alpha / w_mean^(1-alpha) searched over alpha = 0, step, ..., 1 by the layer's
 * output error, with group min-max RTN as the quantizer. The weights of channel c are
 * multiplied by s_c before quantization and its activations are to be divided by s_c (folded
 * into the preceding layer), which leaves the layer's output unchanged before quantization.
 * ------------------------------------------------------------------------------------------ */

/* sums[c] += sum over rows of |X[r][c]| in fp64 (accumulates over calibration batches; zero
 * sums first). X device fp16 or fp32 [n x d] row-major; sums device fp64 [d].
 * Asynchronous. Errors: ARG, CUDA, UNSUPPORTED. */
gptq_status gptq_channel_abs_sum(const void* X, int w_dtype, int64_t n, int d, double* sums,
                                 void* stream);

/* Workspace bytes of awq_lite_search (0 for invalid arguments). */
size_t awq_lite_workspace(int d_out, int d_in, double alpha_step);

/* The grid search, for fp16 W [d_out x d_in] (so that W * s is exact):
 *   x_mean_c = x_abs_sum[c] / n_tokens (x_abs_sum from gptq_channel_abs_sum, device fp64 [d_in]);
 *   w_mean_c = mean over rows of |W[r][c]|;
 *   for alpha_i = i * alpha_step, i = 0 .. round(1/alpha_step):
 *     s_c = fp16(x_mean_c^alpha / w_mean_c^(1-alpha)), 1 where x_mean_c or w_mean_c is 0 or the
 *     fp16 value is not positive and finite;
 *     L_i = tr(D H D^T), D = W - RTN(W * s) / s (RTN: group min-max, sym as in rtn_quantize_ex);
 *   best = argmin L_i (ties to the smaller alpha).
 *   H        device fp32 [d_in x d_in], FULL symmetric (as gptq_hessian_get writes it), H = 2X^T X.
 *   packed, scales, zeros  the RTN of W * s_best (layouts of rtn_minmax_quantize).
 *   s_out    device fp16 [d_in] (s_best) or NULL.
 *   losses   host double [round(1/alpha_step) + 1] or NULL (L_i, fp32-accurate).
 *   best     host int or NULL.
 *   workspace device, >= awq_lite_workspace(d_out, d_in, alpha_step) bytes, 256-byte aligned.
 * Synchronises `stream` once to choose alpha. Errors: ARG (also fp32 W), WORKSPACE, CUDA,
 * TIMEOUT, UNSUPPORTED. */
gptq_status awq_lite_search(const void* W, int w_dtype, int d_out, int d_in,
                            const double* x_abs_sum, int64_t n_tokens, const float* H, int bits,
                            int group_size, int sym, double alpha_step, uint8_t* packed,
                            uint16_t* scales, uint16_t* zeros, uint16_t* s_out,
                            double* losses, int* best, void* workspace, size_t workspace_bytes,
                            void* stream);

/* The unit-weight RMS pre-norm of a block (the input of its gate/up projections):
 * Y[t] = fp16(X[t] / sqrt(mean(X[t]^2) + eps)), fp32 sum of squares.
 *   X, Y device fp16 [n_tokens x d], 16-byte aligned (may not overlap); d a multiple of 8.
 * Asynchronous. Errors: ARG, CUDA, UNSUPPORTED. */
gptq_status gptq_rms_norm(const void* X, int64_t n_tokens, int d, float eps, void* Y,
                          void* stream);

/* The gate of a gated MLP block between its two quantized projections (layer-by-layer GPTQ
 * of a block stack, gtnt.cn §4: the down projection's Hessian comes from these activations):
 * A[t][j] = fp16(silu(GU[t][j]) * GU[t][d_ff + j]), silu(g) = g / (1 + e^-g) in fp32.
 *   GU  device fp16 [n_tokens x 2*d_ff] (gate outputs, then up outputs, per row).
 *   A   device fp16 [n_tokens x d_ff].   d_ff: a multiple of 8; both 16-byte aligned.
 * Asynchronous. Errors: ARG, CUDA, UNSUPPORTED. */
gptq_status gptq_silu_mul(const void* GU, int64_t n_tokens, int d_ff, void* A, void* stream);

/* ------------------------------------------------------------------------------------------
 * Stage timing. When enabled, gptq_quantize_layer records CUDA events around each stage on
 * its stream and gptq_profile_read returns the milliseconds of the last call per stage:
 *   0 prepare (diag statistics, act_order sort, gather + damping of H, gather of W)
 *   1 Cholesky   2 triangular inverse (U)   3 column loop (all blocks)
 *   4 lazy batch updates (all blocks)   5 output assembly   6 reconstruction loss
 * Returns the number of stages written (<= max_stages).
 * ------------------------------------------------------------------------------------------ */
void gptq_profile_enable(int on);
int gptq_profile_read(float* ms_out, int max_stages);

/* Total number of kernels this library has launched in the process (all entry points). */
unsigned long long gptq_launch_count(void);

/* ------------------------------------------------------------------------------------------
 * Test hook for the bounded-wait path (no counterpart on the pages). Every device-side wait of
 * the library gives up after a cycle limit and makes the call return GPTQ_ERR_TIMEOUT instead
 * of hanging. With on != 0, the factorisation's diagonal-block kernel first waits on an
 * mbarrier that nothing arrives at, with a limit of about 1 ms, so the next
 * gptq_quantize_layer / gptq_inverse_factor on the current device returns GPTQ_ERR_TIMEOUT;
 * the kernels after it skip their work on the status word and the CUDA context stays usable.
 * on = 0 restores normal operation. The switch is process-wide (every device) and is read when
 * a factorisation is enqueued; it is for tests only. Errors: CUDA, UNSUPPORTED (no usable
 * device).
 * ------------------------------------------------------------------------------------------ */
gptq_status gptq_test_stall_factor(int on);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_H */
