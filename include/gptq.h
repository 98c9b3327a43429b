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
 *   - gptq_quantize_layer and gptq_inverse_factor also run part of the factorisation on a
 *     second stream that the library owns (one per device). It is forked from `stream` and
 *     joined back to it by events inside the call, so the call stays ordered on `stream`.
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
 *     fits up to d_out = 2615 and d_in = 512 up to d_out = 4646; d_in = 4096 does not fit.
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
 * on = 0 restores normal operation. The switch is per device (current device) and process-wide;
 * it is for tests only. Errors: CUDA, UNSUPPORTED.
 * ------------------------------------------------------------------------------------------ */
gptq_status gptq_test_stall_factor(int on);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_H */
