// AWQ-lite: activation-aware per-channel scales with a grid search over alpha
// (gtnt.cn/news/115337 §3, awq_lite; 0539edu.com/news/6111416 §3.2).
//
//   x_mean_c = mean over tokens of |x_tc|      (gptq_channel_abs_sum, accumulated in fp64)
//   w_mean_c = mean over rows of |w_rc|
//   for alpha_i = i * alpha_step, i = 0 .. round(1/alpha_step):
//       s_c   = fp16(x_mean_c^alpha / w_mean_c^(1-alpha))   (1 where degenerate)
//       Q     = group min-max RTN of W * s (exact products: fp16 weight x fp16 scale)
//       D     = W - Q / s                                    (fp32)
//       L_i   = tr(D H D^T)                                  (3xTF32 tcgen05 GEMM, dot epilogue)
//   best = argmin L_i (ties to the smaller alpha); outputs the RTN of W * s_best and s_best.
// The weights of channel c are scaled up by s_c and its activations down by it (folded into
// the preceding layer), which leaves the layer's output unchanged before quantization.
#include <algorithm>
#include <vector>

#include "internal.cuh"
#include "quant.cuh"
#include "tcgemm.cuh"

namespace gq {

// sums[c] += sum over rows of |X[r][c]| (fp16 or fp32 X [n x d], row-major), fp64 partial sums:
// each thread owns two adjacent columns over a slice of rows, then one atomic add per column
template <typename T>
__global__ void __launch_bounds__(256) col_abs_sum_kernel(const T* __restrict__ X, int64_t n,
                                                          int d, int64_t rows_per_slice,
                                                          double* __restrict__ sums) {
    const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 2;
    if (c >= d) return;
    const int64_t r0 = blockIdx.y * rows_per_slice;
    const int64_t r1 = min(n, r0 + rows_per_slice);
    double a0 = 0.0, a1 = 0.0;
    const bool two = c + 1 < d;
    for (int64_t r = r0; r < r1; ++r) {
        const T* row = X + r * d;
        a0 += fabs(static_cast<double>(static_cast<float>(row[c])));
        if (two) a1 += fabs(static_cast<double>(static_cast<float>(row[c + 1])));
    }
    atomicAdd(&sums[c], a0);
    if (two) atomicAdd(&sums[c + 1], a1);
}

template <typename T>
static gptq_status col_abs_sum(const T* X, int64_t n, int d, double* sums, cudaStream_t s) {
    const int cols_blocks = (d + 511) / 512;
    const int64_t want = std::max<int64_t>(1, (static_cast<int64_t>(num_sms()) * 8) / cols_blocks);
    const int64_t slices = std::min<int64_t>(std::max<int64_t>(1, n / 64), std::min<int64_t>(want, 65535));
    const int64_t rps = (n + slices - 1) / slices;
    const dim3 grid(cols_blocks, static_cast<unsigned>((n + rps - 1) / rps));
    col_abs_sum_kernel<T><<<grid, 256, 0, s>>>(X, n, d, rps, sums);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

// s[i][c] for every alpha of the grid (fp16 values held in fp32)
__global__ void awq_scales_kernel(const double* __restrict__ x_sum, double x_count,
                                  const double* __restrict__ w_sum, double w_count, int d,
                                  int n_alpha, double alpha_step, float* __restrict__ s) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    const int i = blockIdx.y;
    if (c >= d || i >= n_alpha) return;
    const double xm = x_sum[c] / x_count, wm = w_sum[c] / w_count;
    // alpha = i*step and 1 - alpha rounded on their own, as the grid is defined (no fused
    // multiply-add)
    const double a = __dmul_rn(static_cast<double>(i), alpha_step);
    const double v = pow(xm, a) / pow(wm, __dsub_rn(1.0, a));
    const float h = __half2float(__double2half(v));
    const bool ok = xm > 0.0 && wm > 0.0 && isfinite(h) && h > 0.0f;
    s[static_cast<int64_t>(i) * d + c] = ok ? h : 1.0f;
}

// One warp per (row, group): W * s (exact for fp16 W and an fp16 s) -> group min-max grid ->
// codes; D = W - Q/s (fp32) when D is given, and the scaled weights W * s when ws_out is given
// (for the final RTN pass)
template <typename T>
__global__ void __launch_bounds__(256) awq_delta_kernel(const T* __restrict__ W, int d_out, int d,
                                                        int g, int bits, int sym,
                                                        const float* __restrict__ s,
                                                        float* __restrict__ D,
                                                        float* __restrict__ ws_out) {
    const int maxq = (1 << bits) - 1;
    const int ng = d / g;
    const int64_t units = static_cast<int64_t>(d_out) * ng;
    const int lane = threadIdx.x & 31;
    const int64_t wstride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t u = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         u < units; u += wstride) {
        const int64_t r = u / ng;
        const int c0 = static_cast<int>(u - r * ng) * g;
        const T* w = W + r * d + c0;
        float mn = 0.0f, mx = 0.0f;
        bool first = true;
        for (int i = lane; i < g; i += 32) {
            const float v = static_cast<float>(w[i]) * s[c0 + i];     // exact
            mn = first ? v : fminf(mn, v);
            mx = first ? v : fmaxf(mx, v);
            first = false;
        }
        if (first) {             // lanes without an element (g < 32) take a neutral value
            const float v = static_cast<float>(w[0]) * s[c0];
            mn = mx = v;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        }
        const QParams p = group_params_any(mn, mx, maxq, sym != 0);
        for (int i = lane; i < g; i += 32) {
            const float wv = static_cast<float>(w[i]);
            const float v = wv * s[c0 + i];
            if (D) D[r * d + c0 + i] = wv - dequant(quant_code(v, p, maxq), p) / s[c0 + i];
            if (ws_out) ws_out[r * d + c0 + i] = v;
        }
    }
}

// fp16 bit patterns of fp32 values that are fp16 values (exact)
__global__ void f32_to_f16_kernel(const float* __restrict__ src, uint16_t* __restrict__ dst,
                                  int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) dst[i] = half_bits(src[i]);
}

struct AwqWorkspace {
    double* w_sum;
    double* losses;
    float* s;        // [n_alpha][d]
    float* D;        // [d_out][d]
    int* status;
    size_t bytes;
};

static AwqWorkspace awq_layout(void* base, int d_out, int d, int n_alpha) {
    AwqWorkspace w{};
    size_t off = 0;
    auto take = [&](size_t b) {
        const size_t o = off;
        off += (b + 255) & ~static_cast<size_t>(255);
        return static_cast<uint8_t*>(base) + o;
    };
    w.status = reinterpret_cast<int*>(take(sizeof(int)));
    w.w_sum = reinterpret_cast<double*>(take(static_cast<size_t>(d) * 8));
    w.losses = reinterpret_cast<double*>(take(static_cast<size_t>(n_alpha) * 8));
    w.s = reinterpret_cast<float*>(take(static_cast<size_t>(n_alpha) * d * 4));
    w.D = reinterpret_cast<float*>(take(static_cast<size_t>(d_out) * d * 4));
    w.bytes = off;
    return w;
}

static int awq_n_alpha(double step) {
    const double nd = 1.0 / step;
    if (!(nd < 1000.0)) return -1;
    return static_cast<int>(nearbyint(nd)) + 1;
}

template <typename T>
static gptq_status awq_run(const T* W, int w_dtype, int d_out, int d, const double* x_sum,
                           int64_t n_tokens, const float* H, int bits, int g, int sym,
                           double alpha_step, int n_alpha, uint8_t* packed, uint16_t* scales,
                           uint16_t* zeros, uint16_t* s_out, double* losses_host, int* best_host,
                           const AwqWorkspace& ws, cudaStream_t st) {
    GPTQ_CUDA_TRY(cudaMemsetAsync(ws.status, 0, sizeof(int), st));
    GPTQ_CUDA_TRY(cudaMemsetAsync(ws.w_sum, 0, static_cast<size_t>(d) * 8, st));
    GPTQ_CUDA_TRY(cudaMemsetAsync(ws.losses, 0, static_cast<size_t>(n_alpha) * 8, st));
    GPTQ_TRY(col_abs_sum(W, d_out, d, ws.w_sum, st));
    {
        const dim3 grid((d + 255) / 256, n_alpha);
        awq_scales_kernel<<<grid, 256, 0, st>>>(x_sum, static_cast<double>(n_tokens), ws.w_sum,
                                                static_cast<double>(d_out), d, n_alpha,
                                                alpha_step, ws.s);
        GPTQ_LAUNCHED();
    }
    const int64_t units = static_cast<int64_t>(d_out) * (d / g);
    const int dblocks = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>((units + 7) / 8, static_cast<int64_t>(num_sms()) * 16)));
    for (int i = 0; i < n_alpha; ++i) {
        awq_delta_kernel<T><<<dblocks, 256, 0, st>>>(W, d_out, d, g, bits, sym,
                                                      ws.s + static_cast<int64_t>(i) * d, ws.D,
                                                      nullptr);
        GPTQ_LAUNCHED();
        TcGemmArgs a{};   // losses[i] = sum((D H) .* D) = tr(D H D^T); H symmetric, K-major
        a.M = d_out; a.N = d; a.K = d; a.alpha = 1.f; a.beta = 0.f;
        a.A = ws.D; a.lda = d; a.B = H; a.ldb = d; a.D = ws.D; a.ldd = d;
        a.dot = ws.losses + i; a.status = ws.status;
        GPTQ_TRY(tcgemm_launch(a, true, TC_EPI_DOT, true, true, st));
    }
    std::vector<double> L(n_alpha);
    int status = 0;
    GPTQ_CUDA_TRY(cudaMemcpyAsync(L.data(), ws.losses, static_cast<size_t>(n_alpha) * 8,
                                  cudaMemcpyDeviceToHost, st));
    GPTQ_CUDA_TRY(cudaMemcpyAsync(&status, ws.status, sizeof(int), cudaMemcpyDeviceToHost, st));
    GPTQ_CUDA_TRY(cudaStreamSynchronize(st));
    if (status) return static_cast<gptq_status>(status);
    int best = 0;
    for (int i = 1; i < n_alpha; ++i)
        if (L[i] < L[best]) best = i;
    if (losses_host)
        for (int i = 0; i < n_alpha; ++i) losses_host[i] = L[i];
    if (best_host) *best_host = best;
    // the chosen scales: W * s into D's buffer, then the RTN kernels on those fp32 weights
    awq_delta_kernel<T><<<dblocks, 256, 0, st>>>(W, d_out, d, g, bits, sym,
                                                  ws.s + static_cast<int64_t>(best) * d, nullptr,
                                                  ws.D);
    GPTQ_LAUNCHED();
    GPTQ_TRY(rtn_launch(ws.D, GPTQ_DTYPE_F32, d_out, d, bits, g, sym, packed, scales, zeros, st));
    if (s_out) {
        f32_to_f16_kernel<<<(d + 255) / 256, 256, 0, st>>>(ws.s + static_cast<int64_t>(best) * d,
                                                           s_out, d);
        GPTQ_LAUNCHED();
    }
    (void)w_dtype;
    return GPTQ_OK;
}

}  // namespace gq

extern "C" {

gptq_status gptq_channel_abs_sum(const void* X, int w_dtype, int64_t n, int d, double* sums,
                                 void* stream) {
    if (!X || !sums || n < 1 || d < 1) return GPTQ_ERR_ARG;
    if (w_dtype != GPTQ_DTYPE_F16 && w_dtype != GPTQ_DTYPE_F32) return GPTQ_ERR_ARG;
    GPTQ_TRY(gq::check_device());
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (w_dtype == GPTQ_DTYPE_F16) return gq::col_abs_sum(static_cast<const __half*>(X), n, d, sums, s);
    return gq::col_abs_sum(static_cast<const float*>(X), n, d, sums, s);
}

size_t awq_lite_workspace(int d_out, int d_in, double alpha_step) {
    const int n_alpha = gq::awq_n_alpha(alpha_step);
    if (d_out < 1 || d_in < 1 || n_alpha < 1) return 0;
    return gq::awq_layout(nullptr, d_out, d_in, n_alpha).bytes;
}

gptq_status awq_lite_search(const void* W, int w_dtype, int d_out, int d_in,
                            const double* x_abs_sum, int64_t n_tokens, const float* H, int bits,
                            int group_size, int sym, double alpha_step, uint8_t* packed,
                            uint16_t* scales, uint16_t* zeros, uint16_t* s_out,
                            double* losses, int* best, void* workspace, size_t workspace_bytes,
                            void* stream) {
    if (!W || !x_abs_sum || !H || !packed || !scales || !zeros || !workspace) return GPTQ_ERR_ARG;
    if (w_dtype != GPTQ_DTYPE_F16) return GPTQ_ERR_ARG;   // W * s exact needs fp16 weights
    if (d_out < 1 || d_in < 8 || d_in % 8 || bits < 2 || bits > 8 || sym < 0 || sym > 1)
        return GPTQ_ERR_ARG;
    if (group_size < 1 || d_in % group_size || n_tokens < 1) return GPTQ_ERR_ARG;
    if (!(alpha_step > 0.0) || !(alpha_step <= 1.0)) return GPTQ_ERR_ARG;
    const int n_alpha = gq::awq_n_alpha(alpha_step);
    if (n_alpha < 1) return GPTQ_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(W) & 15) || (reinterpret_cast<uintptr_t>(H) & 15) ||
        (reinterpret_cast<uintptr_t>(packed) & 15) || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return GPTQ_ERR_ARG;
    const gq::AwqWorkspace ws = gq::awq_layout(workspace, d_out, d_in, n_alpha);
    if (workspace_bytes < ws.bytes) return GPTQ_ERR_WORKSPACE;
    GPTQ_TRY(gq::check_device());
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    return gq::awq_run(static_cast<const __half*>(W), w_dtype, d_out, d_in, x_abs_sum,
                       n_tokens, H, bits, group_size, sym, alpha_step, n_alpha, packed, scales,
                       zeros, s_out, losses, best, ws, s);
}

}  // extern "C"
