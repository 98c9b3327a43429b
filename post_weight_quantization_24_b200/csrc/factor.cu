// Damping, act_order permutation, and the fp32 factorisation that yields U with U^T U = H_d^-1.
//
// GPTQ deep-dive (hncyxsy.com/news/243429) §3.1 steps 1-2 and §3.3: lambda on the diagonal
// (damp_percent, a ratio on the Hessian diagonal, default 0.01), then a Cholesky
// factorisation used in place of repeated inversion; §2.4: the factorisation is what makes
// the column updates cheap and stable. bhfrc.com/news/5741 §2.3 and hncyxsy.com §3.3:
// desc_act processes columns by descending Hessian diagonal.
//
// Route: with P the index reversal, factor A = P·H_d·P = L L^T (right-looking blocked
// Cholesky, 128-wide panels), invert L blockwise (right-looking triangular solve of L X = I
// using the inverses of the diagonal blocks), and U = P·L^-1·P, which is upper triangular with
// U^T U = H_d^-1 (the unique upper Cholesky factor of the inverse). The permutation and the
// reversal are folded into one gather of H.
#include <algorithm>

#include "internal.cuh"
#include "sgemm.cuh"

namespace gq {

// ---------------------------------------------------------------------------------------
// lambda = percdamp * mean(diag H), computed in fp64 by one block in a fixed order
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) diag_stats_kernel(const float* __restrict__ H, int d,
                                                          double percdamp, DevState* st) {
    double s = 0.0;
    int bad = 0;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
        const float v = H[static_cast<int64_t>(i) * d + i];
        if (!isfinite(v)) bad = 1;
        s += static_cast<double>(v);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        s += __shfl_xor_sync(0xffffffffu, s, off);
        bad |= __shfl_xor_sync(0xffffffffu, bad, off);
    }
    __shared__ double ws[32];
    __shared__ int wb[32];
    if ((threadIdx.x & 31) == 0) {
        ws[threadIdx.x >> 5] = s;
        wb[threadIdx.x >> 5] = bad;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        int b = 0;
        for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
            t += ws[w];
            b |= wb[w];
        }
        st->diag_sum = t;
        const double lam = percdamp * (t / d);
        st->lam = lam;
        if (b) set_status(&st->status, GPTQ_ERR_NONFINITE);
        else if (!(lam > 0.0) || !isfinite(lam)) set_status(&st->status, GPTQ_ERR_NOT_PD);
    }
}

gptq_status diag_stats_launch(const float* H, int d, double percdamp, DevState* st,
                              cudaStream_t s) {
    diag_stats_kernel<<<1, 1024, 0, s>>>(H, d, percdamp, st);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

// ---------------------------------------------------------------------------------------
// processing order: rank of each column by descending diag(H), ties by lower index
// ---------------------------------------------------------------------------------------
__global__ void identity_perm_kernel(int d, int* perm, int* invperm) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < d) {
        perm[i] = i;
        invperm[i] = i;
    }
}

__global__ void __launch_bounds__(256) act_order_rank_kernel(const float* __restrict__ H, int d,
                                                             int* perm, int* invperm) {
    constexpr int CHUNK = 4096;
    __shared__ float keys[CHUNK];
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const float ki = i < d ? H[static_cast<int64_t>(i) * d + i] : 0.0f;
    int rank = 0;
    for (int base = 0; base < d; base += CHUNK) {
        const int cnt = min(CHUNK, d - base);
        __syncthreads();
        for (int t = threadIdx.x; t < cnt; t += blockDim.x)
            keys[t] = H[static_cast<int64_t>(base + t) * d + base + t];
        __syncthreads();
        if (i < d) {
            for (int t = 0; t < cnt; ++t) {
                const float kj = keys[t];
                rank += (kj > ki) || (kj == ki && base + t < i);
            }
        }
    }
    // ranks are a permutation for finite keys; with NaN keys (reported as NONFINITE) slots
    // may collide, and the identity written first keeps every entry a valid index
    if (i < d) {
        perm[rank] = i;
        invperm[i] = rank;
    }
}

gptq_status act_order_launch(const float* H, int d, int act_order, int* perm, int* invperm,
                             cudaStream_t s) {
    identity_perm_kernel<<<(d + 255) / 256, 256, 0, s>>>(d, perm, invperm);
    GPTQ_LAUNCHED();
    if (act_order) {
        act_order_rank_kernel<<<(d + 255) / 256, 256, 0, s>>>(H, d, perm, invperm);
        GPTQ_LAUNCHED();
    }
    return GPTQ_OK;
}

// ---------------------------------------------------------------------------------------
// gathers
// ---------------------------------------------------------------------------------------
__global__ void gather_h_kernel(const float* __restrict__ H, int d, const int* __restrict__ perm,
                                const DevState* __restrict__ st, int reversed,
                                float* __restrict__ A, int* status) {
    const int j = blockIdx.x * 32 + threadIdx.x;
    if (j >= d) return;
    const int b = reversed ? perm[d - 1 - j] : perm[j];
    const double lam = reversed ? st->lam : 0.0;
    int bad = 0;
    for (int k = threadIdx.y; k < 32; k += blockDim.y) {
        const int i = blockIdx.y * 32 + k;
        if (i >= d) break;
        const int a = reversed ? perm[d - 1 - i] : perm[i];
        const int lo = min(a, b), hi = max(a, b);
        float v = H[static_cast<int64_t>(lo) * d + hi];
        if (!isfinite(v)) bad = 1;
        if (i == j && reversed) v = static_cast<float>(static_cast<double>(v) + lam);
        A[static_cast<int64_t>(i) * d + j] = v;
    }
    if (bad) set_status(status, GPTQ_ERR_NONFINITE);
}

gptq_status gather_h_launch(const float* H, int d, const int* perm, const DevState* st,
                            int reversed, float* A, int* status, cudaStream_t s) {
    const dim3 grid((d + 31) / 32, (d + 31) / 32), block(32, 8);
    gather_h_kernel<<<grid, block, 0, s>>>(H, d, perm, st, reversed, A, status);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

template <typename T>
__global__ void gather_w_kernel(const T* __restrict__ W, int d_out, int d_in,
                                const int* __restrict__ perm, float* __restrict__ Wk,
                                int* status) {
    const int64_t n = static_cast<int64_t>(d_out) * d_in;
    int bad = 0;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = e / d_in;
        const int p = static_cast<int>(e - r * d_in);
        const float v = static_cast<float>(W[r * d_in + perm[p]]);
        if (!isfinite(v)) bad = 1;
        Wk[e] = v;
    }
    if (bad) set_status(status, GPTQ_ERR_NONFINITE);
}

gptq_status gather_w_launch(const void* W, int w_dtype, int d_out, int d_in, const int* perm,
                            float* Wk, int* status, cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(d_out) * d_in;
    const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, num_sms() * 32));
    if (w_dtype == GPTQ_DTYPE_F16)
        gather_w_kernel<__half><<<blocks, 256, 0, s>>>(static_cast<const __half*>(W), d_out, d_in,
                                                       perm, Wk, status);
    else
        gather_w_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(W), d_out, d_in,
                                                      perm, Wk, status);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

// ---------------------------------------------------------------------------------------
// blocked Cholesky
// ---------------------------------------------------------------------------------------
// One CTA factors the nbc x nbc diagonal block A[k0:, k0:] in shared memory (right-looking,
// one barrier per pivot: the trailing update uses the unscaled column divided by the pivot,
// and the columns are scaled by 1/sqrt(pivot) at the end), writes L11 back, and computes
// Dinv = L11^-1 by forward elimination on the identity (again one barrier per row).
__global__ void __launch_bounds__(1024) potrf_diag_kernel(float* __restrict__ A, int d, int k0,
                                                          int nbc, float* __restrict__ Dinv,
                                                          int nb, int* status) {
    if (status_bad(status)) return;
    extern __shared__ float sm[];
    const int LD = nb + 1;
    float* S = sm;
    float* X = sm + nb * LD;
    float* dsq = X + nb * LD;
    const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;

    for (int i = ty; i < nbc; i += 32)
        for (int j = tx; j <= i; j += 32)
            S[i * LD + j] = A[static_cast<int64_t>(k0 + i) * d + k0 + j];
    __syncthreads();

    for (int c = 0; c < nbc; ++c) {
        const float piv = S[c * LD + c];
        if (tid == 0 && !(piv > 0.0f && isfinite(piv))) set_status(status, GPTQ_ERR_NOT_PD);
        const float rinv = 1.0f / piv;
        for (int i = c + 1 + ty; i < nbc; i += 32) {
            const float lic = S[i * LD + c] * rinv;
            for (int j = c + 1 + tx; j <= i; j += 32) S[i * LD + j] -= lic * S[j * LD + c];
        }
        __syncthreads();
    }
    for (int c = tid; c < nbc; c += blockDim.x) dsq[c] = sqrtf(S[c * LD + c]);
    __syncthreads();
    for (int i = ty; i < nbc; i += 32)
        for (int j = tx; j <= i; j += 32) {
            const float l = S[i * LD + j] / dsq[j];
            S[i * LD + j] = l;
            A[static_cast<int64_t>(k0 + i) * d + k0 + j] = l;
        }
    for (int i = ty; i < nb; i += 32)
        for (int j = tx; j < nb; j += 32) X[i * LD + j] = (i == j) ? 1.0f : 0.0f;
    __syncthreads();

    for (int k = 0; k < nbc; ++k) {
        const float lkk_inv = 1.0f / S[k * LD + k];
        for (int i = k + 1 + ty; i < nbc; i += 32) {
            const float f = S[i * LD + k] * lkk_inv;
            for (int j = tx; j <= k; j += 32) X[i * LD + j] -= f * X[k * LD + j];
        }
        __syncthreads();
    }
    for (int i = ty; i < nb; i += 32)
        for (int j = tx; j < nb; j += 32) {
            float v = 0.0f;
            if (i < nbc && j <= i) v = X[i * LD + j] / S[i * LD + i];
            Dinv[i * nb + j] = v;
        }
}

__global__ void copy2d_kernel(const float* __restrict__ src, int lds, float* __restrict__ dst,
                              int ldd, int rows, int cols4) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    const int r = blockIdx.y;
    if (r < rows && c < cols4)
        reinterpret_cast<float4*>(dst + static_cast<int64_t>(r) * ldd)[c] =
            reinterpret_cast<const float4*>(src + static_cast<int64_t>(r) * lds)[c];
}

static gptq_status copy2d(const float* src, int lds, float* dst, int ldd, int rows, int cols,
                          cudaStream_t s) {
    if (rows <= 0 || cols <= 0) return GPTQ_OK;
    const int cols4 = cols / 4;
    const dim3 grid((cols4 + 127) / 128, rows);
    copy2d_kernel<<<grid, 128, 0, s>>>(src, lds, dst, ldd, rows, cols4);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

static int g_potrf_smem = 0;

gptq_status cholesky_launch(float* A, int d, float* Dinv, float* P, int* status, cudaStream_t s) {
    const int nb = kCholBlock;
    const int smem = (2 * nb * (nb + 1) + nb) * 4;
    if (g_potrf_smem != smem) {
        GPTQ_CUDA_TRY(cudaFuncSetAttribute(potrf_diag_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
        g_potrf_smem = smem;
    }
    const int nbl = (d + nb - 1) / nb;
    for (int m = 0; m < nbl; ++m) {
        const int k0 = m * nb, nbc = std::min(nb, d - k0);
        float* Dm = Dinv + static_cast<int64_t>(m) * nb * nb;
        potrf_diag_kernel<<<1, 1024, smem, s>>>(A, d, k0, nbc, Dm, nb, status);
        GPTQ_LAUNCHED();
        const int rem = d - k0 - nbc;
        if (rem <= 0) continue;
        float* A21 = A + static_cast<int64_t>(k0 + nbc) * d + k0;
        SgemmArgs t{};  // P = A21 * Dinv_m^T
        t.M = rem; t.N = nbc; t.K = nbc; t.alpha = 1.f; t.beta = 0.f;
        t.A = A21; t.lda = d; t.B = Dm; t.ldb = nb; t.C = P; t.ldc = nb;
        t.abort_flag = status;
        GPTQ_TRY(sgemm_launch(t, true, EPI_STORE, s));
        GPTQ_TRY(copy2d(P, nb, A21, d, rem, nbc, s));
        SgemmArgs u{};  // A22 -= P P^T (lower tiles)
        u.M = rem; u.N = rem; u.K = nbc; u.alpha = -1.f; u.beta = 1.f;
        u.A = P; u.lda = nb; u.B = P; u.ldb = nb;
        u.C = A + static_cast<int64_t>(k0 + nbc) * d + (k0 + nbc); u.ldc = d;
        u.lower_only = 1; u.abort_flag = status;
        GPTQ_TRY(sgemm_launch(u, true, EPI_STORE, s));
    }
    return GPTQ_OK;
}

// ---------------------------------------------------------------------------------------
// triangular inverse and reversal
// ---------------------------------------------------------------------------------------
__global__ void set_identity_kernel(float* X, int d) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < d) X[static_cast<int64_t>(i) * d + i] = 1.0f;
}

// U[p][q] = X[d-1-p][d-1-q]: swap element e with element d*d-1-e
__global__ void reverse_inplace_kernel(float* X, int64_t half) {
    const int64_t n = 2 * half;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < half;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float a = X[e], b = X[n - 1 - e];
        X[e] = b;
        X[n - 1 - e] = a;
    }
}

gptq_status trtri_reverse_launch(const float* A, int d, const float* Dinv, float* X, float* P,
                                 int* status, cudaStream_t s) {
    const int nb = kCholBlock;
    GPTQ_CUDA_TRY(cudaMemsetAsync(X, 0, static_cast<size_t>(d) * d * 4, s));
    set_identity_kernel<<<(d + 255) / 256, 256, 0, s>>>(X, d);
    GPTQ_LAUNCHED();
    const int nbl = (d + nb - 1) / nb;
    for (int m = 0; m < nbl; ++m) {
        const int k0 = m * nb, nbc = std::min(nb, d - k0), ncol = k0 + nbc;
        const float* Dm = Dinv + static_cast<int64_t>(m) * nb * nb;
        SgemmArgs t{};  // P = Dinv_m * X[k0:k0+nbc, 0:ncol]
        t.M = nbc; t.N = ncol; t.K = nbc; t.alpha = 1.f; t.beta = 0.f;
        t.A = Dm; t.lda = nb; t.B = X + static_cast<int64_t>(k0) * d; t.ldb = d;
        t.C = P; t.ldc = d; t.abort_flag = status;
        GPTQ_TRY(sgemm_launch(t, false, EPI_STORE, s));
        GPTQ_TRY(copy2d(P, d, X + static_cast<int64_t>(k0) * d, d, nbc, ncol, s));
        const int rem = d - ncol;
        if (rem <= 0) continue;
        SgemmArgs u{};  // X[ncol:, 0:ncol] -= L[ncol:, k0:ncol] * X[k0:ncol, 0:ncol]
        u.M = rem; u.N = ncol; u.K = nbc; u.alpha = -1.f; u.beta = 1.f;
        u.A = A + static_cast<int64_t>(ncol) * d + k0; u.lda = d;
        u.B = X + static_cast<int64_t>(k0) * d; u.ldb = d;
        u.C = X + static_cast<int64_t>(ncol) * d; u.ldc = d; u.abort_flag = status;
        GPTQ_TRY(sgemm_launch(u, false, EPI_STORE, s));
    }
    const int64_t half = static_cast<int64_t>(d) * d / 2;
    const int blocks = static_cast<int>(std::min<int64_t>((half + 255) / 256, num_sms() * 16));
    reverse_inplace_kernel<<<blocks, 256, 0, s>>>(X, half);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

}  // namespace gq
