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
#include "tcgemm.cuh"

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
// ---- diagonal block: one CTA factors the 128 x 128 block A[k0:, k0:] and inverts its factor.
// The block is split into four 32-column sub-panels. For each one, a single warp factors the
// 32 x 32 diagonal sub-block in registers (lane i holds row i; pivots and columns travel by
// shuffles, so the 32 sequential pivot steps need no block barrier) and inverts it the same
// way; then all warps solve the sub-panel below it against that inverse and apply the rank-32
// update to the trailing part of the block. Finally the inverse of the whole 128 x 128 factor
// is assembled from the four sub-block inverses by block forward substitution. Rows and
// columns beyond the matrix edge (last block) are padded with the identity. The solve, update
// and assembly loops work on 4-column strips so one shared-memory load feeds four FMAs; the
// operands they stream across columns are kept transposed for that.
namespace pd {
constexpr int NB = 128, SUB = 32, THREADS = 512;
constexpr int LD = NB + 1;        // S: scalar row access
constexpr int LDV = NB + 4;       // Dv, LT: float4 row access
constexpr int LDX = SUB + 4;      // XT: float4 row access
constexpr int SMEM = (NB * LD + NB * LDV + SUB * LDV + 4 * SUB * LDX) * 4;
}  // namespace pd

// v: row `lane` of a 32 x 32 SPD block (lower part used). On return v holds row `lane` of its
// Cholesky factor L (zeros above the diagonal) and x holds row `lane` of L^-1.
__device__ __forceinline__ void warp_chol_inv32(float (&v)[32], float (&x)[32], int lane,
                                                bool& bad) {
    const unsigned full = 0xffffffffu;
    float rdiag = 1.0f;   // 1 / L[lane][lane]
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        const float piv = __shfl_sync(full, v[c], c);
        if (!(piv > 0.0f) || !isfinite(piv)) bad = true;
        float r = rsqrtf(piv);
        r = r * fmaf(-0.5f * piv, r * r, 1.5f);   // one Newton step: r = 1/sqrt(piv)
        if (lane == c) rdiag = r;
        const float lic = (lane >= c) ? v[c] * r : 0.0f;
        v[c] = lic;
#pragma unroll
        for (int j = c + 1; j < 32; ++j) {
            const float ljc = __shfl_sync(full, lic, j);
            v[j] = fmaf(-lic, ljc, v[j]);
        }
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        if (j > lane) v[j] = 0.0f;
        x[j] = (j == lane) ? 1.0f : 0.0f;
    }
    // forward substitution on the identity with the row scaling deferred: when row k is
    // broadcast it is scaled by 1/L[k][k] on the fly; each lane scales its own row at the end
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const float rkk = __shfl_sync(full, rdiag, k);
        const float nlik = (lane > k) ? -v[k] : 0.0f;
#pragma unroll
        for (int j = 0; j <= k; ++j) {
            const float xkj = __shfl_sync(full, x[j], k) * rkk;
            x[j] = fmaf(nlik, xkj, x[j]);
        }
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] *= rdiag;
}

__global__ void __launch_bounds__(pd::THREADS) potrf_diag_kernel(float* __restrict__ A, int d,
                                                                int k0, int nbc,
                                                                float* __restrict__ Dinv,
                                                                int* status) {
    if (status_bad(status)) return;
    extern __shared__ __align__(16) float sm[];
    float* S = sm;                          // [NB][LD]: the block, then its factor L
    float* Dv = S + pd::NB * pd::LD;        // [NB][LDV]: L^-1
    float* LT = Dv + pd::NB * pd::LDV;      // [SUB][LDV]: current sub-panel of L, transposed
    float* XT = LT + pd::SUB * pd::LDV;     // [4][SUB][LDX]: sub-block inverses, transposed
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int NW = pd::THREADS / 32;

    // load: 32 independent loads per thread, then the stores (identity padding past the edge)
    {
        float vals[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int e = tid + t * pd::THREADS, i = e >> 7, j = e & 127;
            vals[t] = (i < nbc && j <= i) ? A[static_cast<int64_t>(k0 + i) * d + k0 + j] : 0.0f;
        }
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int e = tid + t * pd::THREADS, i = e >> 7, j = e & 127;
            S[i * pd::LD + j] = (i >= nbc && i == j) ? 1.0f : vals[t];
        }
    }
    __syncthreads();

    bool bad = false;
    for (int sp = 0; sp < 4; ++sp) {
        const int c0 = pd::SUB * sp;
        float* X = XT + sp * pd::SUB * pd::LDX;      // X^T: X[j][k] stored at [k][j]
        if (warp == 0) {
            float v[32], x[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = (j <= lane) ? S[(c0 + lane) * pd::LD + c0 + j] : 0.0f;
            warp_chol_inv32(v, x, lane, bad);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                if (j <= lane) S[(c0 + lane) * pd::LD + c0 + j] = v[j];
                X[j * pd::LDX + lane] = x[j];        // row lane of X -> column lane of X^T
                LT[j * pd::LDV + c0 + lane] = v[j];  // L[c0+lane][c0+j] -> LT[j][c0+lane]
            }
        }
        __syncthreads();
        // sub-panel below: L[r][c0+j] = sum_{k<=j} A[r][c0+k] * X[j][k], computed for 4
        // consecutive j per thread (rows r0..127: at most 96 x 8 strips, 2 per thread)
        const int r0 = c0 + pd::SUB, nr = pd::NB - r0;
        float4 out[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int idx = tid + t * pd::THREADS;
            out[t] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (idx < nr * 8) {
                const int r = r0 + (idx >> 3), j4 = (idx & 7) * 4;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int k = 0; k < j4 + 4; ++k) {
                    const float a = S[r * pd::LD + c0 + k];
                    const float4 xv = *reinterpret_cast<const float4*>(&X[k * pd::LDX + j4]);
                    acc.x = fmaf(a, xv.x, acc.x);
                    acc.y = fmaf(a, xv.y, acc.y);
                    acc.z = fmaf(a, xv.z, acc.z);
                    acc.w = fmaf(a, xv.w, acc.w);
                }
                out[t] = acc;
            }
        }
        __syncthreads();
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int idx = tid + t * pd::THREADS;
            if (idx < nr * 8) {
                const int r = r0 + (idx >> 3), j4 = (idx & 7) * 4;
                float* dst = &S[r * pd::LD + c0 + j4];
                dst[0] = out[t].x; dst[1] = out[t].y; dst[2] = out[t].z; dst[3] = out[t].w;
                LT[(j4 + 0) * pd::LDV + r] = out[t].x;
                LT[(j4 + 1) * pd::LDV + r] = out[t].y;
                LT[(j4 + 2) * pd::LDV + r] = out[t].z;
                LT[(j4 + 3) * pd::LDV + r] = out[t].w;
            }
        }
        __syncthreads();
        // trailing update: S[r][c..c+3] -= sum_k L[r][c0+k] L[c..c+3][c0+k] for r0 <= c <= r
        for (int r = r0 + warp; r < pd::NB; r += NW) {
            for (int cq = r0 / 4 + lane; cq * 4 <= r; cq += 32) {
                const int c = cq * 4;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
                for (int k = 0; k < pd::SUB; ++k) {
                    const float a = S[r * pd::LD + c0 + k];
                    const float4 lv = *reinterpret_cast<const float4*>(&LT[k * pd::LDV + c]);
                    acc.x = fmaf(a, lv.x, acc.x);
                    acc.y = fmaf(a, lv.y, acc.y);
                    acc.z = fmaf(a, lv.z, acc.z);
                    acc.w = fmaf(a, lv.w, acc.w);
                }
                float* dst = &S[r * pd::LD + c];
                dst[0] -= acc.x;
                if (c + 1 <= r) dst[1] -= acc.y;
                if (c + 2 <= r) dst[2] -= acc.z;
                if (c + 3 <= r) dst[3] -= acc.w;
            }
        }
        __syncthreads();
    }
    if (warp == 0 && lane == 0 && bad) set_status(status, GPTQ_ERR_NOT_PD);

    // inverse of the whole factor: diagonal 32-blocks are the sub-block inverses;
    // Dv[I][J] = -X_I * sum_{K=J}^{I-1} L[I][K] Dv[K][J] for J < I
    for (int e = tid; e < pd::NB * pd::NB; e += pd::THREADS) {
        const int i = e >> 7, j = e & 127, I = i >> 5, J = j >> 5;
        Dv[i * pd::LDV + j] =
            (I == J) ? XT[I * pd::SUB * pd::LDX + (j & 31) * pd::LDX + (i & 31)] : 0.0f;
    }
    __syncthreads();
    for (int I = 1; I < 4; ++I) {
        // T = sum_K L[I][K] Dv[K][J] for all J < I: 32 rows x 8*I four-column strips
        const int nq = 8 * I, total = 32 * nq;
        float4 out[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int idx = tid + t * pd::THREADS;
            out[t] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (idx < total) {
                const int a = idx / nq, col = (idx % nq) * 4, J = col >> 5;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int k = 32 * J; k < 32 * I; ++k) {
                    const float l = S[(32 * I + a) * pd::LD + k];
                    const float4 dv = *reinterpret_cast<const float4*>(&Dv[k * pd::LDV + col]);
                    acc.x = fmaf(l, dv.x, acc.x);
                    acc.y = fmaf(l, dv.y, acc.y);
                    acc.z = fmaf(l, dv.z, acc.z);
                    acc.w = fmaf(l, dv.w, acc.w);
                }
                out[t] = acc;
            }
        }
        __syncthreads();
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int idx = tid + t * pd::THREADS;
            if (idx < total)
                *reinterpret_cast<float4*>(&Dv[(32 * I + idx / nq) * pd::LDV + (idx % nq) * 4]) = out[t];
        }
        __syncthreads();
        // Dv[I][J] = -X_I * T  (X_I lower: X_I[a][k] = XT_I[k][a])
        const float* XI = XT + I * pd::SUB * pd::LDX;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int idx = tid + t * pd::THREADS;
            out[t] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (idx < total) {
                const int a = idx / nq, col = (idx % nq) * 4;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int k = 0; k <= a; ++k) {
                    const float xa = XI[k * pd::LDX + a];
                    const float4 tv = *reinterpret_cast<const float4*>(&Dv[(32 * I + k) * pd::LDV + col]);
                    acc.x = fmaf(xa, tv.x, acc.x);
                    acc.y = fmaf(xa, tv.y, acc.y);
                    acc.z = fmaf(xa, tv.z, acc.z);
                    acc.w = fmaf(xa, tv.w, acc.w);
                }
                out[t] = make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
            }
        }
        __syncthreads();
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int idx = tid + t * pd::THREADS;
            if (idx < total)
                *reinterpret_cast<float4*>(&Dv[(32 * I + idx / nq) * pd::LDV + (idx % nq) * 4]) = out[t];
        }
        __syncthreads();
    }
    for (int e = tid; e < pd::NB * pd::NB; e += pd::THREADS) {
        const int i = e >> 7, j = e & 127;
        const bool in = i < nbc && j < nbc && j <= i;
        Dinv[i * pd::NB + j] = in ? Dv[i * pd::LDV + j] : 0.0f;
        if (in) A[static_cast<int64_t>(k0 + i) * d + k0 + j] = S[i * pd::LD + j];
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
    static_assert(kCholBlock == pd::NB, "diagonal-block kernel is written for 128-wide panels");
    const int smem = pd::SMEM;
    if (g_potrf_smem != smem) {
        GPTQ_CUDA_TRY(cudaFuncSetAttribute(potrf_diag_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
        g_potrf_smem = smem;
    }
    const int nbl = (d + nb - 1) / nb;
    for (int m = 0; m < nbl; ++m) {
        const int k0 = m * nb, nbc = std::min(nb, d - k0);
        float* Dm = Dinv + static_cast<int64_t>(m) * nb * nb;
        potrf_diag_kernel<<<1, pd::THREADS, smem, s>>>(A, d, k0, nbc, Dm, status);
        GPTQ_LAUNCHED();
        const int rem = d - k0 - nbc;
        if (rem <= 0) continue;
        float* A21 = A + static_cast<int64_t>(k0 + nbc) * d + k0;
        TcGemmArgs t{};  // P = A21 * Dinv_m^T
        t.M = rem; t.N = nbc; t.K = nbc; t.alpha = 1.f; t.beta = 0.f;
        t.A = A21; t.lda = d; t.B = Dm; t.ldb = nb; t.C = P; t.ldc = nb; t.status = status;
        GPTQ_TRY(tcgemm_launch(t, true, TC_EPI_STORE, true, true, s));
        GPTQ_TRY(copy2d(P, nb, A21, d, rem, nbc, s));
        TcGemmArgs u{};  // A22 -= P P^T (lower tiles)
        u.M = rem; u.N = rem; u.K = nbc; u.alpha = -1.f; u.beta = 1.f;
        u.A = P; u.lda = nb; u.B = P; u.ldb = nb;
        u.C = A + static_cast<int64_t>(k0 + nbc) * d + (k0 + nbc); u.ldc = d;
        u.lower_only = 1; u.status = status;
        GPTQ_TRY(tcgemm_launch(u, true, TC_EPI_STORE, true, true, s));
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
        TcGemmArgs t{};  // P = Dinv_m * X[k0:k0+nbc, 0:ncol]
        t.M = nbc; t.N = ncol; t.K = nbc; t.alpha = 1.f; t.beta = 0.f;
        t.A = Dm; t.lda = nb; t.B = X + static_cast<int64_t>(k0) * d; t.ldb = d;
        t.C = P; t.ldc = d; t.status = status;
        GPTQ_TRY(tcgemm_launch(t, false, TC_EPI_STORE, true, true, s));
        GPTQ_TRY(copy2d(P, d, X + static_cast<int64_t>(k0) * d, d, nbc, ncol, s));
        const int rem = d - ncol;
        if (rem <= 0) continue;
        TcGemmArgs u{};  // X[ncol:, 0:ncol] -= L[ncol:, k0:ncol] * X[k0:ncol, 0:ncol]
        u.M = rem; u.N = ncol; u.K = nbc; u.alpha = -1.f; u.beta = 1.f;
        u.A = A + static_cast<int64_t>(ncol) * d + k0; u.lda = d;
        u.B = X + static_cast<int64_t>(k0) * d; u.ldb = d;
        u.C = X + static_cast<int64_t>(ncol) * d; u.ldc = d; u.status = status;
        GPTQ_TRY(tcgemm_launch(u, false, TC_EPI_STORE, true, true, s));
    }
    const int64_t half = static_cast<int64_t>(d) * d / 2;
    const int blocks = static_cast<int>(std::min<int64_t>((half + 255) / 256, num_sms() * 16));
    reverse_inplace_kernel<<<blocks, 256, 0, s>>>(X, half);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

}  // namespace gq
