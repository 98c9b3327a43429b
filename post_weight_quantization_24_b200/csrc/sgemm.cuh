// fp32 GEMM on the FMA pipe: C = beta*C + alpha * A * op(B), row-major, with two epilogues:
//   EPI_STORE  write C
//   EPI_DOT    no C: accumulate sum(acc .* D) into a double (for trace forms tr(A B D^T))
// A is [M x K] (lda); B is [K x N] (ldb) when B_T is false, or [N x K] (ldb) when B_T is true.
// 128 x 128 x 8 tiles, 256 threads, an 8 x 8 register tile per thread split 4+4 in each
// direction so shared-memory reads are conflict-free float4s; double-buffered smem with
// register prefetch. `lower_only` skips tiles that lie entirely above the diagonal (SYRK).
// Requirements (checked by sgemm_launch): K % 4 == 0, N % 4 == 0, lda/ldb/ldc/ldd % 4 == 0,
// all base pointers 16-byte aligned.
#pragma once

#include "common.cuh"

namespace gq {

enum { EPI_STORE = 0, EPI_DOT = 1 };

struct SgemmArgs {
    int M, N, K;
    float alpha, beta;
    const float* A;
    int lda;
    const float* B;
    int ldb;
    float* C;
    int ldc;
    const float* D;   // EPI_DOT operand, [M x N], ldd
    int ldd;
    double* dot;      // EPI_DOT accumulator (device)
    int lower_only;
    const int* abort_flag;  // optional: skip all work when *abort_flag != 0
};

namespace sg {
constexpr int BM = 128, BN = 128, BK = 8, THREADS = 256;
}

template <bool B_T, int EPI>
__global__ void __launch_bounds__(sg::THREADS, 2) sgemm_kernel(const SgemmArgs a) {
    if (status_bad(a.abort_flag)) return;
    const int m0 = blockIdx.y * sg::BM, n0 = blockIdx.x * sg::BN;
    if (a.lower_only && m0 + sg::BM - 1 < n0) return;

    __shared__ __align__(16) float As[2][sg::BK][sg::BM + 4];
    __shared__ __align__(16) float Bs[2][sg::BK][sg::BN + 4];

    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;

    // global -> register loaders (one float4 of A and one of B per thread per k-tile)
    const int a_row = tid >> 1, a_k = (tid & 1) * 4;
    const int bt_row = tid >> 1, bt_k = (tid & 1) * 4;        // B_T: B is [N x K]
    const int bn_k = tid >> 5, bn_col = (tid & 31) * 4;       // !B_T: B is [K x N]

    const bool a_ok = (m0 + a_row) < a.M;
    const float* a_ptr = a.A + static_cast<int64_t>(m0 + a_row) * a.lda + a_k;
    const bool bt_ok = (n0 + bt_row) < a.N;
    const float* bt_ptr = a.B + static_cast<int64_t>(n0 + bt_row) * a.ldb + bt_k;
    const bool bn_ok = (n0 + bn_col) < a.N;
    const float* bn_ptr = a.B + static_cast<int64_t>(bn_k) * a.ldb + n0 + bn_col;

    float4 ra, rb;
    auto load_tile = [&](int k0) {
        ra = (a_ok && k0 + a_k < a.K) ? *reinterpret_cast<const float4*>(a_ptr + k0)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
        if (B_T) {
            rb = (bt_ok && k0 + bt_k < a.K) ? *reinterpret_cast<const float4*>(bt_ptr + k0)
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
            rb = (bn_ok && k0 + bn_k < a.K)
                     ? *reinterpret_cast<const float4*>(bn_ptr + static_cast<int64_t>(k0) * a.ldb)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto store_tile = [&](int buf) {
        As[buf][a_k + 0][a_row] = ra.x;
        As[buf][a_k + 1][a_row] = ra.y;
        As[buf][a_k + 2][a_row] = ra.z;
        As[buf][a_k + 3][a_row] = ra.w;
        if (B_T) {
            Bs[buf][bt_k + 0][bt_row] = rb.x;
            Bs[buf][bt_k + 1][bt_row] = rb.y;
            Bs[buf][bt_k + 2][bt_row] = rb.z;
            Bs[buf][bt_k + 3][bt_row] = rb.w;
        } else {
            *reinterpret_cast<float4*>(&Bs[buf][bn_k][bn_col]) = rb;
        }
    };

    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    const int n_kt = (a.K + sg::BK - 1) / sg::BK;
    load_tile(0);
    store_tile(0);
    __syncthreads();
    for (int kt = 0; kt < n_kt; ++kt) {
        const int buf = kt & 1;
        if (kt + 1 < n_kt) load_tile((kt + 1) * sg::BK);
#pragma unroll
        for (int k = 0; k < sg::BK; ++k) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][k][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][k][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][k][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][k][64 + tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        if (kt + 1 < n_kt) store_tile(buf ^ 1);
        __syncthreads();
    }

    if (EPI == EPI_STORE) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
            if (r >= a.M) continue;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c = n0 + h * 64 + tx * 4;
                if (c >= a.N) continue;
                float* cp = a.C + static_cast<int64_t>(r) * a.ldc + c;
                float4 v = make_float4(a.alpha * acc[i][4 * h], a.alpha * acc[i][4 * h + 1],
                                       a.alpha * acc[i][4 * h + 2], a.alpha * acc[i][4 * h + 3]);
                if (a.beta != 0.f) {
                    const float4 o = *reinterpret_cast<const float4*>(cp);
                    v.x = fmaf(a.beta, o.x, v.x);
                    v.y = fmaf(a.beta, o.y, v.y);
                    v.z = fmaf(a.beta, o.z, v.z);
                    v.w = fmaf(a.beta, o.w, v.w);
                }
                *reinterpret_cast<float4*>(cp) = v;
            }
        }
    } else {
        double s = 0.0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
            if (r >= a.M) continue;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c = n0 + h * 64 + tx * 4;
                if (c >= a.N) continue;
                const float4 dv =
                    *reinterpret_cast<const float4*>(a.D + static_cast<int64_t>(r) * a.ldd + c);
                float part = acc[i][4 * h] * dv.x;
                part = fmaf(acc[i][4 * h + 1], dv.y, part);
                part = fmaf(acc[i][4 * h + 2], dv.z, part);
                part = fmaf(acc[i][4 * h + 3], dv.w, part);
                s += static_cast<double>(part);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        __shared__ double red[sg::THREADS / 32];
        if ((tid & 31) == 0) red[tid >> 5] = s;
        __syncthreads();
        if (tid == 0) {
            double t = 0.0;
            for (int w = 0; w < sg::THREADS / 32; ++w) t += red[w];
            atomicAdd(a.dot, static_cast<double>(a.alpha) * t);
        }
    }
}

gptq_status sgemm_launch(const SgemmArgs& a, bool b_trans, int epi, cudaStream_t s);

}  // namespace gq
