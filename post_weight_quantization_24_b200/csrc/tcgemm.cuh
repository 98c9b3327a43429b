// fp32-accurate GEMM on the tensor cores: tcgen05.mma kind::tf32 with operand splitting.
// Used for the lazy batch update, the loss denominator and the Cholesky / triangular-inverse
// updates. See tcgemm.cu.
#pragma once

#include "common.cuh"

namespace gq {

enum { TC_EPI_STORE = 0, TC_EPI_DOT = 1 };

// x rounded to tf32 (10 explicit mantissa bits), nearest with ties away from zero
__device__ __forceinline__ float tf32_rna(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

struct TcGemmArgs {
    int M, N, K;
    float alpha, beta;
    const float* A;   // [M x K], row stride lda (K contiguous)
    int lda;
    const float* B;   // b_kmajor ? [N x K] (K contiguous) : [K x N] (N contiguous), stride ldb
    int ldb;
    float* C;         // TC_EPI_STORE: C = alpha*A*B + beta*C, [M x N], stride ldc
    int ldc;
    const float* D;   // TC_EPI_DOT: *dot += alpha * sum(A*B .* D), [M x N], stride ldd
    int ldd;
    double* dot;
    int lower_only;   // skip output tiles entirely above the diagonal
    const int* status;  // optional: skip all work when *status != 0; receives TIMEOUT
    // Pre-split operands (tcgemm_presplit_launch): A and B hold the tf32 hi parts, A_lo and
    // B_lo the lo parts, with the layouts of A and B and the strides lda_lo, ldb_lo (0: lda,
    // ldb).
    const float* A_lo;
    const float* B_lo;
    int lda_lo, ldb_lo;
    int max_ctas;     // > 0: launch at most this many CTAs (leaves SMs to concurrent work)
};

// split_a / split_b: represent that operand as hi + lo tf32 parts (an operand that is already
// exactly representable in tf32, e.g. fp16 data, needs no split). Requirements: lda, ldb, ldc,
// ldd multiples of 4; A, B 16-byte aligned; N a multiple of 4.
gptq_status tcgemm_launch(const TcGemmArgs& a, bool b_kmajor, int epi, bool split_a, bool split_b,
                          cudaStream_t s);

// C = alpha*A*B + beta*C (store epilogue) with both operands already split into tf32 hi and lo
// (hi = tf32_rna(x), lo = tf32_rna(x - hi), as tcgemm_split_launch writes them); B MN-major,
// or K-major with b_kmajor. Operands reused by many tiles are split once instead of in every
// tile, and the kernel runs without converter warps.
gptq_status tcgemm_presplit_launch(const TcGemmArgs& a, cudaStream_t s, bool b_kmajor = false);

// hi[i][j] = tf32_rna(x), lo[i][j] = tf32_rna(x - hi) for x = src[i][j], j0(i) <= j < cols,
// j0(i) = upper ? i & ~3 : 0 (src rows of stride ld, hi and lo rows of strides ld_hi, ld_lo;
// 0 means ld; hi may alias src)
gptq_status tcgemm_split_launch(const float* src, float* hi, float* lo, int rows, int cols, int ld,
                                bool upper, cudaStream_t s, int ld_hi = 0, int ld_lo = 0);

}  // namespace gq
