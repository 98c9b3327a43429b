// fp32-accurate GEMM on the tensor cores: tcgen05.mma kind::tf32 with operand splitting.
// Used for the lazy batch update, the loss denominator and the Cholesky / triangular-inverse
// updates. See tcgemm.cu.
#pragma once

#include "common.cuh"

namespace gq {

enum { TC_EPI_STORE = 0, TC_EPI_DOT = 1 };

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
};

// split_a / split_b: represent that operand as hi + lo tf32 parts (an operand that is already
// exactly representable in tf32, e.g. fp16 data, needs no split). Requirements: lda, ldb, ldc,
// ldd multiples of 4; A, B 16-byte aligned; N a multiple of 4.
gptq_status tcgemm_launch(const TcGemmArgs& a, bool b_kmajor, int epi, bool split_a, bool split_b,
                          cudaStream_t s);

}  // namespace gq
