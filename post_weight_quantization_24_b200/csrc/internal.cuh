// Declarations shared between the library's translation units.
#pragma once

#include <mutex>

#include "common.cuh"

namespace gq {

// The library's second stream on the current device and the events that order it with the
// caller's stream (created on first use; one set per device). Hold side_streams_mutex() while
// enqueuing work that uses them.
struct SideStreams {
    cudaStream_t side = nullptr;
    cudaEvent_t fork = nullptr, trsm = nullptr, rest = nullptr, join = nullptr;
    cudaEvent_t aux1 = nullptr, aux2 = nullptr;
};
std::mutex& side_streams_mutex();
gptq_status side_streams(SideStreams** out);

// Per-call device state at the head of the quantizer workspace (zeroed at the start of a call).
struct DevState {
    int status;        // first error code recorded by any kernel (0 = none)
    int pad;
    double lam;        // damping term percdamp * mean(diag H)
    double diag_sum;
    double err_sq;     // sum of e^2 over all columns = tr(D H_d D^T) (OBS increments)
    double delta_sq;   // ||W - What||_F^2
    double loss_den;   // tr(W H W^T)
};

constexpr int kCholBlock = 128;   // panel width of the blocked Cholesky / triangular inverse
// From this width on, the factorisation applies its trailing and inverse updates once per
// outer panel of kOuterCols columns (K = 512, accumulated in 128-deep chunks) instead of once
// per 128 columns: a quarter of the passes over the d x d matrices. Measured crossover: at
// d = 8192 the 128-column scheme is still faster (6.2 against 6.4 ms), at d = 11008 the outer
// panels are (10.3 against 11.7 ms).
#ifndef GPTQ_OUTER_MIN_D
#define GPTQ_OUTER_MIN_D 9216
#endif
constexpr int kOuterMinD = GPTQ_OUTER_MIN_D;
constexpr int kOuterCols = 512;
// Width of the factorisation's split panels (the scratch F is 4 x d x this many floats).
inline int factor_panel_cols(int d) { return d >= kOuterMinD ? kOuterCols : kCholBlock; }
constexpr int kSuperCols = 512;   // columns whose errors are collected before the far update

// rtn.cu
gptq_status rtn_launch(const void* W, int w_dtype, int d_out, int d_in, int bits,
                       int group_size, int sym, uint8_t* out, uint16_t* scales, uint16_t* zeros,
                       cudaStream_t s);

// hessian.cu
gptq_status hessian_launch(float* H, int d, const void* X, int64_t n, int unit_tokens,
                           int* status, cudaStream_t s);
gptq_status mirror_upper_launch(const float* H, float* out, int d, cudaStream_t s);

// factor.cu
gptq_status diag_stats_launch(const float* H, int d, double percdamp, DevState* st,
                              cudaStream_t s);
gptq_status act_order_launch(const float* H, int d, int act_order, int* perm, int* invperm,
                             cudaStream_t s);
// reversed = 1: A[i][j] = Hsym[perm[d-1-i]][perm[d-1-j]] + lambda*delta_ij (damped, reversed)
// reversed = 0: A[i][j] = Hsym[perm[i]][perm[j]] (undamped)
gptq_status gather_h_launch(const float* H, int d, const int* perm, const DevState* st,
                            int reversed, float* A, int* status, cudaStream_t s);
gptq_status gather_w_launch(const void* W, int w_dtype, int d_out, int d_in, const int* perm,
                            float* Wk, int* status, cudaStream_t s);
// In-place lower Cholesky factor L of A (lda = d), the inverses of its diagonal blocks in Dinv
// (ceil(d/nb) blocks of nb x nb, row-major, zero above the diagonal), and U = reverse(L^-1) in
// X. F is scratch of 4 x d x factor_panel_cols(d) floats (the tf32 hi/lo parts of one panel of
// L and of one panel of rows of L^-1). Uses a second stream of its own, forked from and joined back to s.
gptq_status factor_inverse_launch(float* A, int d, float* Dinv, float* X, float* F, int* status,
                                  cudaStream_t s);
// Test switch: the diagonal-block kernel waits on a barrier nothing arrives at (bounded).
gptq_status factor_stall_set(int on);

// gptq.cu
// Per-row images of U's diagonal blocks for the column loop: img [d x 128],
// img[R][k] = U[R][R+1+k] inside R's block of block_size columns (else 0); rdiag[R] = 1/U[R][R].
gptq_status column_images_launch(const float* U, int d, int block_size, float* img, float* rdiag,
                                 cudaStream_t s);
// The column loop of the block [j0, j0+bw), with img/rdiag as column_images_launch writes them.
// sym: symmetric quantizer. preset_perm != nullptr: the grids are preset in scales/zeros and
// processing position p uses grid preset_perm[p] / group_size (else each group's grid is found
// at its first column and written there).
gptq_status gptq_block_launch(float* Wk, int d_out, int d_in, int j0, int bw, const float* img,
                              const float* rdiag, int group_size, int bits, int sym,
                              const int* preset_perm, uint8_t* codes_p, uint16_t* scales,
                              uint16_t* zeros, float* Err, float* ErrLo, int err_ld,
                              double* err_sq, int* status, cudaStream_t s);
// Preset grids of the original weights: scales/zeros [d_out x d_in/group_size]
gptq_status group_grid_launch(const void* W, int w_dtype, int d_out, int d_in, int group_size,
                              int bits, int sym, uint16_t* scales, uint16_t* zeros,
                              cudaStream_t s);
// W[:, c0:c1] -= Err[:, 0:k1-k0] * U[k0:k1, c0:c1], both operands given as tf32 hi/lo parts
gptq_status lazy_update_launch(float* Wk, int d_out, int d_in, int k0, int k1, int c0, int c1,
                               const float* U_hi, const float* U_lo, const float* Err_hi,
                               const float* Err_lo, int err_ld, const int* status,
                               cudaStream_t s, int max_ctas = 0);
// CTAs of one column-loop launch for d_out rows
int gptq_rows_ctas(int d_out);
gptq_status assemble_launch(const uint8_t* codes_p, int d_out, int d_in, const int* perm,
                            const int* invperm, int group_size, int act_order, int preset,
                            uint8_t* codes, int32_t* g_idx, int32_t* perm_out, cudaStream_t s);
gptq_status loss_launch(const void* W, int w_dtype, int d_out, int d_in, const float* H,
                        const int* perm, const uint8_t* codes_p, const uint16_t* scales,
                        const uint16_t* zeros, int group_size, int preset, float* Wk, float* Hp,
                        DevState* st, cudaStream_t s);

}  // namespace gq
