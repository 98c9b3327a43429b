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
#include <atomic>
#include <mutex>

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
    // the Cholesky reads only the lower triangle of the reversed matrix: skip tiles above it
    if (reversed && blockIdx.y < blockIdx.x) return;
    const int j = blockIdx.x * 32 + threadIdx.x;
    if (j >= d) return;
    const int b = reversed ? perm[d - 1 - j] : perm[j];
    const double lam = reversed ? st->lam : 0.0;
    int bad = 0;
    for (int k = threadIdx.y; k < 32; k += blockDim.y) {
        const int i = blockIdx.y * 32 + k;
        if (i >= d) break;
        if (reversed && i < j) continue;
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
    int bad = 0;
    for (int r = blockIdx.x; r < d_out; r += gridDim.x) {
        const T* wr = W + static_cast<int64_t>(r) * d_in;
        float* out = Wk + static_cast<int64_t>(r) * d_in;
        for (int p = threadIdx.x; p < d_in; p += blockDim.x) {
            const float v = static_cast<float>(wr[perm[p]]);
            if (!isfinite(v)) bad = 1;
            out[p] = v;
        }
    }
    if (bad) set_status(status, GPTQ_ERR_NONFINITE);
}

gptq_status gather_w_launch(const void* W, int w_dtype, int d_out, int d_in, const int* perm,
                            float* Wk, int* status, cudaStream_t s) {
    const int blocks = std::min(d_out, num_sms() * 16);
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
// ---- diagonal block: one CTA of 384 threads factors the 128 x 128 block A[k0:, k0:] and
// inverts its factor, blocked in four sub-panels of 32 columns (right-looking):
//   for k = 0..3 (b = 32k), three phases separated by block barriers:
//     A(k)  warp 0 factors L_kk = chol(A_kk), 32 steps in registers, while other warps run
//           the block products that are ready: the rest of the previous sub-panel's trailing
//           update and the inverse's partial sums W_ij += L_im X_mj
//     B(k)  one thread per row below solves L_rk = A_rk L_kk^-T (forward substitution),
//           and one more warp forms I_kk = L_kk^-1 (one column per lane)
//     C(k)  the trailing update of block column k+1 (what A(k+1) and B(k+1) read) and the
//           inverse blocks that I_kk completes, X_kj = -I_kk W_kj
// so the inverse X = L^-1 (block forward substitution, accumulated right-looking) is done
// with the factorisation. In the factor warp, lane i holds row i of A_kk. At step c the pivot
// a_cc is broadcast by shuffle, lane i forms L[i][c] = a_ic / sqrt(a_cc), publishes it in row c
// of LkT (L_kk transposed, the exchange buffer), and applies the rank-1 update a_im -= L[i][c]
// L[m][c] to its row. Lane c+1 computes the next pivot before the exchange, so the chain from
// one pivot to the next is a reciprocal square root, two multiply-adds and one shuffle.
// A 32 x 32 block product is one warp's (4 x 8 register tiles) in phase A, where it runs
// beside the factor warp, and four warps' (8 rows each) in phase C, where it is on the chain.
// Dinv is written block by block as blocks become final (the blocks above the diagonal, all
// zero, first); L itself is not written back: nothing reads the diagonal block afterwards.
// Rows and columns beyond the matrix edge are padded with the identity.
namespace pd {
constexpr int NB = 128, SB = 32, NSB = NB / SB, THREADS = 384;
constexpr int LD = NB + 4;          // row stride (floats) of S, X and LT: 16-byte rows, and
                                    // consecutive rows start four banks apart
constexpr int KLD = SB + 4;         // row stride of LkT
// S [NB][LD]: the block, overwritten by L; X [NB][LD]: L^-1 (its blocks below the diagonal
// hold the partial sums W until they are final); LT [SB][LD]: the current sub-panel's L_rk,
// transposed; LkT [SB][KLD]: L_kk transposed; rinv [SB]: 1 / L_cc; then the stall-test mbarrier
constexpr int SMEM_FLOATS = 2 * NB * LD + SB * LD + SB * KLD + SB;
constexpr int SMEM = SMEM_FLOATS * 4 + 16;
constexpr long long STALL_LIMIT_CYCLES = 2000000;   // about 1 ms
}  // namespace pd

// Test switch for the bounded-wait path (set by gptq_test_stall_factor, passed to each launch):
// when nonzero, every thread of the diagonal-block kernel first waits on an mbarrier that
// nothing arrives at. The wait gives up after STALL_LIMIT_CYCLES, the kernel records
// GPTQ_ERR_TIMEOUT and returns, and the rest of the factorisation skips its work on the status
// word. No copy or MMA is in flight when it gives up.
static std::atomic<int> g_factor_stall{0};

// 1/sqrt(x): the hardware estimate refined by one Newton-Raphson step r' = r (1 + (1 - x r^2)/2)
__device__ __forceinline__ float rsqrt_nr(float x) {
    float r;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    const float e = fmaf(-(x * r), r, 1.0f);
    return fmaf(0.5f * r, e, r);
}

// One warp: L_kk of the 32 x 32 block at S[b:, b:], written back into S (zeros above the
// diagonal) and, transposed, into LkT; rinv[c] = 1 / L_cc. Returns true on a pivot that is
// not a positive normal number. Each row c of LkT is written once (at step c) and read after
// the step's __syncwarp, so it is also the exchange buffer.
__device__ __forceinline__ bool potrf32_warp(float* S, float* LkT, float* rinv, int b, int lane) {
    constexpr unsigned FULL = 0xffffffffu;
    float dr[pd::SB];
    const float4* src = reinterpret_cast<const float4*>(S + (b + lane) * pd::LD + b);
#pragma unroll
    for (int q = 0; q < pd::SB / 4; ++q) {
        const float4 v = src[q];
        dr[4 * q] = v.x; dr[4 * q + 1] = v.y; dr[4 * q + 2] = v.z; dr[4 * q + 3] = v.w;
    }
    bool bad = false;
    float p = __shfl_sync(FULL, dr[0], 0);
#pragma unroll
    for (int c = 0; c < pd::SB; ++c) {
        bad = bad || !(p >= 1.17549435e-38f && p <= 3.40282347e38f);
        const float r = rsqrt_nr(p);                       // 1 / L_cc
        const float l = (lane >= c) ? dr[c] * r : 0.0f;     // L[lane][c]
        dr[c] = l;
        float* lk = LkT + c * pd::KLD;
        lk[lane] = l;
        if (lane == 0) rinv[c] = r;
        if (c + 1 == pd::SB) break;
        p = __shfl_sync(FULL, fmaf(-l, l, dr[c + 1]), c + 1);
        __syncwarp();
#pragma unroll
        for (int m4 = (c + 1) & ~3; m4 < pd::SB; m4 += 4) {
            const float4 v = *reinterpret_cast<const float4*>(lk + m4);   // L[m4 .. m4+3][c]
            const float lv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (m4 + u > c) dr[m4 + u] = fmaf(-l, lv[u], dr[m4 + u]);
        }
    }
    float4* dst = reinterpret_cast<float4*>(S + (b + lane) * pd::LD + b);
#pragma unroll
    for (int q = 0; q < pd::SB / 4; ++q)
        dst[q] = make_float4(dr[4 * q], dr[4 * q + 1], dr[4 * q + 2], dr[4 * q + 3]);
    return bad;
}

// One thread: v[0..31] <- v L_kk^-T in place (solve x L_kk^T = v by forward substitution:
// x_c = v_c / L_cc, then v_m -= x_c L[m][c] for m > c), with L_kk from LkT and rinv.
__device__ __forceinline__ void trsv32(float (&v)[pd::SB], const float* LkT, const float* rinv) {
#pragma unroll
    for (int c = 0; c < pd::SB; ++c) {
        const float x = v[c] * rinv[c];
        v[c] = x;
        const float* lk = LkT + c * pd::KLD;
#pragma unroll
        for (int m4 = (c + 1) & ~3; m4 < pd::SB; m4 += 4) {
            const float4 q = *reinterpret_cast<const float4*>(lk + m4);
            const float lv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (m4 + u > c) v[m4 + u] = fmaf(-x, lv[u], v[m4 + u]);
        }
    }
}

// One warp, H x 8 rows of a 32 x 32 block (H = 4: the whole block): acc[h][q] = sum_m
// P[ti + 8h][m] Q[m][col(q)], m < 32, with ti = lane / 4, tj = lane % 4, col(q) = 4 tj + q
// (q < 4) and 16 + 4 tj + q - 4 (q >= 4). P and Q are row-major with 16-byte rows; a P load is
// shared by the four lanes of a row group, a Q load by the eight lanes of a column group.
template <int H>
__device__ __forceinline__ void block_mma32(const float* P, int ldp, const float* Q, int ldq,
                                            int lane, float (&acc)[H][8]) {
    const int ti = lane >> 2, tj = lane & 3;
#pragma unroll
    for (int h = 0; h < H; ++h)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[h][q] = 0.0f;
#pragma unroll 2
    for (int m4 = 0; m4 < pd::SB; m4 += 4) {
        float a[H][4];
#pragma unroll
        for (int h = 0; h < H; ++h) {
            const float4 v = *reinterpret_cast<const float4*>(P + (ti + 8 * h) * ldp + m4);
            a[h][0] = v.x; a[h][1] = v.y; a[h][2] = v.z; a[h][3] = v.w;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float* qr = Q + (m4 + u) * ldq + 4 * tj;
            const float4 q0 = *reinterpret_cast<const float4*>(qr);
            const float4 q1 = *reinterpret_cast<const float4*>(qr + 16);
            const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int h = 0; h < H; ++h)
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[h][q] = fmaf(a[h][u], qv[q], acc[h][q]);
        }
    }
}

// The H x 8 tile of block_mma32 in a row-major block C: op(C[r][c], acc) for each entry.
template <int H, typename Op>
__device__ __forceinline__ void block_tile_apply(float* C, int ldc, int lane,
                                                 const float (&acc)[H][8], Op op) {
    const int ti = lane >> 2, tj = lane & 3;
#pragma unroll
    for (int h = 0; h < H; ++h)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float4* o = reinterpret_cast<float4*>(C + (ti + 8 * h) * ldc + 16 * half + 4 * tj);
            float4 v = *o;
            v.x = op(v.x, acc[h][4 * half]);
            v.y = op(v.y, acc[h][4 * half + 1]);
            v.z = op(v.z, acc[h][4 * half + 2]);
            v.w = op(v.w, acc[h][4 * half + 3]);
            *o = v;
        }
}

// Block-product tasks of phases A(k) and C(k), one warp each, coded kind << 6 | i << 4 |
// j << 2 | m:
//   U  S_ij -= L_im L_jm^T   (trailing update with sub-panel m, its L_rm transposed in LT)
//   W  X_ij += L_im X_mj     (inverse partial sum)
//   F  X_ij = -X_ii X_ij     (inverse block final; also stored to Dinv)
namespace pt {
constexpr int U = 0, W = 1, F = 2;
constexpr unsigned char T(int kind, int i, int j, int m) {
    return static_cast<unsigned char>(kind << 6 | i << 4 | j << 2 | m);
}
}  // namespace pt
__constant__ unsigned char c_tasks[26] = {
    // C(0): block column 1 of sub-panel 0's update
    pt::T(pt::U, 1, 1, 0), pt::T(pt::U, 2, 1, 0), pt::T(pt::U, 3, 1, 0),
    // A(1): the rest of sub-panel 0's update; W_i0 += L_i0 X_00
    pt::T(pt::U, 2, 2, 0), pt::T(pt::U, 3, 2, 0), pt::T(pt::U, 3, 3, 0),
    pt::T(pt::W, 1, 0, 0), pt::T(pt::W, 2, 0, 0), pt::T(pt::W, 3, 0, 0),
    // C(1): block column 2 of sub-panel 1's update; X_10
    pt::T(pt::U, 2, 2, 1), pt::T(pt::U, 3, 2, 1), pt::T(pt::F, 1, 0, 0),
    // A(2): the rest of sub-panel 1's update; W_i1 += L_i1 X_11, W_i0 += L_i1 X_10
    pt::T(pt::U, 3, 3, 1), pt::T(pt::W, 2, 1, 1), pt::T(pt::W, 3, 1, 1),
    pt::T(pt::W, 2, 0, 1), pt::T(pt::W, 3, 0, 1),
    // C(2): block column 3 of sub-panel 2's update; X_20, X_21
    pt::T(pt::U, 3, 3, 2), pt::T(pt::F, 2, 0, 0), pt::T(pt::F, 2, 1, 0),
    // A(3): W_3j += L_32 X_2j
    pt::T(pt::W, 3, 0, 2), pt::T(pt::W, 3, 1, 2), pt::T(pt::W, 3, 2, 2),
    // C(3): X_30, X_31, X_32
    pt::T(pt::F, 3, 0, 0), pt::T(pt::F, 3, 1, 0), pt::T(pt::F, 3, 2, 0)};
// tasks of phase p (A(k) = 2k, C(k) = 2k + 1): c_tasks[c_task_off[p] .. c_task_off[p + 1])
__constant__ unsigned char c_task_off[9] = {0, 0, 3, 9, 12, 17, 20, 23, 26};

// Rows r0 + ti + 8h (h < H) of the 32 x 32 block (i, j) of X into Dinv, zero past the edge;
// lane tile as in block_mma32
template <int H>
__device__ __forceinline__ void dinv_store_tile(float* Dinv, int i, int j, int r0, int nbc,
                                                int lane, const float (&v)[H][8]) {
    const int ti = lane >> 2, tj = lane & 3;
#pragma unroll
    for (int h = 0; h < H; ++h) {
        const int r = pd::SB * i + r0 + ti + 8 * h;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int c = pd::SB * j + 16 * half + 4 * tj;
            const bool ok = r < nbc;
            *reinterpret_cast<float4*>(Dinv + r * pd::NB + c) = make_float4(
                ok && c < nbc ? v[h][4 * half] : 0.f, ok && c + 1 < nbc ? v[h][4 * half + 1] : 0.f,
                ok && c + 2 < nbc ? v[h][4 * half + 2] : 0.f,
                ok && c + 3 < nbc ? v[h][4 * half + 3] : 0.f);
        }
    }
}

// Named barrier for the `count` threads (whole warps) of one task.
__device__ __forceinline__ void bar_sync_named(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// One task of c_tasks, shared by 4 / H warps: this warp (part `part`) takes rows
// 8 H part .. 8 H (part + 1) - 1 of the block. bar_id names the barrier of the task's warps
// (an F task reads all of W_ij before any part of X_ij is written).
template <int H>
__device__ __forceinline__ void run_task(unsigned char t, float* S, float* X, const float* LT,
                                         float* Dinv, int nbc, int lane, int part, int bar_id) {
    const int kind = t >> 6, i = (t >> 4) & 3, j = (t >> 2) & 3, m = t & 3;
    const int r0 = 8 * H * part;
    float acc[H][8];
    if (kind == pt::U) {
        block_mma32<H>(S + (pd::SB * i + r0) * pd::LD + pd::SB * m, pd::LD,
                       LT + (pd::SB * j - pd::SB * m - pd::SB), pd::LD, lane, acc);
        block_tile_apply<H>(S + (pd::SB * i + r0) * pd::LD + pd::SB * j, pd::LD, lane, acc,
                            [](float c, float a) { return c - a; });
    } else if (kind == pt::W) {
        block_mma32<H>(S + (pd::SB * i + r0) * pd::LD + pd::SB * m, pd::LD,
                       X + (pd::SB * m) * pd::LD + pd::SB * j, pd::LD, lane, acc);
        block_tile_apply<H>(X + (pd::SB * i + r0) * pd::LD + pd::SB * j, pd::LD, lane, acc,
                            [](float c, float a) { return c + a; });
    } else {
        block_mma32<H>(X + (pd::SB * i + r0) * pd::LD + pd::SB * i, pd::LD,
                       X + (pd::SB * i) * pd::LD + pd::SB * j, pd::LD, lane, acc);
        if (H == 4) __syncwarp();         // every lane has read W_ij before it is overwritten
        else bar_sync_named(bar_id, 32 * (4 / H));
#pragma unroll
        for (int h = 0; h < H; ++h)
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[h][q] = -acc[h][q];
        block_tile_apply<H>(X + (pd::SB * i + r0) * pd::LD + pd::SB * j, pd::LD, lane, acc,
                            [](float, float a) { return a; });
        dinv_store_tile<H>(Dinv, i, j, r0, nbc, lane, acc);
    }
}

// The two task shapes, out of line (each phase runs one of them once per warp)
__device__ __noinline__ void run_task_whole(unsigned char t, float* S, float* X, const float* LT,
                                            float* Dinv, int nbc, int lane) {
    run_task<4>(t, S, X, LT, Dinv, nbc, lane, 0, 0);
}
__device__ __noinline__ void run_task_quarter(unsigned char t, float* S, float* X,
                                              const float* LT, float* Dinv, int nbc, int lane,
                                              int part, int bar_id) {
    run_task<1>(t, S, X, LT, Dinv, nbc, lane, part, bar_id);
}

__global__ void __launch_bounds__(pd::THREADS, 1) potrf_diag_kernel(const float* __restrict__ A,
                                                                   int d, int k0, int nbc,
                                                                   float* __restrict__ Dinv,
                                                                   int* status, int stall) {
    extern __shared__ __align__(16) float sm[];
    float* S = sm;                            // [NB][LD]
    float* X = S + pd::NB * pd::LD;           // [NB][LD]
    float* LT = X + pd::NB * pd::LD;          // [SB][LD]
    float* LkT = LT + pd::SB * pd::LD;        // [SB][KLD]
    float* rinv = LkT + pd::SB * pd::KLD;     // [SB]
    uint64_t* mb = reinterpret_cast<uint64_t*>(rinv + pd::SB);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // Before the wait on the previous kernel (none of this reads what it writes): X = 0, the
    // identity in S's rows from nbc on, zeros in S's chunks above the diagonal, and Dinv's six
    // blocks above the block diagonal (zero)
    for (int e = tid; e < pd::NB * (pd::NB / 4); e += pd::THREADS) {
        const int r = e >> 5, c4 = (e & 31) * 4;
        if (r >= nbc || c4 > r) {
            const bool eye = r >= nbc && (r >> 2) == (c4 >> 2);
            const int u = r & 3;
            *reinterpret_cast<float4*>(S + r * pd::LD + c4) =
                make_float4(eye && u == 0 ? 1.f : 0.f, eye && u == 1 ? 1.f : 0.f,
                            eye && u == 2 ? 1.f : 0.f, eye && u == 3 ? 1.f : 0.f);
        }
        *reinterpret_cast<float4*>(X + r * pd::LD + c4) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int e = tid; e < 6 * pd::SB * (pd::SB / 4); e += pd::THREADS) {
        const int blk = e >> 8, row = (e >> 3) & 31, c4 = (e & 7) * 4;
        const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
        const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
        *reinterpret_cast<float4*>(Dinv + (pd::SB * bi + row) * pd::NB + pd::SB * bj + c4) =
            make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (tid == 0) {
        mbar_init(mb, 1);
        fence_mbar_init();
    }

    pdl_wait();
    // the block's lower triangle, rows below nbc: 16-byte async copies of the chunks that
    // reach it
    for (int e = tid; e < pd::NB * (pd::NB / 4); e += pd::THREADS) {
        const int r = e >> 5, c4 = (e & 31) * 4;
        if (r < nbc && c4 <= r)
            cp_async16(S + r * pd::LD + c4, A + static_cast<int64_t>(k0 + r) * d + k0 + c4);
    }
    cp_async_commit();
    const bool skip = status_bad(status);     // read while the copies are in flight
    cp_async_wait<0>();
    if (__syncthreads_or(skip)) return;
    // the copied diagonal chunks also brought up to three entries above the diagonal
    if (tid < nbc)
        for (int c = tid + 1; c <= (tid | 3); ++c) S[tid * pd::LD + c] = 0.0f;
    __syncthreads();
    if (stall) {
        const bool ok = mbar_wait_cycles(mb, 0, pd::STALL_LIMIT_CYCLES);
        if (!ok && tid == 0) set_status(status, GPTQ_ERR_TIMEOUT);
        if (__syncthreads_or(!ok)) return;
    }

    bool bad = false;
#pragma unroll 1
    for (int k = 0; k < pd::NSB; ++k) {
        const int b = k * pd::SB;
        // A(k): the factor warp, and the block products that are ready
        if (warp == 0) {
            bad = potrf32_warp(S, LkT, rinv, b, lane) || bad;
        } else {
            const int t = c_task_off[2 * k] + warp - 1;
            if (t < c_task_off[2 * k + 1]) run_task_whole(c_tasks[t], S, X, LT, Dinv, nbc, lane);
        }
        __syncthreads();
        // B(k): solve (warps 1 .. nrb, one row each lane) and I_kk (the next warp)
        const int nrb = pd::NSB - 1 - k;
        float v[pd::SB];
        if (warp >= 1 && warp <= nrb) {
            const int r = b + pd::SB * warp + lane;
            float4* row = reinterpret_cast<float4*>(S + r * pd::LD + b);
#pragma unroll
            for (int q = 0; q < pd::SB / 4; ++q) {
                const float4 t = row[q];
                v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
            }
            trsv32(v, LkT, rinv);
#pragma unroll
            for (int q = 0; q < pd::SB / 4; ++q)
                row[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
#pragma unroll
            for (int c = 0; c < pd::SB; ++c) LT[c * pd::LD + (r - b - pd::SB)] = v[c];
        } else if (warp == nrb + 1) {
            // column `lane` of I_kk: solve L_kk y = e_lane; as rows, y^T = e_lane^T L_kk^-T
#pragma unroll
            for (int m = 0; m < pd::SB; ++m) v[m] = (m == lane) ? 1.0f : 0.0f;
            trsv32(v, LkT, rinv);
            const bool colok = b + lane < nbc;
#pragma unroll
            for (int c = 0; c < pd::SB; ++c) {
                X[(b + c) * pd::LD + b + lane] = v[c];
                Dinv[(b + c) * pd::NB + b + lane] = (colok && b + c < nbc) ? v[c] : 0.0f;
            }
        }
        __syncthreads();
        // C(k): block column k+1 of the update, and the inverse blocks I_kk completes; four
        // warps per task (these products are on the chain)
        {
            const int t = c_task_off[2 * k + 1] + (warp >> 2);
            if (t < c_task_off[2 * k + 2])
                run_task_quarter(c_tasks[t], S, X, LT, Dinv, nbc, lane, warp & 3, 1 + (warp >> 2));
        }
        __syncthreads();
    }
    if (__syncthreads_or(bad) && tid == 0) set_status(status, GPTQ_ERR_NOT_PD);
}

static int g_potrf_smem = 0;

gptq_status factor_stall_set(int on) {
    g_factor_stall.store(on ? 1 : 0);
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

// ---------------------------------------------------------------------------------------
// factor and inverse on two streams
// ---------------------------------------------------------------------------------------
// Per device: a second stream and the events that order the two streams. The enqueue of one
// factorisation holds the mutex, so the events are never recorded by two sequences at once.
namespace {
constexpr int kMaxDevices = 64;
SideStreams g_side[kMaxDevices];
std::mutex g_side_mu;
}  // namespace

std::mutex& side_streams_mutex() { return g_side_mu; }

gptq_status side_streams(SideStreams** out) {
    int dev = 0;
    GPTQ_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return GPTQ_ERR_UNSUPPORTED;
    SideStreams& ss = g_side[dev];
    if (!ss.side) {
        GPTQ_CUDA_TRY(cudaStreamCreateWithFlags(&ss.side, cudaStreamNonBlocking));
        for (cudaEvent_t* e : {&ss.fork, &ss.trsm, &ss.rest, &ss.join, &ss.aux1, &ss.aux2})
            GPTQ_CUDA_TRY(cudaEventCreateWithFlags(e, cudaEventDisableTiming));
    }
    *out = &ss;
    return GPTQ_OK;
}

#ifndef GPTQ_FACTOR_RESERVE_DIV
#define GPTQ_FACTOR_RESERVE_DIV 16  // at most sms / this many SMs kept free for the main stream
#endif

// Blocked right-looking Cholesky of A with one step of lookahead, and the blocked triangular
// inverse X = L^-1, then U = reverse(X).
//
// Main stream, panel m (columns k0 .. e-1, e = k0 + nbc; rem = d - e rows below):
//   diag(m)   Dinv_m = L11^-1 (one CTA factors the diagonal block; L11 itself is not kept)
//   trsm(m)   L21 = A21 Dinv_m^T, in place (each output tile is the input tile it reads)
//   next(m)   the trailing update of panel m+1's columns only: A[e:, e:e+128] -= L21 L21^T
// Side stream, after trsm(m):
//   split(m)  L21 into tf32 hi and lo parts (Lhi, Llo: rows of 128)
//   rest(m)   the rest of the trailing update: A[e+128:, e+128:] -= L21' L21'^T (lower tiles)
//   inv(m)    X[k0:e, 0:e] = Dinv_m X[k0:e, 0:e] (in place), split into Thi/Tlo, then
//             X[e:, 0:e] -= L21 X[k0:e, 0:e]
// next(m) waits for rest(m-1), the only other writer of its columns; diag(m+1) and trsm(m+1)
// need only next(m), so the side stream's work overlaps them. The side stream's GEMMs (the
// bulk of the flops) take operands split once per panel and run without converter warps;
// the main stream's chain stays as short as it can be.
// The side stream gets most of the GPU: its GEMMs leave as many SMs free as the main stream's
// kernels of the next panel have CTAs, but at most a sixteenth of the GPU (measured: 13.5
// against 17.1 ms at d = 11008 and 174 against 270 ms at d = 28672 when half the GPU was kept
// free; no change at d = 4096).
gptq_status factor_inverse_launch(float* A, int d, float* Dinv, float* X, float* F, int* status,
                                  cudaStream_t s) {
    const int nb = kCholBlock;
    static_assert(kCholBlock == pd::NB, "diagonal-block kernel is written for 128-wide panels");
    const int smem = pd::SMEM;
    if (g_potrf_smem != smem) {
        GPTQ_CUDA_TRY(cudaFuncSetAttribute(potrf_diag_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
        g_potrf_smem = smem;
    }
    std::lock_guard<std::mutex> lock(g_side_mu);
    SideStreams* ss = nullptr;
    GPTQ_TRY(side_streams(&ss));
    cudaStream_t t2 = ss->side;
    const int sms = num_sms();
    // F: L21's hi and lo parts (d x 128 each, indexed by row), then T hi and lo (128 x d each)
    float* Lhi = F;
    float* Llo = F + static_cast<int64_t>(d) * nb;
    float* Thi = F + 2 * static_cast<int64_t>(d) * nb;
    float* Tlo = Thi + static_cast<int64_t>(d) * nb;

    GPTQ_CUDA_TRY(cudaEventRecord(ss->fork, s));
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(t2, ss->fork, 0));
    // Everything below is enqueued on both streams; on an error the side stream is joined
    // back before returning, so a capture of `s` stays well formed.
    auto body = [&]() -> gptq_status {
        GPTQ_CUDA_TRY(cudaMemsetAsync(X, 0, static_cast<size_t>(d) * d * 4, t2));
        set_identity_kernel<<<(d + 255) / 256, 256, 0, t2>>>(X, d);
        GPTQ_LAUNCHED();
        const int nbl = (d + nb - 1) / nb;
        for (int m = 0; m < nbl; ++m) {
            const int k0 = m * nb, nbc = std::min(nb, d - k0), e = k0 + nbc, rem = d - e;
            float* Dm = Dinv + static_cast<int64_t>(m) * nb * nb;
            float* A21 = A + static_cast<int64_t>(e) * d + k0;
            float* L21hi = Lhi + static_cast<int64_t>(e) * nb;
            float* L21lo = Llo + static_cast<int64_t>(e) * nb;
            // SMs kept free for the main stream while this panel's side work runs: diag(m+1)
            // takes one, trsm(m+1) and next(m+1) one per 128 rows below panel m+1
            const int reserve =
                std::min(sms / GPTQ_FACTOR_RESERVE_DIV, std::max(1, (rem + nb - 1) / nb));
            const int side_ctas = std::max(1, sms - reserve);
            GPTQ_CUDA_TRY(launch_pdl(potrf_diag_kernel, dim3(1), dim3(pd::THREADS), smem, s,
                                     static_cast<const float*>(A), d, k0, nbc, Dm, status,
                                     g_factor_stall.load()));
            GPTQ_LAUNCHED();
            if (rem > 0) {
                TcGemmArgs t{};  // A21 = A21 * Dinv_m^T
                t.M = rem; t.N = nbc; t.K = nbc; t.alpha = 1.f; t.beta = 0.f;
                t.A = A21; t.lda = d; t.B = Dm; t.ldb = nb; t.C = A21; t.ldc = d;
                t.status = status;
                GPTQ_TRY(tcgemm_launch(t, true, TC_EPI_STORE, true, true, s));
                GPTQ_CUDA_TRY(cudaEventRecord(ss->trsm, s));
                // next(m) after rest(m-1): the event's last record is still rest(m-1)'s
                if (m > 0) GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, ss->rest, 0));
                TcGemmArgs u{};  // A[e:, e:e+128] -= A21 A21[0:128]^T
                u.M = rem; u.N = std::min(nb, rem); u.K = nbc; u.alpha = -1.f; u.beta = 1.f;
                u.A = A21; u.lda = d; u.B = A21; u.ldb = d;
                u.C = A + static_cast<int64_t>(e) * d + e; u.ldc = d;
                u.lower_only = 1; u.status = status;
                GPTQ_TRY(tcgemm_launch(u, true, TC_EPI_STORE, true, true, s));
                GPTQ_CUDA_TRY(cudaStreamWaitEvent(t2, ss->trsm, 0));
                // (the previous panel's readers of Lhi/Llo ran earlier on this stream)
                GPTQ_TRY(tcgemm_split_launch(A21, L21hi, L21lo, rem, nbc, d, false, t2, nb, nb));
                if (rem > nb) {
                    const float* Lrhi = L21hi + static_cast<int64_t>(nb) * nb;
                    const float* Lrlo = L21lo + static_cast<int64_t>(nb) * nb;
                    TcGemmArgs r{};  // A[e+128:, e+128:] -= A21' A21'^T (lower tiles)
                    r.M = rem - nb; r.N = rem - nb; r.K = nbc; r.alpha = -1.f; r.beta = 1.f;
                    r.A = Lrhi; r.lda = nb; r.A_lo = Lrlo;
                    r.B = Lrhi; r.ldb = nb; r.B_lo = Lrlo;
                    r.C = A + static_cast<int64_t>(e + nb) * d + (e + nb); r.ldc = d;
                    r.lower_only = 1; r.status = status; r.max_ctas = side_ctas;
                    GPTQ_TRY(tcgemm_presplit_launch(r, t2, true));
                }
                GPTQ_CUDA_TRY(cudaEventRecord(ss->rest, t2));
            } else {
                GPTQ_CUDA_TRY(cudaEventRecord(ss->trsm, s));
                GPTQ_CUDA_TRY(cudaStreamWaitEvent(t2, ss->trsm, 0));
            }
            float* Xk = X + static_cast<int64_t>(k0) * d;
            TcGemmArgs v{};  // X[k0:e, 0:e] = Dinv_m * X[k0:e, 0:e], in place
            v.M = nbc; v.N = e; v.K = nbc; v.alpha = 1.f; v.beta = 0.f;
            v.A = Dm; v.lda = nb; v.B = Xk; v.ldb = d; v.C = Xk; v.ldc = d;
            v.status = status; v.max_ctas = side_ctas;
            GPTQ_TRY(tcgemm_launch(v, false, TC_EPI_STORE, true, true, t2));
            if (rem > 0) {
                GPTQ_TRY(tcgemm_split_launch(Xk, Thi, Tlo, nbc, e, d, false, t2));
                TcGemmArgs w{};  // X[e:, 0:e] -= L21 * X[k0:e, 0:e]
                w.M = rem; w.N = e; w.K = nbc; w.alpha = -1.f; w.beta = 1.f;
                w.A = L21hi; w.lda = nb; w.A_lo = L21lo;
                w.B = Thi; w.ldb = d; w.B_lo = Tlo;
                w.C = X + static_cast<int64_t>(e) * d; w.ldc = d;
                w.status = status; w.max_ctas = side_ctas;
                GPTQ_TRY(tcgemm_presplit_launch(w, t2, false));
            }
        }
        const int64_t half = static_cast<int64_t>(d) * d / 2;
        const int blocks =
            static_cast<int>(std::min<int64_t>((half + 255) / 256, num_sms() * 16));
        reverse_inplace_kernel<<<blocks, 256, 0, t2>>>(X, half);
        GPTQ_LAUNCHED();
        return GPTQ_OK;
    };
    // Wide layers: outer panels of kOuterCols columns. The main stream factors a panel's
    // columns in 128-wide steps, each step's solve updating only the panel's own later columns;
    // once per panel it updates the next panel's columns (K = 512) after the previous panel's
    // rest. The second stream splits the panel's L once and applies the rest of the trailing
    // update and the inverse's bulk update with K = 512 (a quarter of the passes over the
    // d x d matrices); the inverse's rows of the panel itself are done in 128-wide steps.
    auto body_outer = [&]() -> gptq_status {
        const int op = kOuterCols;
        float* Phi = F;
        float* Plo = F + static_cast<int64_t>(d) * op;
        float* Thi = F + 2 * static_cast<int64_t>(d) * op;
        float* Tlo = F + 3 * static_cast<int64_t>(d) * op;
        GPTQ_CUDA_TRY(cudaMemsetAsync(X, 0, static_cast<size_t>(d) * d * 4, t2));
        set_identity_kernel<<<(d + 255) / 256, 256, 0, t2>>>(X, d);
        GPTQ_LAUNCHED();
        for (int K0 = 0; K0 < d; K0 += op) {
            const int E = std::min(K0 + op, d), wP = E - K0, remP = d - E;
            const int reserve =
                std::min(sms / GPTQ_FACTOR_RESERVE_DIV, std::max(1, (remP + nb - 1) / nb));
            const int side_ctas = std::max(1, sms - reserve);
            // ---- main: the panel's columns in 128-wide steps ----
            for (int k0 = K0; k0 < E; k0 += nb) {
                const int m = k0 / nb, nbc = std::min(nb, d - k0), e = k0 + nbc, rem = d - e;
                float* Dm = Dinv + static_cast<int64_t>(m) * nb * nb;
                float* A21 = A + static_cast<int64_t>(e) * d + k0;
                GPTQ_CUDA_TRY(launch_pdl(potrf_diag_kernel, dim3(1), dim3(pd::THREADS), smem, s,
                                         static_cast<const float*>(A), d, k0, nbc, Dm, status,
                                         g_factor_stall.load()));
                GPTQ_LAUNCHED();
                if (rem == 0) continue;
                TcGemmArgs t{};  // A21 = A21 * Dinv_m^T
                t.M = rem; t.N = nbc; t.K = nbc; t.alpha = 1.f; t.beta = 0.f;
                t.A = A21; t.lda = d; t.B = Dm; t.ldb = nb; t.C = A21; t.ldc = d;
                t.status = status;
                GPTQ_TRY(tcgemm_launch(t, true, TC_EPI_STORE, true, true, s));
                if (E > e) {
                    TcGemmArgs u{};  // the panel's own later columns: A[e:, e:E] -= A21 A21[0:E-e]^T
                    u.M = rem; u.N = E - e; u.K = nbc; u.alpha = -1.f; u.beta = 1.f;
                    u.A = A21; u.lda = d; u.B = A21; u.ldb = d;
                    u.C = A + static_cast<int64_t>(e) * d + e; u.ldc = d;
                    u.lower_only = 1; u.status = status;
                    GPTQ_TRY(tcgemm_launch(u, true, TC_EPI_STORE, true, true, s));
                }
            }
            GPTQ_CUDA_TRY(cudaEventRecord(ss->trsm, s));      // the panel's L is complete
            const float* Lp = A + static_cast<int64_t>(E) * d + K0;   // L[E:, K0:E]
            if (remP > 0) {
                const int E2 = std::min(E + op, d);
                // the next panel's columns, after the previous panel's rest (their other writer)
                if (K0 > 0) GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, ss->rest, 0));
                TcGemmArgs u{};  // A[E:, E:E2] -= L[E:, K0:E] L[E:E2, K0:E]^T
                u.M = remP; u.N = E2 - E; u.K = wP; u.alpha = -1.f; u.beta = 1.f;
                u.A = Lp; u.lda = d; u.B = Lp; u.ldb = d;
                u.C = A + static_cast<int64_t>(E) * d + E; u.ldc = d;
                u.lower_only = 1; u.status = status;
                GPTQ_TRY(tcgemm_launch(u, true, TC_EPI_STORE, true, true, s));
            }
            // ---- side: split the panel, the rest of the trailing update, the inverse ----
            GPTQ_CUDA_TRY(cudaStreamWaitEvent(t2, ss->trsm, 0));
            if (remP > 0) {
                const int E2 = std::min(E + op, d);
                float* Ph = Phi + static_cast<int64_t>(E) * op;   // rows E.. of the panel
                float* Pl = Plo + static_cast<int64_t>(E) * op;
                GPTQ_TRY(tcgemm_split_launch(Lp, Ph, Pl, remP, wP, d, false, t2, op, op));
                if (E2 < d) {
                    const int64_t off = static_cast<int64_t>(E2 - E) * op;
                    TcGemmArgs r{};  // A[E2:, E2:] -= L[E2:, K0:E] L[E2:, K0:E]^T (lower tiles)
                    r.M = d - E2; r.N = d - E2; r.K = wP; r.alpha = -1.f; r.beta = 1.f;
                    r.A = Ph + off; r.lda = op; r.A_lo = Pl + off;
                    r.B = Ph + off; r.ldb = op; r.B_lo = Pl + off;
                    r.C = A + static_cast<int64_t>(E2) * d + E2; r.ldc = d;
                    r.lower_only = 1; r.status = status; r.max_ctas = side_ctas;
                    GPTQ_TRY(tcgemm_presplit_launch(r, t2, true));
                }
            }
            GPTQ_CUDA_TRY(cudaEventRecord(ss->rest, t2));
            for (int k0 = K0; k0 < E; k0 += nb) {
                const int m = k0 / nb, nbc = std::min(nb, d - k0), e = k0 + nbc;
                float* Dm = Dinv + static_cast<int64_t>(m) * nb * nb;
                float* Xk = X + static_cast<int64_t>(k0) * d;
                TcGemmArgs v{};  // X[k0:e, 0:e] = Dinv_m * X[k0:e, 0:e], in place
                v.M = nbc; v.N = e; v.K = nbc; v.alpha = 1.f; v.beta = 0.f;
                v.A = Dm; v.lda = nb; v.B = Xk; v.ldb = d; v.C = Xk; v.ldc = d;
                v.status = status; v.max_ctas = side_ctas;
                GPTQ_TRY(tcgemm_launch(v, false, TC_EPI_STORE, true, true, t2));
                if (E > e) {
                    TcGemmArgs w{};  // X[e:E, 0:e] -= L[e:E, k0:e] * X[k0:e, 0:e]
                    w.M = E - e; w.N = e; w.K = nbc; w.alpha = -1.f; w.beta = 1.f;
                    w.A = A + static_cast<int64_t>(e) * d + k0; w.lda = d;
                    w.B = Xk; w.ldb = d; w.C = X + static_cast<int64_t>(e) * d; w.ldc = d;
                    w.status = status; w.max_ctas = side_ctas;
                    GPTQ_TRY(tcgemm_launch(w, false, TC_EPI_STORE, true, true, t2));
                }
            }
            if (remP > 0) {
                float* XP = X + static_cast<int64_t>(K0) * d;      // X[K0:E, 0:E]
                GPTQ_TRY(tcgemm_split_launch(XP, Thi, Tlo, wP, E, d, false, t2));
                TcGemmArgs w{};  // X[E:, 0:E] -= L[E:, K0:E] * X[K0:E, 0:E]
                w.M = remP; w.N = E; w.K = wP; w.alpha = -1.f; w.beta = 1.f;
                w.A = Phi + static_cast<int64_t>(E) * op; w.lda = op;
                w.A_lo = Plo + static_cast<int64_t>(E) * op;
                w.B = Thi; w.ldb = d; w.B_lo = Tlo;
                w.C = X + static_cast<int64_t>(E) * d; w.ldc = d;
                w.status = status; w.max_ctas = side_ctas;
                GPTQ_TRY(tcgemm_presplit_launch(w, t2, false));
            }
        }
        const int64_t half = static_cast<int64_t>(d) * d / 2;
        const int blocks =
            static_cast<int>(std::min<int64_t>((half + 255) / 256, num_sms() * 16));
        reverse_inplace_kernel<<<blocks, 256, 0, t2>>>(X, half);
        GPTQ_LAUNCHED();
        return GPTQ_OK;
    };
    const gptq_status rc = d >= kOuterMinD ? body_outer() : body();
    const cudaError_t e1 = cudaEventRecord(ss->join, t2);
    const cudaError_t e2 = cudaStreamWaitEvent(s, ss->join, 0);
    if (rc != GPTQ_OK) return rc;
    if (e1 != cudaSuccess || e2 != cudaSuccess) return GPTQ_ERR_CUDA;
    return GPTQ_OK;
}

}  // namespace gq
