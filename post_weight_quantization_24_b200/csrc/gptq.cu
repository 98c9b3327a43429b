// GPTQ column loop, lazy batch update, output assembly and reconstruction loss.
//
// GPTQ deep-dive (hncyxsy.com/news/243429):
//   §2.2  quantizing column q moves the not-yet-quantized columns by
//         delta = -(w_q - quant(w_q)) / [H_F^-1]_qq * (H_F^-1)_{q,.}; with U^T U = H_d^-1 the
//         same update reads  e = (w_q - What_q) / U_qq,  w_c -= e * U_qc  for c > q;
//   §2.4  fixed column order; lazy batch updates: errors of a block are accumulated and the
//         later columns are updated once per block (a GEMM);
//   §3.1  step 3: per block of 128 columns, column by column: pick the scale, round, record
//         the error; then update the remaining columns.
// gtnt.cn/news/115337 §4: block_size is a multiple of group_size, so groups never straddle
// blocks. Rows of W are independent given U, which is what the kernels parallelise over.
#include <algorithm>

#include "internal.cuh"
#include "quant.cuh"
#include "sgemm.cuh"
#include "tcgemm.cuh"

namespace gq {

namespace gb {
constexpr int MAXB = 128;            // widest block handled in one launch
constexpr int LANES_PER_ROW = 16;    // 8 columns per lane, two rows per warp
constexpr int WARPS = 8;
constexpr int THREADS = WARPS * 32;
constexpr int SMEM = (MAXB * MAXB + MAXB) * 4;
}  // namespace gb

// In-block column loop. The block's U[j0:j0+bw, j0:j0+bw] (zero below the diagonal) and the
// reciprocals of its diagonal sit in shared memory. Each half-warp owns one row and holds its
// bw (<= 128) block weights in registers, 8 per lane. Column i is owned by lane i/8: it is
// broadcast with a shuffle, every lane of the row computes the same code and error, and each
// lane applies the rank-1 update to its 8 columns with one row of U (entries left of column
// i are zero, so no masking is needed). Group scale/zero come from a half-warp min/max
// reduction over the group's current weights at the group's first column.
__global__ void __launch_bounds__(gb::THREADS) gptq_block_kernel(
    float* __restrict__ Wk, int d_out, int d_in, int j0, int bw, const float* __restrict__ U,
    int g, int bits, uint8_t* __restrict__ codes_p, uint16_t* __restrict__ scales,
    uint16_t* __restrict__ zeros, float* __restrict__ Err, int err_ld, double* err_sq,
    const int* status) {
    if (status_bad(status)) return;
    extern __shared__ float smem[];
    float* Us = smem;                      // [MAXB][MAXB]
    float* dinv = smem + gb::MAXB * gb::MAXB;
    const int maxq = (1 << bits) - 1;
    const int n_groups_row = d_in / g;

    for (int e = threadIdx.x; e < gb::MAXB * gb::MAXB / 4; e += blockDim.x) {
        const int i = e / (gb::MAXB / 4), c4 = (e % (gb::MAXB / 4)) * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < bw && c4 < bw) {
            v = *reinterpret_cast<const float4*>(U + static_cast<int64_t>(j0 + i) * d_in + j0 + c4);
            if (c4 + 0 < i) v.x = 0.f;
            if (c4 + 1 < i) v.y = 0.f;
            if (c4 + 2 < i) v.z = 0.f;
            if (c4 + 3 < i) v.w = 0.f;
        }
        *reinterpret_cast<float4*>(Us + i * gb::MAXB + c4) = v;
    }
    for (int i = threadIdx.x; i < gb::MAXB; i += blockDim.x)
        dinv[i] = i < bw ? 1.0f / U[static_cast<int64_t>(j0 + i) * d_in + j0 + i] : 0.0f;
    __syncthreads();

    const int lane = lane_id(), half = lane >> 4, hl = lane & 15;
    const int c0 = hl * 8;                           // this lane's first block column
    const unsigned full = 0xffffffffu;
    const int warps_total = gridDim.x * gb::WARPS;
    const int n_pairs = (d_out + 1) / 2;
    double esq = 0.0;   // this lane's sum of squared errors (its own columns)
    for (int pair = blockIdx.x * gb::WARPS + warp_id(); pair < n_pairs; pair += warps_total) {
        const int r = pair * 2 + half;
        const bool row_ok = r < d_out;
        float w[8];
        float* wrow = Wk + static_cast<int64_t>(r) * d_in + j0;
        if (row_ok && c0 < bw) {
            const float4 a = *reinterpret_cast<const float4*>(wrow + c0);
            const float4 b = *reinterpret_cast<const float4*>(wrow + c0 + 4);
            w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
            w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) w[k] = 0.f;
        }
        float e[8];
        uint32_t qlo = 0, qhi = 0;
        QParams P;
        P.scale = 1.f; P.zero = 0.f; P.inv_scale = 1.f;
#pragma unroll 1
        for (int i0 = 0; i0 < bw; i0 += 8) {
            const int owner = (half << 4) | (i0 >> 3);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int i = i0 + c;
                if (i >= bw) break;
                if ((j0 + i) % g == 0) {
                    // group [i, i+g) of the block: min/max of its current weights in this row
                    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int col = c0 + k;
                        if (col >= i && col < i + g && col < bw) {
                            mn = fminf(mn, w[k]);
                            mx = fmaxf(mx, w[k]);
                        }
                    }
#pragma unroll
                    for (int off = 8; off > 0; off >>= 1) {
                        mn = fminf(mn, __shfl_xor_sync(full, mn, off));
                        mx = fmaxf(mx, __shfl_xor_sync(full, mx, off));
                    }
                    P = group_params(mn, mx, maxq);
                    if (hl == 0 && row_ok) {
                        const int64_t gi = static_cast<int64_t>(r) * n_groups_row + (j0 + i) / g;
                        scales[gi] = half_bits(P.scale);
                        zeros[gi] = half_bits(P.zero);
                    }
                }
                const float wi = __shfl_sync(full, w[c], owner);
                const int qi = quant_code(wi, P, maxq);
                const float err = (wi - dequant(qi, P)) * dinv[i];
                if (hl == (i0 >> 3)) {
                    e[c] = err;
                    if (c < 4) qlo |= static_cast<uint32_t>(qi) << (8 * c);
                    else qhi |= static_cast<uint32_t>(qi) << (8 * (c - 4));
                }
                const float4 u0 = *reinterpret_cast<const float4*>(Us + i * gb::MAXB + c0);
                const float4 u1 = *reinterpret_cast<const float4*>(Us + i * gb::MAXB + c0 + 4);
                w[0] = fmaf(-err, u0.x, w[0]);
                w[1] = fmaf(-err, u0.y, w[1]);
                w[2] = fmaf(-err, u0.z, w[2]);
                w[3] = fmaf(-err, u0.w, w[3]);
                w[4] = fmaf(-err, u1.x, w[4]);
                w[5] = fmaf(-err, u1.y, w[5]);
                w[6] = fmaf(-err, u1.z, w[6]);
                w[7] = fmaf(-err, u1.w, w[7]);
            }
        }
        if (row_ok && c0 < bw) {
            uint2 qv;
            qv.x = qlo;
            qv.y = qhi;
            *reinterpret_cast<uint2*>(codes_p + static_cast<int64_t>(r) * d_in + j0 + c0) = qv;
            float* er = Err + static_cast<int64_t>(r) * err_ld + c0;
            *reinterpret_cast<float4*>(er) = make_float4(e[0], e[1], e[2], e[3]);
            *reinterpret_cast<float4*>(er + 4) = make_float4(e[4], e[5], e[6], e[7]);
            float part = 0.0f;
#pragma unroll
            for (int k = 0; k < 8; ++k) part = fmaf(e[k], e[k], part);
            esq += static_cast<double>(part);
        }
    }
    // the OBS increments e^2 add up to tr(D H_d D^T) for the whole layer
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) esq += __shfl_xor_sync(full, esq, off);
    if (lane == 0 && esq != 0.0) atomicAdd(err_sq, esq);
}

// ---------------------------------------------------------------------------------------
// Row-resident column loop (group sizes that are a multiple of 4).
//
// One thread owns one row of the block and keeps its (up to 128) block weights in registers,
// so quantizing a column is done once per row, with no cross-lane traffic; U sits in shared
// memory and every lane reads the same U entries (broadcast loads). The column loop runs in
// chunks of 4 columns: at the start of the chunk that begins at block column i0, register
// w[c] holds block column i0 + c. Step k of the chunk quantizes w[k] and applies
// w[c] -= err * U[i0+k][i0+c] to the columns c > k; the last step writes each result four
// registers lower, so the window moves by 4 columns per chunk without copies and every
// register index stays a compile-time constant. A chunk's entries of U start at column i0, a
// multiple of 4, so they are read as aligned float4. The register window shrinks in phases
// of 16 columns (W = 128, 112, ..., 16): a chunk in phase p only touches w[0..W).
// Group starts fall on chunk starts (group_size % 4 == 0, blocks start on group starts).
// ---------------------------------------------------------------------------------------
namespace gr {
constexpr int MAXB = 128;                    // widest block handled in one launch
constexpr int LD = MAXB + 16;                // shared row stride of U (floats), zero padded
constexpr int PH = 16;                       // block columns per window phase
constexpr int NPH = MAXB / PH;
constexpr int WARPS = 2;
constexpr int THREADS = WARPS * 32;          // one row per thread
constexpr int SMEM = MAXB * LD * 4 + WARPS * MAXB * 4 + NPH * 8;
}  // namespace gr

struct RowCtx {
    const float* Us;      // [MAXB][LD]: Us[i][c] = U[j0+i][j0+c] for i, c < bw, else 0 (c >= bw)
    const float* dinv;    // this warp's copy of 1 / U[j0+i][j0+i]
    int bw, g, maxq, j0, d_in, n_groups_row, err_ld;
    bool row_ok;
    int64_t r;
    uint8_t* codes_p;
    uint16_t* scales;
    uint16_t* zeros;
    float* Err;
    QParams P;
    int next_gs;          // block column of the next group start
    double esq;           // this row's sum of squared OBS errors
};

template <int W>
__device__ __forceinline__ void rows_phase(float (&w)[gr::MAXB], int p0, RowCtx& x) {
    const int i_end = min(p0 + gr::PH, x.bw);
#pragma unroll 1
    for (int i0 = p0; i0 < i_end; i0 += 4) {
        if (i0 == x.next_gs) {
            // group [i0, i0+g): min/max of its current weights, w[0..g)
            x.next_gs += x.g;
            float mn = w[0], mx = w[0];
#pragma unroll
            for (int c4 = 0; c4 < W; c4 += 4) {
                if (c4 >= x.g) break;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    mn = fminf(mn, w[c4 + t]);
                    mx = fmaxf(mx, w[c4 + t]);
                }
            }
            x.P = group_params(mn, mx, x.maxq);
            if (x.row_ok) {
                const int64_t gi = x.r * x.n_groups_row + (x.j0 + i0) / x.g;
                x.scales[gi] = half_bits(x.P.scale);
                x.zeros[gi] = half_bits(x.P.zero);
            }
        }
        const float4 dv = *reinterpret_cast<const float4*>(x.dinv + i0);
        const float dk[4] = {dv.x, dv.y, dv.z, dv.w};
        float e[4];
        uint32_t qword = 0u;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float wi = w[k];
            const int qi = quant_code(wi, x.P, x.maxq);
            const float err = (wi - dequant(qi, x.P)) * dk[k];
            e[k] = err;
            qword |= static_cast<uint32_t>(qi) << (8 * k);
            const float* urow = x.Us + (i0 + k) * gr::LD + i0;
            if (k < 3) {
#pragma unroll
                for (int c4 = 0; c4 < W; c4 += 4) {
                    const float4 u = *reinterpret_cast<const float4*>(urow + c4);
                    const float uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int t = 0; t < 4; ++t)
                        if (c4 + t > k) w[c4 + t] = fmaf(-err, uu[t], w[c4 + t]);
                }
            } else {
#pragma unroll
                for (int c4 = 4; c4 < W; c4 += 4) {
                    const float4 u = *reinterpret_cast<const float4*>(urow + c4);
                    const float uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) w[c4 - 4 + t] = fmaf(-err, uu[t], w[c4 + t]);
                }
#pragma unroll
                for (int t = 0; t < 4; ++t) w[W - 4 + t] = 0.0f;
            }
        }
        if (x.row_ok) {
            *reinterpret_cast<float4*>(x.Err + x.r * x.err_ld + i0) =
                make_float4(e[0], e[1], e[2], e[3]);
            *reinterpret_cast<uint32_t*>(x.codes_p + x.r * x.d_in + x.j0 + i0) = qword;
        }
        float part = e[0] * e[0];
        part = fmaf(e[1], e[1], part);
        part = fmaf(e[2], e[2], part);
        part = fmaf(e[3], e[3], part);
        x.esq += static_cast<double>(part);
    }
}

// Waits for phase P's rows of U, derives their 1/U_ii, runs the phase, then the next one.
// Returns false if a wait ran out of its cycle limit.
template <int P>
__device__ __forceinline__ bool rows_phases(float (&w)[gr::MAXB], RowCtx& x, uint64_t* bars,
                                            float* dinv, int lane) {
    if constexpr (P < gr::NPH) {
        const int p0 = P * gr::PH;
        if (p0 >= x.bw) return true;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[P], 0));
        if (!ok) return false;
        if (lane < gr::PH) {
            const int i = p0 + lane;
            dinv[i] = i < x.bw ? 1.0f / x.Us[i * gr::LD + i] : 0.0f;
        }
        __syncwarp();
        rows_phase<gr::MAXB - P * gr::PH>(w, p0, x);
        return rows_phases<P + 1>(w, x, bars, dinv, lane);
    }
    return true;
}

__global__ void __launch_bounds__(gr::THREADS, 3) gptq_rows_kernel(
    const float* __restrict__ Wk, int d_out, int d_in, int j0, int bw, const float* __restrict__ U,
    int g, int bits, uint8_t* __restrict__ codes_p, uint16_t* __restrict__ scales,
    uint16_t* __restrict__ zeros, float* __restrict__ Err, int err_ld, double* err_sq,
    int* status) {
    if (status_bad(status)) return;
    extern __shared__ __align__(128) unsigned char rows_smem[];
    float* Us = reinterpret_cast<float*>(rows_smem);
    float* dinv_all = Us + gr::MAXB * gr::LD;
    uint64_t* bars = reinterpret_cast<uint64_t*>(dinv_all + gr::WARPS * gr::MAXB);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // zero the pad columns [bw, LD) of the rows in use; the bulk copies fill [0, bw)
    const int pad = gr::LD - bw;
    for (int e = tid; e < bw * pad; e += gr::THREADS) Us[(e / pad) * gr::LD + bw + e % pad] = 0.f;
    if (tid == 0) {
        for (int p = 0; p < gr::NPH; ++p) mbar_init(&bars[p], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == 0) {
        // rows [16p, 16p+16) of U's diagonal block arrive on barrier p
        if (lane < gr::NPH) {
            const int rows = min(max(bw - lane * gr::PH, 0), gr::PH);
            if (rows > 0) mbar_arrive_expect_tx(&bars[lane], static_cast<uint32_t>(rows * bw * 4));
        }
        __syncwarp();
        for (int i = lane; i < bw; i += 32)
            bulk_load_1d(Us + i * gr::LD, U + static_cast<int64_t>(j0 + i) * d_in + j0,
                         static_cast<uint32_t>(bw * 4), &bars[i / gr::PH]);
    }

    RowCtx x;
    x.Us = Us;
    x.dinv = dinv_all + warp * gr::MAXB;
    x.bw = bw; x.g = g; x.maxq = (1 << bits) - 1; x.j0 = j0; x.d_in = d_in;
    x.n_groups_row = d_in / g; x.err_ld = err_ld;
    x.r = static_cast<int64_t>(blockIdx.x) * gr::THREADS + tid;
    x.row_ok = x.r < d_out;
    x.codes_p = codes_p; x.scales = scales; x.zeros = zeros; x.Err = Err;
    x.P.scale = 1.f; x.P.zero = 0.f; x.P.inv_scale = 1.f;
    x.next_gs = 0;   // j0 is a multiple of g
    x.esq = 0.0;

    float w[gr::MAXB];
    const float* wrow = Wk + x.r * d_in + j0;
#pragma unroll
    for (int c4 = 0; c4 < gr::MAXB; c4 += 4) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (x.row_ok && c4 < bw) a = *reinterpret_cast<const float4*>(wrow + c4);
        w[c4] = a.x; w[c4 + 1] = a.y; w[c4 + 2] = a.z; w[c4 + 3] = a.w;
    }

    if (!rows_phases<0>(w, x, bars, dinv_all + warp * gr::MAXB, lane)) {
        set_status(status, GPTQ_ERR_TIMEOUT);
        // let the copies still in flight land before the block exits (bounded again)
        if (warp == 0 && lane < gr::NPH && lane * gr::PH < bw) mbar_wait(&bars[lane], 0);
        __syncwarp();
        return;
    }
    // the OBS increments e^2 add up to tr(D H_d D^T) for the whole layer
    double esq = x.esq;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) esq += __shfl_xor_sync(0xffffffffu, esq, off);
    if (lane == 0 && esq != 0.0) atomicAdd(err_sq, esq);
}

static bool g_rows_attr_set = false;

static bool g_block_attr_set = false;

gptq_status gptq_block_launch(float* Wk, int d_out, int d_in, int j0, int bw, const float* U,
                              int group_size, int bits, uint8_t* codes_p, uint16_t* scales,
                              uint16_t* zeros, float* Err, int err_ld, double* err_sq,
                              int* status, cudaStream_t s) {
    if (group_size % 4 == 0) {
        if (!g_rows_attr_set) {
            GPTQ_CUDA_TRY(cudaFuncSetAttribute(gptq_rows_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               gr::SMEM));
            g_rows_attr_set = true;
        }
        const int grid = (d_out + gr::THREADS - 1) / gr::THREADS;
        gptq_rows_kernel<<<grid, gr::THREADS, gr::SMEM, s>>>(Wk, d_out, d_in, j0, bw, U,
                                                            group_size, bits, codes_p, scales,
                                                            zeros, Err, err_ld, err_sq, status);
        GPTQ_LAUNCHED();
        return GPTQ_OK;
    }
    if (!g_block_attr_set) {
        GPTQ_CUDA_TRY(cudaFuncSetAttribute(gptq_block_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, gb::SMEM));
        g_block_attr_set = true;
    }
    const int n_pairs = (d_out + 1) / 2;
    const int need = (n_pairs + gb::WARPS - 1) / gb::WARPS;
    const int grid = std::max(1, std::min(need, num_sms() * 3));
    gptq_block_kernel<<<grid, gb::THREADS, gb::SMEM, s>>>(Wk, d_out, d_in, j0, bw, U, group_size,
                                                          bits, codes_p, scales, zeros, Err,
                                                          err_ld, err_sq, status);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

// W[:, j1:] -= Err_block * U[j0:j1, j1:]  (3xTF32 on the tensor cores)
gptq_status lazy_update_launch(float* Wk, int d_out, int d_in, int j0, int bw, const float* U,
                               const float* Err, int err_ld, const int* status, cudaStream_t s) {
    const int j1 = j0 + bw;
    if (j1 >= d_in) return GPTQ_OK;
    TcGemmArgs a{};
    a.M = d_out; a.N = d_in - j1; a.K = bw; a.alpha = -1.f; a.beta = 1.f;
    a.A = Err; a.lda = err_ld;
    a.B = U + static_cast<int64_t>(j0) * d_in + j1; a.ldb = d_in;
    a.C = Wk + j1; a.ldc = d_in; a.status = status;
    return tcgemm_launch(a, false, TC_EPI_STORE, true, true, s);
}

// codes[r][c] = codes_p[r][invperm[c]]; g_idx[c] = invperm[c] / g; perm_out = perm
__global__ void assemble_kernel(const uint8_t* __restrict__ codes_p, int d_out, int d_in,
                                const int* __restrict__ perm, const int* __restrict__ invperm,
                                int g, int act_order, uint8_t* __restrict__ codes,
                                int32_t* __restrict__ g_idx, int32_t* __restrict__ perm_out) {
    const int64_t n = static_cast<int64_t>(d_out) * d_in;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (int64_t c = t0; c < d_in; c += stride) {
        g_idx[c] = invperm[c] / g;
        if (perm_out) perm_out[c] = perm[c];
    }
    if (!act_order) return;
    for (int64_t e = t0; e < n; e += stride) {
        const int64_t r = e / d_in;
        const int c = static_cast<int>(e - r * d_in);
        codes[e] = codes_p[r * d_in + invperm[c]];
    }
}

gptq_status assemble_launch(const uint8_t* codes_p, int d_out, int d_in, const int* perm,
                            const int* invperm, int group_size, int act_order, uint8_t* codes,
                            int32_t* g_idx, int32_t* perm_out, cudaStream_t s) {
    const int64_t n = act_order ? static_cast<int64_t>(d_out) * d_in : d_in;
    const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, num_sms() * 16));
    assemble_kernel<<<std::max(blocks, 1), 256, 0, s>>>(codes_p, d_out, d_in, perm, invperm,
                                                       group_size, act_order, codes, g_idx,
                                                       perm_out);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

// sum over the layer of (W[r][perm[p]] - What[r][p])^2, What from codes, scales and zeros
template <typename T>
__global__ void __launch_bounds__(256) delta_sq_kernel(
    const T* __restrict__ W, int d_out, int d_in, const int* __restrict__ perm,
    const uint8_t* __restrict__ codes_p, const uint16_t* __restrict__ scales,
    const uint16_t* __restrict__ zeros, int g, double* out) {
    const int64_t n = static_cast<int64_t>(d_out) * d_in;
    const int ng = d_in / g;
    double acc = 0.0;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = e / d_in;
        const int p = static_cast<int>(e - r * d_in);
        const int64_t gi = r * ng + p / g;
        const float s = __half2float(__ushort_as_half(scales[gi]));
        const float z = __half2float(__ushort_as_half(zeros[gi]));
        const float wh = s * (static_cast<float>(codes_p[e]) - z);
        const float dlt = static_cast<float>(W[r * d_in + perm[p]]) - wh;
        acc += static_cast<double>(dlt) * dlt;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    __shared__ double red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < 8; ++w) t += red[w];
        atomicAdd(out, t);
    }
}

// Reconstruction loss tr(D H D^T) / tr(W H W^T) with the undamped H.
// Numerator: the column loop already summed the OBS increments e^2, whose total is
// tr(D H_d D^T) with H_d = H + lambda*I, so tr(D H D^T) = sum e^2 - lambda*||D||^2 (one pass
// over the outputs). Denominator: tr(W H W^T) as a GEMM (W_p * H_p) whose epilogue dots with
// W_p, in the processing order (a common permutation leaves the trace unchanged).
// sum_{i,j} H[i][j] * G[i][j] / 2 from the upper triangles of two symmetric matrices
// (G = 2 W^T W, as the Hessian kernel writes it), accumulated in fp64
__global__ void __launch_bounds__(256) upper_dot_kernel(const float* __restrict__ H,
                                                        const float* __restrict__ G, int d,
                                                        double* out) {
    double acc = 0.0;
    for (int i = blockIdx.x; i < d; i += gridDim.x) {
        const float* h = H + static_cast<int64_t>(i) * d;
        const float* g = G + static_cast<int64_t>(i) * d;
        for (int c = (i & ~3) + 4 * static_cast<int>(threadIdx.x); c < d; c += 4 * 256) {
            const float4 a = *reinterpret_cast<const float4*>(h + c);
            const float4 b = *reinterpret_cast<const float4*>(g + c);
            const float pa[4] = {a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w};
            float v = 0.0f;
#pragma unroll
            for (int t = 0; t < 4; ++t) v += (c + t > i) ? 2.0f * pa[t] : (c + t == i ? pa[t] : 0.0f);
            acc += static_cast<double>(v);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    __shared__ double red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < 8; ++w) t += red[w];
        atomicAdd(out, 0.5 * t);
    }
}

// The denominator tr(W H W^T) equals <H, W^T W>. For fp16 W, G = 2 W^T W comes from the
// Hessian kernel (W's rows play the tokens; exact fp16 products, fp32 accumulation) into the
// d_in^2 scratch G, followed by one pass over the two upper triangles. fp32 W (not exact in
// fp16) takes the tf32x3 GEMM route: tr(W H W^T) with W and H in the processing order.
gptq_status loss_launch(const void* W, int w_dtype, int d_out, int d_in, const float* H,
                        const int* perm, const uint8_t* codes_p, const uint16_t* scales,
                        const uint16_t* zeros, int group_size, float* Wk, float* Hp,
                        DevState* st, cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(d_out) * d_in;
    const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, num_sms() * 8));
    if (w_dtype == GPTQ_DTYPE_F16)
        delta_sq_kernel<__half><<<blocks, 256, 0, s>>>(static_cast<const __half*>(W), d_out,
                                                       d_in, perm, codes_p, scales, zeros,
                                                       group_size, &st->delta_sq);
    else
        delta_sq_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(W), d_out, d_in,
                                                      perm, codes_p, scales, zeros, group_size,
                                                      &st->delta_sq);
    GPTQ_LAUNCHED();
    if (w_dtype == GPTQ_DTYPE_F16) {
        float* G = Hp;
        GPTQ_CUDA_TRY(cudaMemsetAsync(G, 0, static_cast<size_t>(d_in) * d_in * sizeof(float), s));
        GPTQ_TRY(hessian_launch(G, d_in, W, d_out, 0, &st->status, s));
        const int gb = std::max(1, std::min(d_in, num_sms() * 8));
        upper_dot_kernel<<<gb, 256, 0, s>>>(H, G, d_in, &st->loss_den);
        GPTQ_LAUNCHED();
        return GPTQ_OK;
    }
    GPTQ_TRY(gather_h_launch(H, d_in, perm, st, 0, Hp, &st->status, s));
    GPTQ_TRY(gather_w_launch(W, w_dtype, d_out, d_in, perm, Wk, &st->status, s));
    // Hp is symmetric, so it serves as the K-major [N x K] operand directly
    TcGemmArgs a{};
    a.M = d_out; a.N = d_in; a.K = d_in; a.alpha = 1.f; a.beta = 0.f;
    a.A = Wk; a.lda = d_in; a.B = Hp; a.ldb = d_in; a.D = Wk; a.ldd = d_in;
    a.dot = &st->loss_den; a.status = &st->status;
    return tcgemm_launch(a, true, TC_EPI_DOT, true, true, s);
}

}  // namespace gq
