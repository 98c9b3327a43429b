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
#include "tcgemm.cuh"

namespace gq {

// ---------------------------------------------------------------------------------------
// Column loop, one row per thread.
//
// One thread owns one row of the block and keeps its (up to 128) block weights in registers,
// so each column is quantized once per row, with no cross-lane traffic. Register w[k] holds
// block column i + k while column i is processed: the step quantizes w[0] and applies
// w[c] -= err * U[i][i+c] to the later columns, writing each result one register lower, so
// the window moves by one column per step without copies and every register index stays a
// compile-time constant. The loop body is a single step (a few KB of code, so it stays in
// the instruction cache); the window narrows in phases of 16 columns (W = 128, 112, ..., 16).
// The step reads row i of U starting at column i+1, so the block's U comes as an image whose
// row i is U[i][i+1 ...] (16-byte aligned, zero past the block), brought into shared memory
// by bulk copies, 16 rows per mbarrier, together with the reciprocals of U's diagonal.
// Errors and codes are kept for four columns and stored together.
// ---------------------------------------------------------------------------------------
namespace gr {
constexpr int MAXB = 128;                    // widest block handled in one launch
constexpr int PH = 16;                       // block columns per window phase
constexpr int NPH = MAXB / PH;
#ifndef GPTQ_ROWS_WARPS
#define GPTQ_ROWS_WARPS 2
#endif
constexpr int WARPS = GPTQ_ROWS_WARPS;       // rows (warps of 32) per CTA
constexpr int THREADS = WARPS * 32;          // one row per thread
constexpr int SMEM = MAXB * MAXB * 4 + MAXB * 4 + NPH * 8 + MAXB * 4;   // + grid indices
}  // namespace gr

// img[R][k] = U[R][R+1+k] while R+1+k stays inside R's block (else 0); rdiag[R] = 1/U[R][R]
__global__ void column_images_kernel(const float* __restrict__ U, int d, int bs,
                                     float* __restrict__ img, float* __restrict__ rdiag) {
    const int R = blockIdx.x, k = threadIdx.x;
    const int j0 = (R / bs) * bs, bw = min(bs, d - j0), i = R - j0;
    const float* urow = U + static_cast<int64_t>(R) * d;
    img[static_cast<int64_t>(R) * gr::MAXB + k] = (i + 1 + k < bw) ? urow[R + 1 + k] : 0.0f;
    if (k == 0) rdiag[R] = 1.0f / urow[R];
}

gptq_status column_images_launch(const float* U, int d, int block_size, float* img, float* rdiag,
                                 cudaStream_t s) {
    column_images_kernel<<<d, gr::MAXB, 0, s>>>(U, d, block_size, img, rdiag);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

struct RowCtx {
    const float* Us;      // [MAXB][MAXB]: Us[i][k] = U[j0+i][j0+i+1+k] inside the block, else 0
    const float* rd;      // [MAXB]: 1 / U[j0+i][j0+i]
    int bw, g, maxq, j0, d_in, n_groups_row, err_ld;
    bool row_ok;
    int64_t r;
    uint8_t* codes_p;
    uint16_t* scales;
    uint16_t* zeros;
    float* Err;           // tf32 hi and lo parts of the errors (the lazy update's operand)
    float* ErrLo;
    QParams P;
    int next_gs;          // block column of the next group start (grids found in the loop)
    bool sym;             // symmetric quantizer
    const int* pidx;      // preset grids: grid index of each block column (else nullptr)
    int cur_k;            // preset grids: the grid P holds
    float e0, e1, e2, e3; // errors of the last four columns (e0 newest)
    uint32_t qword;       // their codes, oldest in the low byte
    double esq;           // this row's sum of squared OBS errors
};

template <int W>
__device__ __forceinline__ void rows_phase(float (&w)[gr::MAXB], int p0, RowCtx& x) {
    const int i_end = min(p0 + gr::PH, x.bw);
#pragma unroll 1
    for (int i = p0; i < i_end; ++i) {
        if (x.pidx) {
            // preset grids (per-channel, static groups): this column's grid, from the outputs
            const int k = x.pidx[i];
            if (k != x.cur_k) {
                x.cur_k = k;
                if (x.row_ok) {
                    const int64_t gi = x.r * x.n_groups_row + k;
                    x.P = stored_params(x.scales[gi], x.zeros[gi]);
                }
            }
        } else if (i == x.next_gs) {
            // group [i, i+g): min/max of its current weights, w[0..g)
            x.next_gs += x.g;
            float mn = w[0], mx = w[0];
#pragma unroll
            for (int c4 = 0; c4 < W; c4 += 4) {
                if (c4 >= x.g) break;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    if (c4 + t < x.g) {
                        mn = fminf(mn, w[c4 + t]);
                        mx = fmaxf(mx, w[c4 + t]);
                    }
                }
            }
            x.P = group_params_any(mn, mx, x.maxq, x.sym);
            if (x.row_ok) {
                const int64_t gi = x.r * x.n_groups_row + (x.j0 + i) / x.g;
                x.scales[gi] = half_bits(x.P.scale);
                x.zeros[gi] = half_bits(x.P.zero);
            }
        }
        const float wi = w[0];
        const int qi = quant_code(wi, x.P, x.maxq);
        const float err = (wi - dequant(qi, x.P)) * x.rd[i];
        x.e3 = x.e2; x.e2 = x.e1; x.e1 = x.e0; x.e0 = err;
        x.qword = (x.qword >> 8) | (static_cast<uint32_t>(qi) << 24);
        const float* urow = x.Us + i * gr::MAXB;   // urow[k] = U[i][i+1+k]
#pragma unroll
        for (int k4 = 0; k4 < W; k4 += 4) {
            const float4 u = *reinterpret_cast<const float4*>(urow + k4);
            const float uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int t = 0; t < 4; ++t)
                if (k4 + t + 1 < W) w[k4 + t] = fmaf(-err, uu[t], w[k4 + t + 1]);
        }
        w[W - 1] = 0.0f;
        if ((i & 3) == 3) {
            if (x.row_ok) {
                const float ev[4] = {x.e3, x.e2, x.e1, x.e0};
                float hv[4], lv[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    hv[t] = tf32_rna(ev[t]);
                    lv[t] = tf32_rna(ev[t] - hv[t]);
                }
                *reinterpret_cast<float4*>(x.Err + x.r * x.err_ld + i - 3) =
                    make_float4(hv[0], hv[1], hv[2], hv[3]);
                *reinterpret_cast<float4*>(x.ErrLo + x.r * x.err_ld + i - 3) =
                    make_float4(lv[0], lv[1], lv[2], lv[3]);
                *reinterpret_cast<uint32_t*>(x.codes_p + x.r * x.d_in + x.j0 + i - 3) = x.qword;
            }
            float part = x.e0 * x.e0;
            part = fmaf(x.e1, x.e1, part);
            part = fmaf(x.e2, x.e2, part);
            part = fmaf(x.e3, x.e3, part);
            x.esq += static_cast<double>(part);
        }
    }
}

// Waits for phase P's rows of the image, runs the phase, then the next one. Returns false if
// a wait ran out of its cycle limit.
template <int P>
__device__ __forceinline__ bool rows_phases(float (&w)[gr::MAXB], RowCtx& x, uint64_t* bars) {
    if constexpr (P < gr::NPH) {
        const int p0 = P * gr::PH;
        if (p0 >= x.bw) return true;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[P], 0));
        if (!ok) return false;
        rows_phase<gr::MAXB - P * gr::PH>(w, p0, x);
        return rows_phases<P + 1>(w, x, bars);
    }
    return true;
}

__global__ void __launch_bounds__(gr::THREADS, gr::WARPS <= 2 ? 3 : 2) gptq_rows_kernel(
    const float* __restrict__ Wk, int d_out, int d_in, int j0, int bw,
    const float* __restrict__ img, const float* __restrict__ rdiag, int g, int bits, int sym,
    const int* __restrict__ preset_perm, uint8_t* __restrict__ codes_p,
    uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros, float* __restrict__ Err,
    float* __restrict__ ErrLo, int err_ld, double* err_sq, int* status) {
    pdl_wait();
    if (status_bad(status)) return;
    extern __shared__ __align__(128) unsigned char rows_smem[];
    float* Us = reinterpret_cast<float*>(rows_smem);
    float* rd = Us + gr::MAXB * gr::MAXB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(rd + gr::MAXB);
    int* pidx = reinterpret_cast<int*>(bars + gr::NPH);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (tid == 0) {
        for (int p = 0; p < gr::NPH; ++p) mbar_init(&bars[p], 1);
        fence_mbar_init();
    }
    // preset grids: the grid of block column i is the group of its original column
    if (preset_perm)
        for (int i = tid; i < bw; i += gr::THREADS) pidx[i] = preset_perm[j0 + i] / g;
    __syncthreads();
    if (warp == 0 && lane < gr::NPH) {
        // image rows [16p, 16p+16) of the block arrive on barrier p (+ the diagonal on 0)
        const int p = lane, rows = min(max(bw - p * gr::PH, 0), gr::PH);
        if (rows > 0) {
            const uint32_t bytes = static_cast<uint32_t>(rows * gr::MAXB * 4);
            mbar_arrive_expect_tx(&bars[p], bytes + (p == 0 ? static_cast<uint32_t>(bw * 4) : 0u));
            bulk_load_1d(Us + p * gr::PH * gr::MAXB,
                         img + static_cast<int64_t>(j0 + p * gr::PH) * gr::MAXB, bytes, &bars[p]);
            if (p == 0) bulk_load_1d(rd, rdiag + j0, static_cast<uint32_t>(bw * 4), &bars[0]);
        }
    }

    RowCtx x;
    x.Us = Us;
    x.rd = rd;
    x.bw = bw; x.g = g; x.maxq = (1 << bits) - 1; x.j0 = j0; x.d_in = d_in;
    x.n_groups_row = d_in / g; x.err_ld = err_ld;
    x.r = static_cast<int64_t>(blockIdx.x) * gr::THREADS + tid;
    x.row_ok = x.r < d_out;
    x.codes_p = codes_p; x.scales = scales; x.zeros = zeros; x.Err = Err; x.ErrLo = ErrLo;
    x.P.scale = 1.f; x.P.zero = 0.f; x.P.inv_scale = 1.f;
    x.next_gs = 0;   // j0 is a multiple of g
    x.sym = sym != 0;
    x.pidx = preset_perm ? pidx : nullptr;
    x.cur_k = -1;
    x.e0 = x.e1 = x.e2 = x.e3 = 0.f;
    x.qword = 0u;
    x.esq = 0.0;

    float w[gr::MAXB];
    const float* wrow = Wk + x.r * d_in + j0;
#pragma unroll
    for (int c4 = 0; c4 < gr::MAXB; c4 += 4) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (x.row_ok && c4 < bw) a = *reinterpret_cast<const float4*>(wrow + c4);
        w[c4] = a.x; w[c4 + 1] = a.y; w[c4 + 2] = a.z; w[c4 + 3] = a.w;
    }

    if (!rows_phases<0>(w, x, bars)) {
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

gptq_status gptq_block_launch(float* Wk, int d_out, int d_in, int j0, int bw, const float* img,
                              const float* rdiag, int group_size, int bits, int sym,
                              const int* preset_perm, uint8_t* codes_p, uint16_t* scales,
                              uint16_t* zeros, float* Err, float* ErrLo, int err_ld,
                              double* err_sq, int* status, cudaStream_t s) {
    if (!g_rows_attr_set) {
        GPTQ_CUDA_TRY(cudaFuncSetAttribute(gptq_rows_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           gr::SMEM));
        g_rows_attr_set = true;
    }
    const int grid = (d_out + gr::THREADS - 1) / gr::THREADS;
    GPTQ_CUDA_TRY(launch_pdl(gptq_rows_kernel, dim3(grid), dim3(gr::THREADS), gr::SMEM, s, Wk,
                             d_out, d_in, j0, bw, img, rdiag, group_size, bits, sym, preset_perm,
                             codes_p, scales, zeros, Err, ErrLo, err_ld, err_sq, status));
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

// Preset grids: the scale and zero of every group of the ORIGINAL weights in the original
// column order (static groups; one group per row for per-channel), before any column is
// quantized. One warp per (row, group): lane-strided min/max, a warp reduction, and the
// group's scalars in fp64 as the column loop computes them.
template <typename T>
__global__ void __launch_bounds__(256) group_grid_kernel(const T* __restrict__ W, int d_out,
                                                         int d_in, int g, int bits, int sym,
                                                         uint16_t* __restrict__ scales,
                                                         uint16_t* __restrict__ zeros) {
    const int maxq = (1 << bits) - 1;
    const int ng = d_in / g;
    const int64_t n_units = static_cast<int64_t>(d_out) * ng;
    const int lane = threadIdx.x & 31;
    const int64_t wstride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t u = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         u < n_units; u += wstride) {
        const int64_t r = u / ng;
        const int k = static_cast<int>(u - r * ng);
        const T* w = W + r * d_in + static_cast<int64_t>(k) * g;
        float mn = static_cast<float>(w[0]), mx = mn;
        for (int i = lane; i < g; i += 32) {
            const float v = static_cast<float>(w[i]);
            mn = fminf(mn, v);
            mx = fmaxf(mx, v);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        }
        if (lane == 0) {
            const QParams p = group_params_any(mn, mx, maxq, sym != 0);
            scales[u] = half_bits(p.scale);
            zeros[u] = half_bits(p.zero);
        }
    }
}

gptq_status group_grid_launch(const void* W, int w_dtype, int d_out, int d_in, int group_size,
                              int bits, int sym, uint16_t* scales, uint16_t* zeros,
                              cudaStream_t s) {
    const int64_t units = static_cast<int64_t>(d_out) * (d_in / group_size);
    const int blocks = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>((units + 7) / 8, static_cast<int64_t>(num_sms()) * 16)));
    if (w_dtype == GPTQ_DTYPE_F16)
        group_grid_kernel<__half><<<blocks, 256, 0, s>>>(static_cast<const __half*>(W), d_out,
                                                         d_in, group_size, bits, sym, scales,
                                                         zeros);
    else
        group_grid_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(W), d_out, d_in,
                                                        group_size, bits, sym, scales, zeros);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

// W[:, c0:c1] -= Err[:, 0:k1-k0] * U[k0:k1, c0:c1]  (3xTF32 on the tensor cores, with both
// operands split into tf32 hi/lo once: U after the factorisation, Err by the column loop)
int gptq_rows_ctas(int d_out) { return (d_out + gr::THREADS - 1) / gr::THREADS; }

gptq_status lazy_update_launch(float* Wk, int d_out, int d_in, int k0, int k1, int c0, int c1,
                               const float* U_hi, const float* U_lo, const float* Err_hi,
                               const float* Err_lo, int err_ld, const int* status,
                               cudaStream_t s, int max_ctas) {
    if (c1 <= c0 || k1 <= k0) return GPTQ_OK;
    const int64_t boff = static_cast<int64_t>(k0) * d_in + c0;
    TcGemmArgs a{};
    a.M = d_out; a.N = c1 - c0; a.K = k1 - k0; a.alpha = -1.f; a.beta = 1.f;
    a.A = Err_hi; a.A_lo = Err_lo; a.lda = err_ld;
    a.B = U_hi + boff; a.B_lo = U_lo + boff; a.ldb = d_in;
    a.C = Wk + c0; a.ldc = d_in; a.status = status; a.max_ctas = max_ctas;
    return tcgemm_presplit_launch(a, s);
}

// codes[r][c] = codes_p[r][invperm[c]]; g_idx[c] = invperm[c] / g; perm_out = perm
__global__ void assemble_kernel(const uint8_t* __restrict__ codes_p, int d_out, int d_in,
                                const int* __restrict__ perm, const int* __restrict__ invperm,
                                int g, int act_order, int preset, uint8_t* __restrict__ codes,
                                int32_t* __restrict__ g_idx, int32_t* __restrict__ perm_out) {
    const int t0 = blockIdx.x * blockDim.x + threadIdx.x, stride = gridDim.x * blockDim.x;
    for (int c = t0; c < d_in; c += stride) {
        g_idx[c] = (preset ? c : invperm[c]) / g;
        if (perm_out) perm_out[c] = perm[c];
    }
    if (!act_order) return;
    for (int r = blockIdx.x; r < d_out; r += gridDim.x) {
        const uint8_t* src = codes_p + static_cast<int64_t>(r) * d_in;
        uint8_t* dst = codes + static_cast<int64_t>(r) * d_in;
        for (int c = threadIdx.x; c < d_in; c += blockDim.x) dst[c] = src[invperm[c]];
    }
}

gptq_status assemble_launch(const uint8_t* codes_p, int d_out, int d_in, const int* perm,
                            const int* invperm, int group_size, int act_order, int preset,
                            uint8_t* codes, int32_t* g_idx, int32_t* perm_out, cudaStream_t s) {
    const int blocks = std::max(1, std::min(std::max(d_out, (d_in + 255) / 256), num_sms() * 16));
    assemble_kernel<<<blocks, 256, 0, s>>>(codes_p, d_out, d_in, perm, invperm, group_size,
                                           act_order, preset, codes, g_idx, perm_out);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

// sum over the layer of (W[r][perm[p]] - What[r][p])^2, What from codes, scales and zeros
template <typename T>
__global__ void __launch_bounds__(256) delta_sq_kernel(
    const T* __restrict__ W, int d_out, int d_in, const int* __restrict__ perm,
    const uint8_t* __restrict__ codes_p, const uint16_t* __restrict__ scales,
    const uint16_t* __restrict__ zeros, int g, int preset, double* out) {
    const int ng = d_in / g;
    const float inv_g = 1.0f / static_cast<float>(g);
    double acc = 0.0;
    for (int r = blockIdx.x; r < d_out; r += gridDim.x) {
        const int64_t row = static_cast<int64_t>(r) * d_in;
        float part = 0.0f;
        for (int p = threadIdx.x; p < d_in; p += blockDim.x) {
            // the grid of processing position p: group of p, or with preset grids the group
            // of its original column; the quotient from a float one, corrected by one either
            // way (< 2^17)
            const int c = preset ? perm[p] : p;
            int q = __float2int_rz(static_cast<float>(c) * inv_g);
            if (q * g > c) --q;
            else if ((q + 1) * g <= c) ++q;
            const int64_t gi = static_cast<int64_t>(r) * ng + q;
            const float s = __half2float(__ushort_as_half(scales[gi]));
            const float z = __half2float(__ushort_as_half(zeros[gi]));
            const float wh = s * (static_cast<float>(codes_p[row + p]) - z);
            const float dlt = static_cast<float>(W[row + perm[p]]) - wh;
            part = fmaf(dlt, dlt, part);
        }
        acc += static_cast<double>(part);
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
                        const uint16_t* zeros, int group_size, int preset, float* Wk, float* Hp,
                        DevState* st, cudaStream_t s) {
    const int blocks = std::min(d_out, num_sms() * 8);
    if (w_dtype == GPTQ_DTYPE_F16)
        delta_sq_kernel<__half><<<blocks, 256, 0, s>>>(static_cast<const __half*>(W), d_out,
                                                       d_in, perm, codes_p, scales, zeros,
                                                       group_size, preset, &st->delta_sq);
    else
        delta_sq_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(W), d_out, d_in,
                                                      perm, codes_p, scales, zeros, group_size,
                                                      preset, &st->delta_sq);
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
