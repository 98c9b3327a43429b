// Group RTN with a clip search per group (gtnt.cn/news/115337 §3, awq_clip: search each
// quantization block's clip bound c in [amax * min_ratio, amax], amax = max |w| of the block,
// truncating the weights to [-c, c] before their min-max scale is taken).
//
// For each group and each grid ratio rho_i = 1 - i*step (i = 0 .. n-1), c = rho_i * amax; the
// group's weights are clamped to [-c, c] and quantized with the scale and zero of the clamped
// group (asymmetric min-max, or symmetric); the criterion is the group's share of the layer's
// output error, d H_gg d with d = w - What (original weights minus the reconstruction) and
// H_gg the group's diagonal block of H = 2 X^T X, or the weight error d.d without H. The
// smallest criterion wins; ties go to the larger ratio (less clipping).
//
// Kernel: one CTA per (group, tile of 128 rows), one thread per row. The CTA stages the
// group's weights transposed in shared memory (row stride 129 floats: conflict-free both when
// a row is written and when the threads of a warp read one column) and, with H, the group's
// g x g block of H made symmetric from its upper triangle. Per ratio a thread builds its row's
// errors d[0..g) in registers and accumulates the quadratic form row by row of H_gg (eight
// independent partial sums per row, H read by broadcast). The group scalars and the codes of
// clamped weights are computed in fp64 and the other codes by the exact rounding of quant.cuh,
// so for a given ratio the codes, scales and zeros equal the fp64 definition bit for bit; the
// criterion itself is fp32.
#include <algorithm>
#include <cmath>

#include "internal.cuh"
#include "quant.cuh"

namespace gq {

namespace rc {
constexpr int ROWS = 128;              // rows per CTA, one per thread
constexpr int MAXG = 128;
constexpr int WS = ROWS + 1;           // transposed weight tile row stride
constexpr int MAX_GRID = 64;
}  // namespace rc

// Scale and zero of the range [lo, hi] (fp64), as group_params computes them from a group's
// min and max: asymmetric widens the range to contain 0; symmetric uses max(|lo|, |hi|).
__device__ __forceinline__ QParams range_params(double lo, double hi, int maxq, bool sym) {
    double s, z;
    if (sym) {
        const double m = fmax(fabs(lo), fabs(hi));
        s = (m == 0.0) ? 1.0 : fp16_ceil(2.0 * m / static_cast<double>(maxq));
        z = static_cast<double>((maxq + 1) / 2);
    } else {
        lo = fmin(lo, 0.0);
        hi = fmax(hi, 0.0);
        const double span = hi - lo;
        s = (span == 0.0) ? 1.0 : fp16_ceil(span / static_cast<double>(maxq));
        z = (isinf(s) ? 0.0 : rint_quotient(-lo, s)) + 0.0;
    }
    QParams p;
    p.scale = static_cast<float>(s);
    p.zero = static_cast<float>(z);
    p.inv_scale = __frcp_rn(p.scale);
    return p;
}

// Code of w under the clamp to [-c, c] and the grid p: clamped weights are quantized at +-c
// in fp64 (c is an fp64 value), the others by the exact fp32 rounding of quant_code.
__device__ __noinline__ int clip_code_slow(float w, double c, QParams p, int maxq) {
    const double wd = static_cast<double>(w);
    if (wd > c || wd < -c) {
        const double q = rint((wd > c ? c : -c) / static_cast<double>(p.scale)) +
                         static_cast<double>(p.zero);
        return static_cast<int>(fmin(fmax(q, 0.0), static_cast<double>(maxq)));
    }
    return quant_code(w, p, maxq);
}

// Fast path: |w| below cf (c rounded down to fp32, so w is not clamped) and w/scale clear of
// a rounding boundary by more than the error of its fp32 quotient; otherwise the exact path.
__device__ __forceinline__ int clip_code(float w, double c, float cf, const QParams& p,
                                         int maxq) {
    const float t = w * p.inv_scale;
    const float k = rintf(t);
    if (fabsf(w) < cf && fabsf(t - k) <= 0.5f - fabsf(t) * 3.0e-7f - 1.0e-30f)
        return static_cast<int>(fminf(fmaxf(k + p.zero, 0.0f), static_cast<float>(maxq)));
    return clip_code_slow(w, c, p, maxq);
}

// c = (1 - i*step) * amax with each operation rounded on its own, as the ratio grid is defined
// (a fused multiply-add would round 1 - i*step once and move c; e.g. 1 - 7*0.05 is
// 0.6499999999999999 with two roundings and 0.65 with one)
__device__ __forceinline__ double clip_bound(int i, double step, double amax) {
    return __dmul_rn(__dsub_rn(1.0, __dmul_rn(static_cast<double>(i), step)), amax);
}

template <int G, typename T>
__global__ void __launch_bounds__(rc::ROWS, 1) rtn_clip_kernel(
    const T* __restrict__ W, int d_out, int d_in, int bits, int sym, const float* __restrict__ H,
    int n_grid, double step, uint8_t* __restrict__ out, uint16_t* __restrict__ scales,
    uint16_t* __restrict__ zeros, uint8_t* __restrict__ ratio_idx) {
    extern __shared__ __align__(16) float clip_smem[];
    float* Wt = clip_smem;                    // [G][WS]: Wt[j][t] = W[r0 + t][k0 + j]
    float* Hs = Wt + G * rc::WS;              // [G][G] symmetric block of H (if H)
    const int t = threadIdx.x;
    const int k = blockIdx.x, r0 = blockIdx.y * rc::ROWS;
    const int64_t k0 = static_cast<int64_t>(k) * G;
    const int maxq = (1 << bits) - 1;
    const int ng = d_in / G;

    for (int rr = 0; rr < rc::ROWS; ++rr) {
        const int r = r0 + rr;
        for (int j = t; j < G; j += rc::ROWS)
            Wt[j * rc::WS + rr] = r < d_out ? static_cast<float>(W[static_cast<int64_t>(r) * d_in + k0 + j]) : 0.0f;
    }
    if (H) {
        for (int e = t; e < G * G; e += rc::ROWS) {
            const int i = e / G, j = e % G;
            const int a = min(i, j), b = max(i, j);
            Hs[e] = H[(k0 + a) * d_in + k0 + b];
        }
    }
    __syncthreads();
    const int r = r0 + t;
    if (r >= d_out) return;

    float mn = Wt[t], mx = Wt[t];
#pragma unroll 8
    for (int j = 1; j < G; ++j) {
        mn = fminf(mn, Wt[j * rc::WS + t]);
        mx = fmaxf(mx, Wt[j * rc::WS + t]);
    }
    const double amax = fmax(fabs(static_cast<double>(mn)), fabs(static_cast<double>(mx)));

    float best = 0.0f;
    int best_i = 0;
    for (int gi = 0; gi < n_grid; ++gi) {
        const double c = clip_bound(gi, step, amax);
        const float cf = __double2float_rd(c);
        const QParams p = range_params(fmax(static_cast<double>(mn), -c),
                                       fmin(static_cast<double>(mx), c), maxq, sym != 0);
        float d[G];
#pragma unroll
        for (int j = 0; j < G; ++j) {
            const float w = Wt[j * rc::WS + t];
            d[j] = w - dequant(clip_code(w, c, cf, p, maxq), p);
        }
        float crit = 0.0f;
        if (H) {
#pragma unroll 1
            for (int i = 0; i < G; ++i) {
                const float* hrow = Hs + i * G;
                float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j4 = 0; j4 < G; j4 += 4) {
                    const float4 h = *reinterpret_cast<const float4*>(hrow + j4);
                    const int u = (j4 / 4) & 1;
                    a[4 * u + 0] = fmaf(h.x, d[j4 + 0], a[4 * u + 0]);
                    a[4 * u + 1] = fmaf(h.y, d[j4 + 1], a[4 * u + 1]);
                    a[4 * u + 2] = fmaf(h.z, d[j4 + 2], a[4 * u + 2]);
                    a[4 * u + 3] = fmaf(h.w, d[j4 + 3], a[4 * u + 3]);
                }
                const float ai = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
                const float w = Wt[i * rc::WS + t];
                const float di = w - dequant(clip_code(w, c, cf, p, maxq), p);
                crit = fmaf(di, ai, crit);
            }
        } else {
#pragma unroll
            for (int j = 0; j < G; ++j) crit = fmaf(d[j], d[j], crit);
        }
        if (gi == 0 || crit < best) {
            best = crit;
            best_i = gi;
        }
    }

    // the chosen ratio's codes, grid and index
    const double c = clip_bound(best_i, step, amax);
    const float cf = __double2float_rd(c);
    const QParams p = range_params(fmax(static_cast<double>(mn), -c),
                                   fmin(static_cast<double>(mx), c), maxq, sym != 0);
    if (bits == 4) {
        uint8_t* o = out + static_cast<int64_t>(r) * (d_in / 2) + k0 / 2;
        for (int j = 0; j < G; j += 2) {
            const int q0 = clip_code(Wt[j * rc::WS + t], c, cf, p, maxq);
            const int q1 = clip_code(Wt[(j + 1) * rc::WS + t], c, cf, p, maxq);
            o[j / 2] = static_cast<uint8_t>(q0 | (q1 << 4));
        }
    } else {
        uint8_t* o = out + static_cast<int64_t>(r) * d_in + k0;
        for (int j = 0; j < G; ++j) o[j] = static_cast<uint8_t>(clip_code(Wt[j * rc::WS + t], c, cf, p, maxq));
    }
    const int64_t gidx = static_cast<int64_t>(r) * ng + k;
    scales[gidx] = half_bits(p.scale);
    zeros[gidx] = half_bits(p.zero);
    if (ratio_idx) ratio_idx[gidx] = static_cast<uint8_t>(best_i);
}

template <int G, typename T>
static gptq_status launch_clip(const T* W, int d_out, int d_in, int bits, int sym,
                               const float* H, int n_grid, double step, uint8_t* out,
                               uint16_t* scales, uint16_t* zeros, uint8_t* ratio_idx,
                               cudaStream_t s) {
    const int smem = (G * rc::WS + (H ? G * G : 0)) * 4;
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(rtn_clip_kernel<G, T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (G * rc::WS + G * G) * 4));
    const dim3 grid(d_in / G, (d_out + rc::ROWS - 1) / rc::ROWS);
    rtn_clip_kernel<G, T><<<grid, rc::ROWS, smem, s>>>(W, d_out, d_in, bits, sym, H, n_grid,
                                                       step, out, scales, zeros, ratio_idx);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

template <typename T>
static gptq_status clip_dispatch(const T* W, int d_out, int d_in, int bits, int g, int sym,
                                 const float* H, int n_grid, double step, uint8_t* out,
                                 uint16_t* scales, uint16_t* zeros, uint8_t* ratio_idx,
                                 cudaStream_t s) {
    switch (g) {
        case 16: return launch_clip<16>(W, d_out, d_in, bits, sym, H, n_grid, step, out, scales, zeros, ratio_idx, s);
        case 32: return launch_clip<32>(W, d_out, d_in, bits, sym, H, n_grid, step, out, scales, zeros, ratio_idx, s);
        case 64: return launch_clip<64>(W, d_out, d_in, bits, sym, H, n_grid, step, out, scales, zeros, ratio_idx, s);
        case 128: return launch_clip<128>(W, d_out, d_in, bits, sym, H, n_grid, step, out, scales, zeros, ratio_idx, s);
        default: return GPTQ_ERR_ARG;
    }
}

gptq_status rtn_clip_launch(const void* W, int w_dtype, int d_out, int d_in, int bits, int g,
                            int sym, const float* H, int n_grid, double step, uint8_t* out,
                            uint16_t* scales, uint16_t* zeros, uint8_t* ratio_idx,
                            cudaStream_t s) {
    if (w_dtype == GPTQ_DTYPE_F16)
        return clip_dispatch(static_cast<const __half*>(W), d_out, d_in, bits, g, sym, H, n_grid,
                             step, out, scales, zeros, ratio_idx, s);
    return clip_dispatch(static_cast<const float*>(W), d_out, d_in, bits, g, sym, H, n_grid,
                         step, out, scales, zeros, ratio_idx, s);
}

// ---------------------------------------------------------------------------------------
// Percentile and fixed-range clipping (bhfrc.com/news/5741 §4.3: take a percentile of the
// values, such as 99.99 %, or an absolute range, such as [-10, 10], instead of the extreme
// values, and truncate what lies outside). Per group: lo and hi are the (1 - p) and p
// quantiles of its values, each interpolated linearly between the two order statistics around
// position frac * (g - 1) (q = v[k] + t * (v[k+1] - v[k]), every operation rounded on its own
// in fp64); with a fixed range a > 0 they are limited to [-a, a]. The weights are clamped to
// [lo, hi] and quantized with the quantizer of that range.
//
// Kernel: the clip search's layout (one CTA per group and 128 rows, the group transposed in
// shared memory, one thread per row). Each thread finds the four order statistics it needs by
// counting, for every value of its row's group, the values below it (index order breaks ties),
// which costs g^2 comparisons per row and group and no sort.
// ---------------------------------------------------------------------------------------
struct RangeClipArgs {
    int kl, kh;          // order-statistic positions of the lower and upper quantile
    double tl, th;       // their interpolation weights
    double abs_range;    // 0: no fixed range
};

// Code of w under the clamp to [lo, hi] and the grid p: clamped weights are quantized at the
// bound in fp64 (lo and hi are fp64 values), the others by the exact rounding of quant_code.
__device__ __noinline__ int range_code_slow(float w, double lo, double hi, QParams p, int maxq) {
    const double wd = static_cast<double>(w);
    if (wd > hi || wd < lo) {
        const double q = rint((wd > hi ? hi : lo) / static_cast<double>(p.scale)) +
                         static_cast<double>(p.zero);
        return static_cast<int>(fmin(fmax(q, 0.0), static_cast<double>(maxq)));
    }
    return quant_code(w, p, maxq);
}

// Fast path: lof < w < hif (the bounds rounded inwards to fp32, so w is not clamped) and
// w/scale clear of a rounding boundary by more than the error of its fp32 quotient.
__device__ __forceinline__ int range_code(float w, double lo, double hi, float lof, float hif,
                                          const QParams& p, int maxq) {
    const float t = w * p.inv_scale;
    const float k = rintf(t);
    if (w > lof && w < hif && fabsf(t - k) <= 0.5f - fabsf(t) * 3.0e-7f - 1.0e-30f)
        return static_cast<int>(fminf(fmaxf(k + p.zero, 0.0f), static_cast<float>(maxq)));
    return range_code_slow(w, lo, hi, p, maxq);
}

__device__ __forceinline__ double lerp_rn(double v0, double v1, double t) {
    return __dadd_rn(v0, __dmul_rn(t, __dsub_rn(v1, v0)));
}

template <int G, typename T>
__global__ void __launch_bounds__(rc::ROWS) rtn_range_kernel(
    const T* __restrict__ W, int d_out, int d_in, int bits, int sym, RangeClipArgs a,
    uint8_t* __restrict__ out, uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros) {
    extern __shared__ __align__(16) float range_smem[];
    float* Wt = range_smem;                   // [G][WS]: Wt[j][t] = W[r0 + t][k0 + j]
    const int t = threadIdx.x;
    const int k = blockIdx.x, r0 = blockIdx.y * rc::ROWS;
    const int64_t k0 = static_cast<int64_t>(k) * G;
    const int maxq = (1 << bits) - 1;
    for (int rr = 0; rr < rc::ROWS; ++rr) {
        const int r = r0 + rr;
        for (int j = t; j < G; j += rc::ROWS)
            Wt[j * rc::WS + rr] = r < d_out ? static_cast<float>(W[static_cast<int64_t>(r) * d_in + k0 + j]) : 0.0f;
    }
    __syncthreads();
    const int r = r0 + t;
    if (r >= d_out) return;

    // the order statistics at positions kl, kl + 1, kh, kh + 1 (clamped to g - 1)
    const int pl0 = a.kl, pl1 = min(a.kl + 1, G - 1), ph0 = a.kh, ph1 = min(a.kh + 1, G - 1);
    float vl0 = 0.f, vl1 = 0.f, vh0 = 0.f, vh1 = 0.f;
#pragma unroll 1
    for (int j = 0; j < G; ++j) {
        const float vj = Wt[j * rc::WS + t];
        int rank = 0;
#pragma unroll 8
        for (int i = 0; i < G; ++i) {
            const float vi = Wt[i * rc::WS + t];
            rank += (vi < vj || (vi == vj && i < j)) ? 1 : 0;
        }
        if (rank == pl0) vl0 = vj;
        if (rank == pl1) vl1 = vj;
        if (rank == ph0) vh0 = vj;
        if (rank == ph1) vh1 = vj;
    }
    double lo = a.kl >= G - 1 ? static_cast<double>(vl0)
                              : lerp_rn(static_cast<double>(vl0), static_cast<double>(vl1), a.tl);
    double hi = a.kh >= G - 1 ? static_cast<double>(vh0)
                              : lerp_rn(static_cast<double>(vh0), static_cast<double>(vh1), a.th);
    if (a.abs_range > 0.0) {
        lo = fmax(lo, -a.abs_range);
        hi = fmin(hi, a.abs_range);
    }
    const float lof = __double2float_ru(lo), hif = __double2float_rd(hi);
    const QParams p = range_params(lo, hi, maxq, sym != 0);
    if (bits == 4) {
        uint8_t* o = out + static_cast<int64_t>(r) * (d_in / 2) + k0 / 2;
        for (int j = 0; j < G; j += 2) {
            const int q0 = range_code(Wt[j * rc::WS + t], lo, hi, lof, hif, p, maxq);
            const int q1 = range_code(Wt[(j + 1) * rc::WS + t], lo, hi, lof, hif, p, maxq);
            o[j / 2] = static_cast<uint8_t>(q0 | (q1 << 4));
        }
    } else {
        uint8_t* o = out + static_cast<int64_t>(r) * d_in + k0;
        for (int j = 0; j < G; ++j)
            o[j] = static_cast<uint8_t>(range_code(Wt[j * rc::WS + t], lo, hi, lof, hif, p, maxq));
    }
    const int64_t gidx = static_cast<int64_t>(r) * (d_in / G) + k;
    scales[gidx] = half_bits(p.scale);
    zeros[gidx] = half_bits(p.zero);
}

template <int G, typename T>
static gptq_status launch_range(const T* W, int d_out, int d_in, int bits, int sym,
                                const RangeClipArgs& a, uint8_t* out, uint16_t* scales,
                                uint16_t* zeros, cudaStream_t s) {
    const int smem = G * rc::WS * 4;
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(rtn_range_kernel<G, T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    const dim3 grid(d_in / G, (d_out + rc::ROWS - 1) / rc::ROWS);
    rtn_range_kernel<G, T><<<grid, rc::ROWS, smem, s>>>(W, d_out, d_in, bits, sym, a, out,
                                                        scales, zeros);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

template <typename T>
static gptq_status range_dispatch(const T* W, int d_out, int d_in, int bits, int g, int sym,
                                  const RangeClipArgs& a, uint8_t* out, uint16_t* scales,
                                  uint16_t* zeros, cudaStream_t s) {
    switch (g) {
        case 16: return launch_range<16>(W, d_out, d_in, bits, sym, a, out, scales, zeros, s);
        case 32: return launch_range<32>(W, d_out, d_in, bits, sym, a, out, scales, zeros, s);
        case 64: return launch_range<64>(W, d_out, d_in, bits, sym, a, out, scales, zeros, s);
        case 128: return launch_range<128>(W, d_out, d_in, bits, sym, a, out, scales, zeros, s);
        default: return GPTQ_ERR_ARG;
    }
}

}  // namespace gq

extern "C" gptq_status rtn_range_clip(const void* W, int w_dtype, int d_out, int d_in, int bits,
                                      int group_size, int sym, double percentile,
                                      double abs_range, uint8_t* packed, uint16_t* scales,
                                      uint16_t* zeros, void* stream) {
    if (!W || !packed || !scales || !zeros) return GPTQ_ERR_ARG;
    if (w_dtype != GPTQ_DTYPE_F16 && w_dtype != GPTQ_DTYPE_F32) return GPTQ_ERR_ARG;
    if (d_out < 1 || d_in < 16 || bits < 2 || bits > 8 || sym < 0 || sym > 1) return GPTQ_ERR_ARG;
    if (group_size != 16 && group_size != 32 && group_size != 64 && group_size != 128)
        return GPTQ_ERR_ARG;
    if (d_in % group_size) return GPTQ_ERR_ARG;
    if (!(percentile >= 50.0 && percentile <= 100.0) || !(abs_range >= 0.0) ||
        std::isinf(abs_range))
        return GPTQ_ERR_ARG;
    // the quantile positions, each operation rounded on its own (as the definition reads)
    const double p = percentile / 100.0;
    const double q_lo = 1.0 - p;
    const double gm1 = static_cast<double>(group_size - 1);
    const double h_hi = p * gm1, h_lo = q_lo * gm1;
    gq::RangeClipArgs a;
    a.kh = static_cast<int>(std::floor(h_hi));
    a.kl = static_cast<int>(std::floor(h_lo));
    a.th = h_hi - a.kh;
    a.tl = h_lo - a.kl;
    a.abs_range = abs_range;
    GPTQ_TRY(gq::check_device());
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (w_dtype == GPTQ_DTYPE_F16)
        return gq::range_dispatch(static_cast<const __half*>(W), d_out, d_in, bits, group_size,
                                  sym, a, packed, scales, zeros, s);
    return gq::range_dispatch(static_cast<const float*>(W), d_out, d_in, bits, group_size, sym,
                              a, packed, scales, zeros, s);
}

extern "C" gptq_status rtn_clip_search(const void* W, int w_dtype, int d_out, int d_in,
                                       int bits, int group_size, int sym, const float* H,
                                       double min_ratio, double step, uint8_t* packed,
                                       uint16_t* scales, uint16_t* zeros, uint8_t* ratio_idx,
                                       void* stream) {
    if (!W || !packed || !scales || !zeros) return GPTQ_ERR_ARG;
    if (w_dtype != GPTQ_DTYPE_F16 && w_dtype != GPTQ_DTYPE_F32) return GPTQ_ERR_ARG;
    if (d_out < 1 || d_in < 16 || bits < 2 || bits > 8 || sym < 0 || sym > 1) return GPTQ_ERR_ARG;
    if (group_size != 16 && group_size != 32 && group_size != 64 && group_size != 128)
        return GPTQ_ERR_ARG;
    if (d_in % group_size) return GPTQ_ERR_ARG;
    if (!(step > 0.0) || !(min_ratio > 0.0) || !(min_ratio <= 1.0)) return GPTQ_ERR_ARG;
    const double nd = (1.0 - min_ratio) / step;
    if (!(nd < gq::rc::MAX_GRID)) return GPTQ_ERR_ARG;
    const int n_grid = static_cast<int>(nearbyint(nd)) + 1;
    if (n_grid > gq::rc::MAX_GRID) return GPTQ_ERR_ARG;
    if (H && (reinterpret_cast<uintptr_t>(H) & 15)) return GPTQ_ERR_ARG;
    GPTQ_TRY(gq::check_device());
    return gq::rtn_clip_launch(W, w_dtype, d_out, d_in, bits, group_size, sym, H, n_grid, step,
                               packed, scales, zeros, ratio_idx,
                               static_cast<cudaStream_t>(stream));
}
