// The asymmetric per-group min-max quantizer, shared by RTN and the GPTQ column loop.
//
// 0539edu.com/news/6111416 §2.1: q = round(x/scale) + zero_point, scale = (max-min)/(qmax-qmin).
// §4.2: one fp16 scale and one fp16 zero point per group.
//
// The group's range [xmin, xmax] is widened to contain 0 (the formula maps real 0 to the code
// zero_point, so the zero point is a code in [0, maxq] and exact in fp16). Group scalars are
// computed in fp64:  scale = smallest fp16 >= (xmax - xmin)/maxq (1 for an all-zero group),
// zero = rint(-xmin/scale) (half to even, +0 rather than -0). Per-element codes
// q = clamp(rint(w/scale) + zero, 0, maxq) are decided EXACTLY in fp32: an approximate
// quotient gives a candidate k, and the sign of w - (k +- 1/2)*scale, computed with a single
// fused multiply-add (one rounding of the exact value, so its sign is exact), moves k by one
// where needed and resolves exact halves to even. The result equals rint of the exact
// quotient for any fp16/fp32 w and fp16 scale.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace gq {

// Smallest fp16 value >= x for x >= 0 (finite), returned as an fp64 holding that value.
// fp16 values near x are spaced 2^(e-10) for x in [2^e, 2^(e+1)), e >= -14, and 2^-24 below
// 2^-14 (subnormals); dividing and multiplying by a power of two is exact, so
// ceil(x / spacing) * spacing is the answer. Above 65504 the result is +inf.
__device__ __forceinline__ double fp16_ceil(double x) {
    if (!(x > 0.0)) return x;
    if (x > 65504.0) return __longlong_as_double(0x7FF0000000000000LL);
    const long long bits = __double_as_longlong(x);
    int e = static_cast<int>((bits >> 52) & 0x7FF) - 1023;   // floor(log2 x) for normal x
    if (e < -14) e = -14;
    // spacing = 2^(e-10) and its exact reciprocal 2^(10-e); x * 2^(10-e) is exact in fp64
    const double spacing = __longlong_as_double(static_cast<long long>(e - 10 + 1023) << 52);
    const double inv_spacing = __longlong_as_double(static_cast<long long>(10 - e + 1023) << 52);
    return ceil(x * inv_spacing) * spacing;
}

struct QParams {
    float scale;      // fp16-representable
    float zero;       // integer-valued
    float inv_scale;  // approximate 1/scale, only used to form the candidate code
};

// rint(-lo / s) (half to even) for -lo >= 0 and 0 < s, with -lo/s <= 2^20: a candidate from an
// approximate quotient, then the exact fp64 residual -lo - k*s (k*s is exact: k has at most 21
// bits and s 11) moves it to the nearest integer and settles exact halves to even. It equals
// rint of the correctly rounded fp64 quotient, which cannot land on a half-integer the exact
// quotient is not on (-lo has 24 significant bits, so a nonzero distance to one is far larger
// than an fp64 rounding).
__device__ __forceinline__ double rint_quotient(double nlo, double s) {
    float r;   // approximate 1/s: the candidate only has to be within one of the answer
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(static_cast<float>(s)));
    double k = rint(nlo * static_cast<double>(r));
    const double e = fma(-k, s, nlo);        // exact
    if (2.0 * e > s) k += 1.0;
    else if (2.0 * e < -s) k -= 1.0;
    const double e2 = fma(-k, s, nlo);       // exact; |e2| <= s/2
    if ((2.0 * e2 == s || 2.0 * e2 == -s) && (static_cast<long long>(k) & 1))
        k += (e2 > 0.0 ? 1.0 : -1.0);        // a tie: take the even neighbour
    return k;
}

__device__ __forceinline__ QParams group_params(float xmin, float xmax, int maxq) {
    const double lo = fmin(static_cast<double>(xmin), 0.0);
    const double hi = fmax(static_cast<double>(xmax), 0.0);
    const double span = hi - lo;
    const double s = (span == 0.0) ? 1.0 : fp16_ceil(span / static_cast<double>(maxq));
    // -lo/s <= span/s <= maxq; an infinite s (span/maxq above the fp16 range) gives zero 0
    const double z = (isinf(s) ? 0.0 : rint_quotient(-lo, s)) + 0.0;
    QParams p;
    p.scale = static_cast<float>(s);
    p.zero = static_cast<float>(z);
    p.inv_scale = __frcp_rn(p.scale);   // fp32 1/scale, within one rounding of the exact value
    return p;
}

// The symmetric quantizer (0539edu.com §2.3: zero point fixed at 0, q = round(x/scale)): the
// range is [-m, m], m = max(|xmin|, |xmax|), split into maxq steps, scale = smallest fp16 >=
// 2m/maxq (1 for an all-zero group), and the signed zero 0 is stored as the code offset
// (maxq + 1)/2, so code = clamp(rint(w/scale) + (maxq + 1)/2, 0, maxq).
__device__ __forceinline__ QParams group_params_sym(float xmin, float xmax, int maxq) {
    const double m = fmax(fabs(static_cast<double>(xmin)), fabs(static_cast<double>(xmax)));
    const double s = (m == 0.0) ? 1.0 : fp16_ceil(2.0 * m / static_cast<double>(maxq));
    QParams p;
    p.scale = static_cast<float>(s);
    p.zero = static_cast<float>((maxq + 1) / 2);
    p.inv_scale = __frcp_rn(p.scale);
    return p;
}

__device__ __forceinline__ QParams group_params_any(float xmin, float xmax, int maxq, bool sym) {
    return sym ? group_params_sym(xmin, xmax, maxq) : group_params(xmin, xmax, maxq);
}

// A stored grid (fp16 scale and zero bit patterns) as the quantizer uses it.
__device__ __forceinline__ QParams stored_params(uint16_t scale_bits, uint16_t zero_bits) {
    QParams p;
    p.scale = __half2float(__ushort_as_half(scale_bits));
    p.zero = __half2float(__ushort_as_half(zero_bits));
    p.inv_scale = __frcp_rn(p.scale);
    return p;
}

// The same, kept out of line: for loops that reach it rarely (once per group) and would
// otherwise carry one inlined copy of the fp64 sequence per unrolled iteration.
static __device__ __noinline__ QParams group_params_call(float xmin, float xmax, int maxq) {
    return group_params(xmin, xmax, maxq);
}

// rint(w / scale) with the exact tie-to-even decision described above.
__device__ __forceinline__ float round_quotient(float w, float scale, float inv_scale) {
    float k = rintf(w * inv_scale);
    if (fabsf(k) >= 4194304.0f) {  // 2^22: k +- 1/2 would not be exact in fp32
        return static_cast<float>(rint(static_cast<double>(w) / static_cast<double>(scale)));
    }
    const float up = fmaf(-(k + 0.5f), scale, w);   // sign of w - (k + 1/2) * scale
    const float dn = fmaf(-(k - 0.5f), scale, w);   // sign of w - (k - 1/2) * scale
    const bool k_odd = (static_cast<int>(k) & 1) != 0;
    if (up > 0.0f || (up == 0.0f && k_odd)) {
        k += 1.0f;
    } else if (dn < 0.0f || (dn == 0.0f && k_odd)) {
        k -= 1.0f;
    }
    return k;
}

__device__ __forceinline__ int quant_code(float w, const QParams& p, int maxq) {
    // Fast path: t = w * (1/scale) is within |t| * 2.4e-7 of the exact quotient (two fp32
    // roundings), so when its distance to the nearest half-integer exceeds that bound, rintf(t)
    // is already the exact rounding. Otherwise (rare) decide exactly with round_quotient.
    const float t = w * p.inv_scale;
    float k = rintf(t);
    if (fabsf(t - k) > 0.5f - fabsf(t) * 3.0e-7f - 1.0e-30f) {
        k = round_quotient(w, p.scale, p.inv_scale);
    }
    const float q = fminf(fmaxf(k + p.zero, 0.0f), static_cast<float>(maxq));
    return static_cast<int>(q);
}

// The same code as quant_code, kept as an integer-valued float (for packing without F2I).
__device__ __forceinline__ float quant_codef(float w, const QParams& p, float maxqf) {
    const float t = w * p.inv_scale;
    float k = rintf(t);
    if (fabsf(t - k) > 0.5f - fabsf(t) * 3.0e-7f - 1.0e-30f) k = round_quotient(w, p.scale, p.inv_scale);
    return fminf(fmaxf(k + p.zero, 0.0f), maxqf);
}

// Integer bits of an integer-valued float in [0, 2^22): add 2^23 and read the mantissa.
__device__ __forceinline__ uint32_t small_int_bits(float v) {
    return __float_as_uint(v + 8388608.0f) - 0x4B000000u;
}

__device__ __forceinline__ float dequant(int q, const QParams& p) {
    return p.scale * (static_cast<float>(q) - p.zero);
}

__device__ __forceinline__ uint16_t half_bits(float v) {
    return __half_as_ushort(__float2half_rn(v));  // exact for fp16-representable v
}

}  // namespace gq
