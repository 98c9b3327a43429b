// Group min-max round-to-nearest (RTN), the cheap baseline of the calibration-methods page
// (bhfrc.com/news/5741 §2.2, group min-max) and of the GPTQ deep-dive (hncyxsy.com §1.2):
// every weight is rounded independently with its group's min-max scale and zero point.
//
// HBM-bound streaming kernel. Each thread owns 8 consecutive weights (one 16-byte load of
// fp16, or two of fp32); the group_size/8 threads of a group reduce min and max with xor
// shuffles, compute the group's scalars in fp64, and write 8 codes (4 bytes packed INT4, or
// 8 bytes) plus, from the group's first thread, the fp16 scale and zero. Bytes per weight:
// 2 (fp16 in) + 0.5 (INT4 out) + 4/group_size (scale + zero).
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "quant.cuh"

namespace gq {

template <typename T>
struct Load8;

template <>
struct Load8<__half> {
    static __device__ __forceinline__ void run(const __half* p, float* v) {
        const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
        const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(h[i]);
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
};

template <>
struct Load8<float> {
    static __device__ __forceinline__ void run(const float* p, float* v) {
        const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
        const float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

// E = weights per thread (8 or 16); TPG = threads per group (group_size / E), a power of two
// in [1, 32]. All loads of an iteration are issued before any arithmetic.
template <typename T, int E, int TPG>
__global__ void __launch_bounds__(256) rtn_kernel(const T* __restrict__ W, int64_t n_chunks,
                                                  int bits, int sym, uint8_t* __restrict__ out,
                                                  uint16_t* __restrict__ scales,
                                                  uint16_t* __restrict__ zeros) {
    const int maxq = (1 << bits) - 1;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    // the loop runs warp-uniformly (full-mask shuffles below); lanes past the end form whole
    // groups because n_chunks is a multiple of TPG, and they only skip their loads and stores
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31);
         base < n_chunks; base += stride) {
        const int64_t t = base + (threadIdx.x & 31);
        const bool ok = t < n_chunks;
        float v[E];
        if (ok) {
#pragma unroll
            for (int h = 0; h < E / 8; ++h) Load8<T>::run(W + t * E + 8 * h, v + 8 * h);
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i) v[i] = 0.0f;
        }
        float mn = v[0], mx = v[0];
#pragma unroll
        for (int i = 1; i < E; ++i) {
            mn = fminf(mn, v[i]);
            mx = fmaxf(mx, v[i]);
        }
#pragma unroll
        for (int off = TPG / 2; off > 0; off >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        }
        if (!ok) continue;
        const QParams p = group_params_any(mn, mx, maxq, sym != 0);
        int q[E];
#pragma unroll
        for (int i = 0; i < E; ++i) q[i] = quant_code(v[i], p, maxq);
        if (bits == 4) {
#pragma unroll
            for (int h = 0; h < E / 8; ++h) {
                uint32_t packed = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) packed |= static_cast<uint32_t>(q[8 * h + i]) << (4 * i);
                __stcs(reinterpret_cast<unsigned int*>(out) + t * (E / 8) + h, packed);
            }
        } else {
#pragma unroll
            for (int h = 0; h < E / 8; ++h) {
                uint2 b;
                b.x = q[8 * h] | (q[8 * h + 1] << 8) | (q[8 * h + 2] << 16) | (q[8 * h + 3] << 24);
                b.y = q[8 * h + 4] | (q[8 * h + 5] << 8) | (q[8 * h + 6] << 16) | (q[8 * h + 7] << 24);
                __stcs(reinterpret_cast<uint2*>(out) + t * (E / 8) + h, b);
            }
        }
        if ((t & (TPG - 1)) == 0) {
            const int64_t gi = t / TPG;
            scales[gi] = half_bits(p.scale);
            zeros[gi] = half_bits(p.zero);
        }
    }
}

namespace rp {
constexpr int WARPS = 8, THREADS = WARPS * 32;
constexpr int E = 32;                          // weights per lane
constexpr int STAGES = 4;                      // per-warp ring of 2 KB stages
constexpr int STAGE_BYTES = 32 * E * 2;        // one warp-iteration: 32 lanes x 32 fp16
constexpr int SMEM = WARPS * STAGES * STAGE_BYTES;   // 64 KB
}  // namespace rp

// The group scalars of group_params (same values, bit for bit) without branches, for the
// streaming kernel: s = smallest fp16 >= span/maxq (the one fp64 division is the same IEEE
// operation), z = rint(-lo/s) corrected with the exact residual (ties to even), and an
// approximate 1/s (relative error <= 2^-23; the codes only use it for a candidate that the
// caller checks).
__device__ __forceinline__ QParams group_params_stream(float xmin, float xmax, int maxq) {
    const double lo = fmin(static_cast<double>(xmin), 0.0);
    const double hi = fmax(static_cast<double>(xmax), 0.0);
    const double span = hi - lo;
    const double q = span / static_cast<double>(maxq);
    // fp16_ceil(q) for q > 0: spacing 2^(e-10), e = max(floor(log2 q), -14)
    const long long qb = __double_as_longlong(q);
    const int e = max(static_cast<int>((qb >> 52) & 0x7FF) - 1023, -14);
    const double spacing = __longlong_as_double(static_cast<long long>(e - 10 + 1023) << 52);
    const double inv_spacing = __longlong_as_double(static_cast<long long>(10 - e + 1023) << 52);
    double sc = ceil(q * inv_spacing) * spacing;
    sc = (q > 65504.0) ? __longlong_as_double(0x7FF0000000000000LL) : sc;
    sc = (span == 0.0) ? 1.0 : sc;
    // z = rint(-lo / sc): candidate, then one exact correction and the tie rule
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(static_cast<float>(sc)));
    const double nlo = -lo;
    double k = rint(nlo * static_cast<double>(r));
    const double e1 = fma(-k, sc, nlo);
    k += (2.0 * e1 > sc) ? 1.0 : ((2.0 * e1 < -sc) ? -1.0 : 0.0);
    const double e2 = fma(-k, sc, nlo);
    const bool tie = (2.0 * e2 == sc || 2.0 * e2 == -sc) && (static_cast<long long>(k) & 1);
    k += tie ? (e2 > 0.0 ? 1.0 : -1.0) : 0.0;
    k = isinf(sc) ? 0.0 : k;
    QParams p;
    p.scale = static_cast<float>(sc);
    p.zero = static_cast<float>(k + 0.0);
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(p.inv_scale) : "f"(p.scale));
    return p;
}

constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23: integers up to 2^22 sit in the low bits

// 32 codes held as kMagic + code, packed (INT4: two per byte, the even index in the low
// nibble; else one per byte) and stored with streaming 16-byte stores at chunk t.
template <bool INT4>
__device__ __forceinline__ void store_codes(const float (&m)[32], uint8_t* __restrict__ out,
                                            int t) {
    if (INT4) {
        // byte b holds codes 2b (low nibble) and 2b+1: the bit pattern of kMagic + q is
        // 0x4B400000 + q, so 16 bits(m_2b+1) + bits(m_2b) has q_2b + 16 q_2b+1 in its low byte
        uint32_t by[16];
#pragma unroll
        for (int b = 0; b < 16; ++b)
            by[b] = (__float_as_uint(m[2 * b + 1]) << 4) + __float_as_uint(m[2 * b]);
        uint32_t word[4];
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4)
            word[w4] = __byte_perm(__byte_perm(by[4 * w4], by[4 * w4 + 1], 0x0040),
                                   __byte_perm(by[4 * w4 + 2], by[4 * w4 + 3], 0x0040), 0x5410);
        __stcs(reinterpret_cast<uint4*>(out) + t, make_uint4(word[0], word[1], word[2], word[3]));
    } else {
        // one code per byte: the low byte of the magic-added pattern is the code
        uint32_t word[8];
#pragma unroll
        for (int w4 = 0; w4 < 8; ++w4)
            word[w4] = __byte_perm(__byte_perm(__float_as_uint(m[4 * w4]), __float_as_uint(m[4 * w4 + 1]), 0x0040),
                                   __byte_perm(__float_as_uint(m[4 * w4 + 2]), __float_as_uint(m[4 * w4 + 3]), 0x0040), 0x5410);
        __stcs(reinterpret_cast<uint4*>(out) + 2 * t, make_uint4(word[0], word[1], word[2], word[3]));
        __stcs(reinterpret_cast<uint4*>(out) + 2 * t + 1, make_uint4(word[4], word[5], word[6], word[7]));
    }
}

// 1/s bracketed by two fp32 values, inv_lo < 1/s < inv_hi, each within 1.5 ulp of it:
// r = RN(1/s), and the sign of 1 - s r (exact in one fma: s has 11 significant bits, r 24, and
// |1 - s r| <= 2^-24 on a grid of 2^-34) says on which side of 1/s r lies. An infinite s
// (range above the fp16 grid) gives 0 for both, the quotient quant_code uses there.
__device__ __forceinline__ void reciprocal_bracket(float s, float& inv_lo, float& inv_hi) {
    const float r = __frcp_rn(s);
    const float e = fmaf(-s, r, 1.0f);
    const uint32_t rb = __float_as_uint(r);
    inv_lo = (e > 0.0f) ? r : __uint_as_float(rb - 1u);
    inv_hi = (e < 0.0f) ? r : __uint_as_float(rb + 1u);
    if (isinf(s)) inv_lo = inv_hi = 0.0f;
}

// kMagic + rint(w/s) + z, rint rounding half to even, for fp16 w and s with |w/s| <= 2^8:
// m1 and m2 round w inv_lo + C and w inv_hi + C (C = z + kMagic, ulp 1) once each. The two
// products bracket w/s within 4.6e-5, and a w/s that is not a half-integer lies at least
// 1.2e-4 from every half-integer (w and s are multiples of 2^(e-10) and 2^(e'-10) with |w| >=
// s/2 near a boundary), so m1 = m2 = the nearest integer, except at an exact tie, where m1
// and m2 are its two neighbours and the one whose w/s part k = m - C is even is taken (the
// parity of k is the low bit of bits(m) ^ bits(C): both lie on the ulp-1 grid).
__device__ __forceinline__ float round_code(float w, float inv_lo, float inv_hi, float C,
                                            uint32_t Cb) {
    const float m1 = fmaf(w, inv_lo, C);
    const float m2 = fmaf(w, inv_hi, C);
    return ((__float_as_uint(m1) ^ Cb) & 1u) ? m2 : m1;
}

// fp16 weights, power-of-two groups of 32..256: a lane quantizes 32 consecutive weights
// (TPG = group_size / 32 lanes per group). Each warp streams its 2 KB per iteration through a
// 4-stage shared-memory ring with per-lane async copies (coalesced: lane L copies bytes
// 16L + 512h), keeping three iterations in flight while it computes one, which is what keeps
// enough bytes outstanding to run at HBM speed. Codes come out of the rounding as float bit
// patterns and are packed with byte permutes. Chunk indices are 32-bit (the launcher checks).
template <int TPG, bool INT4>
__global__ void __launch_bounds__(rp::THREADS, 3) rtn_f16_kernel(const __half* __restrict__ W,
                                                                int n_chunks, int bits, int sym,
                                                                uint8_t* __restrict__ out,
                                                                uint16_t* __restrict__ scales,
                                                                uint16_t* __restrict__ zeros) {
    extern __shared__ __align__(16) uint8_t rtn_smem[];
    const int lane = lane_id(), warp = warp_id();
    uint8_t* ring = rtn_smem + warp * rp::STAGES * rp::STAGE_BYTES;
    const int maxq = (1 << bits) - 1;
    const int n_wit = (n_chunks + 31) / 32;                        // warp-iterations in total
    const int wstride = gridDim.x * rp::WARPS;
    const int w0 = blockIdx.x * rp::WARPS + warp;
    const uint8_t* wbytes = reinterpret_cast<const uint8_t*>(W);
    auto issue = [&](int wi, int st) {
        if (wi < n_wit) {
            const uint8_t* src = wbytes + static_cast<int64_t>(wi) * rp::STAGE_BYTES + 16 * lane;
            uint8_t* dst = ring + st * rp::STAGE_BYTES + 16 * lane;
            const int valid = min(32, n_chunks - wi * 32) * (2 * rp::E) - 16 * lane;   // bytes
#pragma unroll
            for (int h = 0; h < 4; ++h)
                if (512 * h < valid) cp_async16(dst + 512 * h, src + 512 * h);
        }
        cp_async_commit();
    };
#pragma unroll
    for (int k = 0; k < rp::STAGES - 1; ++k) issue(w0 + k * wstride, k);
    int st = 0;
    for (int wi = w0; wi < n_wit; wi += wstride) {
        __syncwarp();     // every lane is done reading the stage the next copy overwrites
        issue(wi + (rp::STAGES - 1) * wstride, (st + rp::STAGES - 1) & (rp::STAGES - 1));
        cp_async_wait<rp::STAGES - 1>();
        __syncwarp();     // this iteration's 2 KB, copied by all lanes, is in shared memory
        const int t = wi * 32 + lane;
        const uint4* mine = reinterpret_cast<const uint4*>(ring + st * rp::STAGE_BYTES + 64 * lane);
        st = (st + 1) & (rp::STAGES - 1);
        uint4 raw[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) raw[h] = mine[h];   // (lanes past the end hold stale data, unused)
        // group min/max on the fp16 pairs (exact: the fp16 -> fp32 conversion is monotone)
        const __half2* hp = reinterpret_cast<const __half2*>(raw);
        __half2 mn2 = __hmin2(hp[0], hp[1]), mx2 = __hmax2(hp[0], hp[1]);
#pragma unroll
        for (int i = 2; i < 16; ++i) {
            mn2 = __hmin2(mn2, hp[i]);
            mx2 = __hmax2(mx2, hp[i]);
        }
        float mn = fminf(__low2float(mn2), __high2float(mn2));
        float mx = fmaxf(__low2float(mx2), __high2float(mx2));
#pragma unroll
        for (int off = TPG / 2; off > 0; off >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        }
        if (t >= n_chunks) continue;
        const QParams p = sym ? group_params_sym(mn, mx, maxq) : group_params_stream(mn, mx, maxq);
        // every code in one rounding per bracket end (round_code), so ties need no second path
        float inv_lo, inv_hi;
        reciprocal_bracket(p.scale, inv_lo, inv_hi);
        const float C = p.zero + kMagic;                         // exact: zero is an integer
        const uint32_t Cb = __float_as_uint(C);
        float m[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float2 f = __half22float2(hp[i]);
            m[2 * i] = round_code(f.x, inv_lo, inv_hi, C, Cb);
            m[2 * i + 1] = round_code(f.y, inv_lo, inv_hi, C, Cb);
        }
        // codes are monotone in w: only a tie at the group's extremes can land one step past
        // [0, maxq] (rint(hi/s) + z <= maxq + 1), and then every lane of the group clamps
        const float maxqf = static_cast<float>(maxq);
        if (round_code(mx, inv_lo, inv_hi, C, Cb) > kMagic + maxqf ||
            round_code(mn, inv_lo, inv_hi, C, Cb) < kMagic) {
#pragma unroll
            for (int i = 0; i < 32; ++i) m[i] = fminf(fmaxf(m[i], kMagic), kMagic + maxqf);
        }
        store_codes<INT4>(m, out, t);
        if ((t & (TPG - 1)) == 0) {
            scales[t / TPG] = half_bits(p.scale);
            zeros[t / TPG] = half_bits(p.zero);
        }
    }
}

template <int TPG, bool INT4>
static gptq_status launch_rtn_f16(const __half* W, int64_t n, int bits, int sym, uint8_t* out,
                                  uint16_t* scales, uint16_t* zeros, cudaStream_t s) {
    static bool attr = false;
    if (!attr) {
        GPTQ_CUDA_TRY(cudaFuncSetAttribute(rtn_f16_kernel<TPG, INT4>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, rp::SMEM));
        attr = true;
    }
    // three resident blocks per SM; warps stride over warp-iterations of 1024 weights
    const int n_chunks = static_cast<int>(n / rp::E);
    const int64_t n_wit = (n_chunks + 31) / 32;
    const int64_t want = (n_wit + rp::WARPS - 1) / rp::WARPS;
    const unsigned grid = static_cast<unsigned>(
        std::max<int64_t>(1, std::min<int64_t>(want, 3 * static_cast<int64_t>(num_sms()))));
    rtn_f16_kernel<TPG, INT4><<<grid, rp::THREADS, rp::SMEM, s>>>(W, n_chunks, bits, sym, out,
                                                                  scales, zeros);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

template <int TPG>
static gptq_status launch_rtn_f16_bits(const __half* W, int64_t n, int bits, int sym,
                                       uint8_t* out, uint16_t* scales, uint16_t* zeros,
                                       cudaStream_t s) {
    return bits == 4 ? launch_rtn_f16<TPG, true>(W, n, bits, sym, out, scales, zeros, s)
                     : launch_rtn_f16<TPG, false>(W, n, bits, sym, out, scales, zeros, s);
}

// Any group size: one thread per group.
template <typename T>
__global__ void rtn_generic_kernel(const T* __restrict__ W, int64_t n_groups, int group_size,
                                   int bits, int sym, uint8_t* __restrict__ out,
                                   uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros) {
    const int maxq = (1 << bits) - 1;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t gi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; gi < n_groups;
         gi += stride) {
        const T* w = W + gi * group_size;
        float mn = static_cast<float>(w[0]), mx = mn;
        for (int i = 1; i < group_size; ++i) {
            const float x = static_cast<float>(w[i]);
            mn = fminf(mn, x);
            mx = fmaxf(mx, x);
        }
        const QParams p = group_params_any(mn, mx, maxq, sym != 0);
        for (int i = 0; i < group_size; ++i) {
            const int64_t e = gi * group_size + i;
            const int q = quant_code(static_cast<float>(w[i]), p, maxq);
            if (bits == 4) {
                // two threads may share a byte when group_size is odd: combine atomically
                const int64_t byte = e >> 1;
                const uint32_t shift = static_cast<uint32_t>((e & 1) * 4 + (byte & 3) * 8);
                atomicOr(reinterpret_cast<unsigned int*>(out + (byte & ~3LL)),
                         static_cast<unsigned int>(q) << shift);
            } else {
                out[e] = static_cast<uint8_t>(q);
            }
        }
        scales[gi] = half_bits(p.scale);
        zeros[gi] = half_bits(p.zero);
    }
}

template <typename T>
static gptq_status launch_rtn(const T* W, int64_t n, int group_size, int bits, int sym,
                              uint8_t* out, uint16_t* scales, uint16_t* zeros, cudaStream_t s) {
    const int sms = num_sms();
    const bool pow2 = (group_size & (group_size - 1)) == 0;
    if (std::is_same<T, __half>::value && pow2 && group_size >= 32 && group_size <= 256 &&
        n / rp::E < (int64_t(1) << 31) - 64) {
        const __half* Wh = reinterpret_cast<const __half*>(W);
        if (group_size == 32) GPTQ_TRY(launch_rtn_f16_bits<1>(Wh, n, bits, sym, out, scales, zeros, s));
        else if (group_size == 64) GPTQ_TRY(launch_rtn_f16_bits<2>(Wh, n, bits, sym, out, scales, zeros, s));
        else if (group_size == 128) GPTQ_TRY(launch_rtn_f16_bits<4>(Wh, n, bits, sym, out, scales, zeros, s));
        else GPTQ_TRY(launch_rtn_f16_bits<8>(Wh, n, bits, sym, out, scales, zeros, s));
        return GPTQ_OK;
    } else if (group_size % 8 == 0 && group_size <= 256 && pow2) {
        // 16 weights per thread when the group allows it, else 8
        const int E = (group_size % 16 == 0) ? 16 : 8;
        const int64_t n_chunks = n / E;
        int64_t blocks = (n_chunks + 255) / 256;
        const int64_t cap = static_cast<int64_t>(sms) * 8;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        const dim3 grid(static_cast<unsigned>(blocks)), block(256);
        if (E == 16) {
            switch (group_size / 16) {
                case 1: rtn_kernel<T, 16, 1><<<grid, block, 0, s>>>(W, n_chunks, bits, sym, out, scales, zeros); break;
                case 2: rtn_kernel<T, 16, 2><<<grid, block, 0, s>>>(W, n_chunks, bits, sym, out, scales, zeros); break;
                case 4: rtn_kernel<T, 16, 4><<<grid, block, 0, s>>>(W, n_chunks, bits, sym, out, scales, zeros); break;
                case 8: rtn_kernel<T, 16, 8><<<grid, block, 0, s>>>(W, n_chunks, bits, sym, out, scales, zeros); break;
                default: rtn_kernel<T, 16, 16><<<grid, block, 0, s>>>(W, n_chunks, bits, sym, out, scales, zeros); break;
            }
        } else {
            rtn_kernel<T, 8, 1><<<grid, block, 0, s>>>(W, n_chunks, bits, sym, out, scales, zeros);
        }
    } else {
        const int64_t n_groups = n / group_size;
        if (bits == 4) GPTQ_CUDA_TRY(cudaMemsetAsync(out, 0, static_cast<size_t>((n + 1) / 2), s));
        int64_t blocks = (n_groups + 127) / 128;
        const int64_t cap = static_cast<int64_t>(sms) * 16;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        rtn_generic_kernel<T><<<static_cast<unsigned>(blocks), 128, 0, s>>>(
            W, n_groups, group_size, bits, sym, out, scales, zeros);
    }
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

gptq_status rtn_launch(const void* W, int w_dtype, int d_out, int d_in, int bits,
                       int group_size, int sym, uint8_t* out, uint16_t* scales, uint16_t* zeros,
                       cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(d_out) * d_in;
    if (n == 0) return GPTQ_OK;
    if (w_dtype == GPTQ_DTYPE_F16)
        return launch_rtn(static_cast<const __half*>(W), n, group_size, bits, sym, out, scales,
                          zeros, s);
    return launch_rtn(static_cast<const float*>(W), n, group_size, bits, sym, out, scales, zeros,
                      s);
}

}  // namespace gq
