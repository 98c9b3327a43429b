// Group min-max round-to-nearest (RTN), the cheap baseline of the calibration-methods page
// (bhfrc.com/news/5741 §2.2, group min-max) and of the GPTQ deep-dive (hncyxsy.com §1.2):
// every weight is rounded independently with its group's min-max scale and zero point.
//
// HBM-bound streaming kernel. Each thread owns 8 consecutive weights (one 16-byte load of
// fp16, or two of fp32); the group_size/8 threads of a group reduce min and max with xor
// shuffles, compute the group's scalars in fp64, and write 8 codes (4 bytes packed INT4, or
// 8 bytes) plus, from the group's first thread, the fp16 scale and zero. Bytes per weight:
// 2 (fp16 in) + 0.5 (INT4 out) + 4/group_size (scale + zero).
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
                                                  int bits, uint8_t* __restrict__ out,
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
        const QParams p = group_params(mn, mx, maxq);
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

// Any group size: one thread per group.
template <typename T>
__global__ void rtn_generic_kernel(const T* __restrict__ W, int64_t n_groups, int group_size,
                                   int bits, uint8_t* __restrict__ out,
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
        const QParams p = group_params(mn, mx, maxq);
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
static gptq_status launch_rtn(const T* W, int64_t n, int group_size, int bits, uint8_t* out,
                              uint16_t* scales, uint16_t* zeros, cudaStream_t s) {
    const int sms = num_sms();
    if (group_size % 8 == 0 && group_size <= 256 && (group_size & (group_size - 1)) == 0) {
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
                case 1: rtn_kernel<T, 16, 1><<<grid, block, 0, s>>>(W, n_chunks, bits, out, scales, zeros); break;
                case 2: rtn_kernel<T, 16, 2><<<grid, block, 0, s>>>(W, n_chunks, bits, out, scales, zeros); break;
                case 4: rtn_kernel<T, 16, 4><<<grid, block, 0, s>>>(W, n_chunks, bits, out, scales, zeros); break;
                case 8: rtn_kernel<T, 16, 8><<<grid, block, 0, s>>>(W, n_chunks, bits, out, scales, zeros); break;
                default: rtn_kernel<T, 16, 16><<<grid, block, 0, s>>>(W, n_chunks, bits, out, scales, zeros); break;
            }
        } else {
            rtn_kernel<T, 8, 1><<<grid, block, 0, s>>>(W, n_chunks, bits, out, scales, zeros);
        }
    } else {
        const int64_t n_groups = n / group_size;
        if (bits == 4) GPTQ_CUDA_TRY(cudaMemsetAsync(out, 0, static_cast<size_t>((n + 1) / 2), s));
        int64_t blocks = (n_groups + 127) / 128;
        const int64_t cap = static_cast<int64_t>(sms) * 16;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        rtn_generic_kernel<T><<<static_cast<unsigned>(blocks), 128, 0, s>>>(
            W, n_groups, group_size, bits, out, scales, zeros);
    }
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

gptq_status rtn_launch(const void* W, int w_dtype, int d_out, int d_in, int bits,
                       int group_size, uint8_t* out, uint16_t* scales, uint16_t* zeros,
                       cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(d_out) * d_in;
    if (n == 0) return GPTQ_OK;
    if (w_dtype == GPTQ_DTYPE_F16)
        return launch_rtn(static_cast<const __half*>(W), n, group_size, bits, out, scales, zeros, s);
    return launch_rtn(static_cast<const float*>(W), n, group_size, bits, out, scales, zeros, s);
}

}  // namespace gq
