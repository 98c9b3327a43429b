// W4A16 layer on the 5th-generation tensor cores: Y = X * What^T (+ R), the layer that serves
// a GPTQ/RTN INT4 checkpoint (0539edu.com/news/6111416 §3.2, §5.2: 4-bit weights, fp16
// activations; GPTQ deep-dive hncyxsy.com/news/243429 §3.3: with desc_act the columns' groups
// are scattered, and inference gathers them).
//
// What[r][c] = fp16(s[r][k] * (q[r][c] - z[r][k])), k the group of column c, fp32 accumulation,
// fp16 output. The act_order gather is done once on each side of the contraction: the codes
// are packed in the processing order (w4a16_pack with the layer's perm), so every group is a
// run of group_size consecutive columns again, and the activations' columns are gathered by
// the same perm (gather_cols_kernel) before the GEMM. The contraction does not depend on the
// order of its terms, so this is the g_idx formulation.
//
// GEMM kernel (persistent, one CTA per SM, output tiles of 256 tokens x 128 channels,
// k-blocks of 64 input channels, 4-stage ring):
//   warp 0      TMA producer: the X tile (two 128 x 64 fp16 boxes, 128-byte swizzle) and the
//               packed codes of the tile's 128 rows (128 x 32 bytes) per k-block.
//   warps 2-9   dequantisers: threads 2r and 2r+1 expand row r's 64 codes (32 each; a build
//               option splits a row over four threads) with its scale and zero (fp16 arithmetic: (1024 + q) - (1024 + z) is exact, times the
//               scale is the one rounding of the exact product) and write them into the B tile
//               in the 128-byte swizzled K-major layout the MMA reads, then fence and signal
//               the stage.
//   warp 1      TMEM allocator and MMA issuer: per k-block 2 x 4 tcgen05.mma kind::f16
//               M128 N128 K16, one group per 128-token half of the tile, both reading the same
//               expanded weight tile, into one of two 256-column TMEM accumulator pairs.
//   warps 10-13 epilogue: tcgen05.ld, + R, fp16, vector stores.
// Each expanded weight tile serves 256 tokens, so a weight is expanded n/256 times: the
// expansion, not the tensor pipe, bounds this kernel (half as many expansions as with
// 128-token tiles).
// Tiles run in bands of 8 token tiles with the token tile varying fastest, so the CTAs that run
// together share the same weight tiles and activation rows in L2. Every mbarrier wait is
// bounded; on timeout the kernel records GPTQ_ERR_TIMEOUT, drains its copies and MMAs, frees
// TMEM and returns.
#include <algorithm>

#include "internal.cuh"
#include "quant.cuh"

namespace gq {

namespace wq {
constexpr int BM = 256, MS = 128, BN = 128, BK = 64, STAGES = 4;
constexpr int A_SUB = MS * BK * 2;                   // 16 KB: one 128-token half
constexpr int A_BYTES = BM * BK * 2;                 // 32 KB
constexpr int B_BYTES = BN * BK * 2;                 // 16 KB
constexpr int C_BYTES = BN * BK / 2;                 // 4 KB packed codes
constexpr int OFF_B = A_BYTES;
constexpr int OFF_C = A_BYTES + B_BYTES;
constexpr int STAGE = A_BYTES + B_BYTES + C_BYTES;   // 52 KB, A and B 1024-aligned
#ifndef GPTQ_W4_TPR
#define GPTQ_W4_TPR 2
#endif
constexpr int TPR = GPTQ_W4_TPR;                     // expanding threads per weight row (2, 4)
constexpr int DQ_WARPS = BN * TPR / 32;
static_assert(TPR == 2 || TPR == 4, "a thread expands 32 or 16 codes of its row");
constexpr int EPI_WARP0 = 2 + DQ_WARPS;
constexpr int THREADS = (EPI_WARP0 + 4) * 32;        // 448 (TPR 2), 704 (TPR 4)
constexpr int BAR_BYTES = 256;
constexpr int SMEM = 1024 + STAGES * STAGE + BAR_BYTES;
constexpr int ACC_COLS = (BM / MS) * BN;             // 256: one tile's two accumulators
constexpr uint32_t TMEM_COLS = 512;                  // two tiles in flight
constexpr int BAND = 8;
// kind::f16: fp16 A and B, fp32 D, both operands K-major, M128 N128
constexpr uint32_t IDESC = (1u << 4) | (static_cast<uint32_t>(BN >> 3) << 17) |
                           (static_cast<uint32_t>(MS >> 4) << 24);
static_assert(2 * ACC_COLS <= static_cast<int>(TMEM_COLS), "two tiles of accumulators");
static_assert(SMEM <= 227 * 1024, "shared memory");
}  // namespace wq

struct WqParams {
    int n_tok, d_in, d_out, g, ng;
    int g_shift;          // log2(g) when g is a power of two, else -1
    int n_mt, n_nt, n_kb;
    long long n_tiles;
    const uint16_t* scales;
    const uint16_t* zeros;
    const __half* R;
    __half* Y;
    int* status;
};

__device__ __forceinline__ bool wq_tile(const WqParams& p, long long t, int& m0, int& n0) {
    const long long per_band = static_cast<long long>(wq::BAND) * p.n_nt;
    const int band = static_cast<int>(t / per_band);
    const int rem = static_cast<int>(t % per_band);
    const int band_m = min(wq::BAND, p.n_mt - band * wq::BAND);
    const int mt = band * wq::BAND + rem % band_m;
    const int nt = rem / band_m;
    m0 = mt * wq::BM;
    n0 = nt * wq::BN;
    return nt < p.n_nt;
}

// 8 codes (4 bytes, column 2i in the low nibble of byte i) -> 8 fp16 weights s*(q - z)
__device__ __forceinline__ uint4 dequant8(uint32_t v, __half2 z1024, __half2 s2) {
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        // byte i at bits 0-7 and 16-23; low nibble -> bits 0-3, high nibble -> bits 16-19
        const uint32_t y = __byte_perm(v, 0u, static_cast<uint32_t>(i | (4 << 4) | (i << 8) | (4 << 12)));
        const uint32_t bits = (y & 0x0000000Fu) | ((y >> 4) & 0x000F0000u) | 0x64006400u;
        __half2 h = *reinterpret_cast<const __half2*>(&bits);     // (1024 + q_lo, 1024 + q_hi)
        h = __hmul2(__hsub2(h, z1024), s2);                        // q - z exact, one rounding
        out[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

__global__ void __launch_bounds__(wq::THREADS, 1)
    w4a16_gemm_kernel(const __grid_constant__ CUtensorMap xmap,
                      const __grid_constant__ CUtensorMap cmap, const WqParams p) {
    if (status_bad(p.status)) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + wq::STAGES * wq::STAGE);
    uint64_t* full = bars;                           // [STAGES] X tile + codes landed
    uint64_t* bready = bars + wq::STAGES;            // [STAGES] weight tile written
    uint64_t* empty = bars + 2 * wq::STAGES;         // [STAGES] MMAs done reading
    uint64_t* acc_full = bars + 3 * wq::STAGES;      // [2]
    uint64_t* acc_empty = acc_full + 2;              // [2]
    uint64_t* drained = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* status = p.status;

    const int warp = warp_id(), lane = lane_id();
    if (threadIdx.x == 0) {
        for (int s = 0; s < wq::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&bready[s], wq::DQ_WARPS);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(drained, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&xmap);
        tma_prefetch_desc(&cmap);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, wq::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int it = 0;
            for (long long t = blockIdx.x; t < p.n_tiles && !*abort_flag; t += gridDim.x) {
                int m0, n0;
                if (!wq_tile(p, t, m0, n0)) continue;
                for (int kb = 0; kb < p.n_kb; ++kb, ++it) {
                    const int st = it % wq::STAGES;
                    if (!mbar_wait(&empty[st], ((it / wq::STAGES) & 1) ^ 1)) {
                        set_status(status, GPTQ_ERR_TIMEOUT);
                        *abort_flag = 1;
                        break;
                    }
                    uint8_t* sa = smem + st * wq::STAGE;
                    mbar_arrive_expect_tx(&full[st], wq::A_BYTES + wq::C_BYTES);
                    tma_load_2d(sa, &xmap, &full[st], kb * wq::BK, m0);
                    tma_load_2d(sa + wq::A_SUB, &xmap, &full[st], kb * wq::BK, m0 + wq::MS);
                    tma_load_2d(sa + wq::OFF_C, &cmap, &full[st], kb * (wq::BK / 2), n0);
                }
            }
            const int n_tail = it < wq::STAGES ? it : wq::STAGES;
            for (int k = it - n_tail; k < it; ++k) {
                if (!mbar_wait(&full[k % wq::STAGES], (k / wq::STAGES) & 1)) {
                    set_status(status, GPTQ_ERR_TIMEOUT);
                    *abort_flag = 1;
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int it = 0, lt = 0;
            bool ok = true;
            for (long long t = blockIdx.x; ok && t < p.n_tiles && !*abort_flag; t += gridDim.x) {
                int m0, n0;
                if (!wq_tile(p, t, m0, n0)) continue;
                const int b = lt & 1;
                if (!mbar_wait(&acc_empty[b], ((lt >> 1) & 1) ^ 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * wq::ACC_COLS);
                for (int kb = 0; kb < p.n_kb; ++kb, ++it) {
                    const int st = it % wq::STAGES;
                    const uint32_t par = (it / wq::STAGES) & 1;
                    if (!mbar_wait(&full[st], par) || !mbar_wait(&bready[st], par)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t s0 = smem_u32(smem + st * wq::STAGE);
#pragma unroll
                    for (int kk = 0; kk < wq::BK / 16; ++kk) {
                        // K-major rows of 128 B; a k-step of 16 fp16 is 32 B along the row
                        const uint64_t bd = umma_desc_sw128(s0 + wq::OFF_B + kk * 32, 16, 1024);
#pragma unroll
                        for (int h = 0; h < wq::BM / wq::MS; ++h) {
                            const uint64_t ad = umma_desc_sw128(s0 + h * wq::A_SUB + kk * 32, 16, 1024);
                            umma_f16(d_tmem + static_cast<uint32_t>(h * wq::BN), ad, bd, wq::IDESC,
                                     (kb > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    umma_commit(&empty[st]);
                }
                if (!ok) break;
                umma_commit(&acc_full[b]);
                ++lt;
            }
            if (!ok) {
                set_status(status, GPTQ_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            umma_commit(drained);
            if (!mbar_wait(drained, 0)) set_status(status, GPTQ_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp < wq::EPI_WARP0) {
        // ---------- dequantisers: TPR threads per weight row, 64/TPR codes each ----------
        constexpr int TPR = wq::TPR, CPT = 8 / TPR;              // 8-column chunks per thread
        const int j = (warp - 2) * 32 + lane;                    // 0 .. TPR*BN-1
        const int jr = j / TPR, hsel = j % TPR;                  // row of the tile, part
        const uint32_t row_off = static_cast<uint32_t>((jr >> 3) * 1024 + (jr & 7) * 128);
        // one group per k-block when groups are whole multiples of it: one scale and zero per
        // k-block, fetched a k-block ahead. Rows past d_out keep scale 0 and expand to zeros.
        const bool one_group = (p.g % wq::BK) == 0;
        int it = 0;
        bool stop = false;
        for (long long t = blockIdx.x; t < p.n_tiles && !stop; t += gridDim.x) {
            int m0, n0;
            if (!wq_tile(p, t, m0, n0)) continue;
            const int r = n0 + jr;
            const bool row_ok = r < p.d_out;
            const int64_t srow = static_cast<int64_t>(row_ok ? r : 0) * p.ng;
            int cur_k = -1;
            __half2 s2 = __float2half2_rn(0.0f), z2 = __float2half2_rn(1024.0f);
            uint16_t s_next = 0, z_next = 0;
            if (one_group && row_ok) {
                s_next = __ldg(p.scales + srow);
                z_next = __ldg(p.zeros + srow);
            }
            for (int kb = 0; kb < p.n_kb; ++kb, ++it) {
                const int st = it % wq::STAGES;
                if (one_group) {
                    s2 = __half2half2(__ushort_as_half(s_next));
                    z2 = __half2half2(__hadd(__float2half_rn(1024.0f), __ushort_as_half(z_next)));
                    const int kn = ((kb + 1) * wq::BK) / p.g;         // next k-block's group
                    if (row_ok && kb + 1 < p.n_kb) {
                        s_next = __ldg(p.scales + srow + kn);
                        z_next = __ldg(p.zeros + srow + kn);
                    }
                }
                int ok = 1;
                if (lane == 0) ok = mbar_wait(&full[st], (it / wq::STAGES) & 1) ? 1 : 0;
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok || __shfl_sync(0xffffffffu, *abort_flag, 0)) {
                    if (lane == 0 && !ok) {
                        set_status(status, GPTQ_ERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    stop = true;
                    break;
                }
                uint8_t* sa = smem + st * wq::STAGE;
                uint32_t cw[CPT];
                if constexpr (CPT == 4) {
                    const uint4 cv = *reinterpret_cast<const uint4*>(sa + wq::OFF_C + j * 16);
                    cw[0] = cv.x; cw[1] = cv.y; cw[2] = cv.z; cw[3] = cv.w;
                } else {
                    const uint2 cv = *reinterpret_cast<const uint2*>(sa + wq::OFF_C + j * 8);
                    cw[0] = cv.x; cw[1] = cv.y;
                }
                uint8_t* brow = sa + wq::OFF_B + row_off;
#pragma unroll
                for (int i = 0; i < CPT; ++i) {
                    const int c = CPT * hsel + i;                     // 8-column chunk
                    if (!one_group) {
                        const int col = kb * wq::BK + 8 * c;
                        const int k = p.g_shift >= 0 ? (col >> p.g_shift) : col / p.g;
                        if (k != cur_k) {
                            cur_k = k;
                            if (row_ok) {
                                const __half sh = __ushort_as_half(__ldg(p.scales + srow + k));
                                const __half zh = __ushort_as_half(__ldg(p.zeros + srow + k));
                                s2 = __half2half2(sh);
                                z2 = __half2half2(__hadd(__float2half_rn(1024.0f), zh));
                            }
                        }
                    }
                    *reinterpret_cast<uint4*>(brow + ((c ^ (jr & 7)) << 4)) = dequant8(cw[i], z2, s2);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bready[st]);
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue ----------------
        const int q = warp & 3;
        const uint32_t t_lane = static_cast<uint32_t>(32 * q) << 16;
        int lt = 0;
        bool stop = false;
        for (long long t = blockIdx.x; t < p.n_tiles && !stop; t += gridDim.x) {
            int m0, n0;
            if (!wq_tile(p, t, m0, n0)) continue;
            const int b = lt & 1;
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&acc_full[b], (lt >> 1) & 1) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok || __shfl_sync(0xffffffffu, *abort_flag, 0)) {
                if (lane == 0 && !ok) {
                    set_status(status, GPTQ_ERR_TIMEOUT);
                    *abort_flag = 1;
                }
                stop = true;
                break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int hc = 0; hc < (wq::BM / wq::MS) * (wq::BN / 32); ++hc) {
                const int h = hc / (wq::BN / 32), c = hc % (wq::BN / 32);
                const int row = m0 + h * wq::MS + 32 * q + lane;
                const bool row_ok = row < p.n_tok;
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + t_lane +
                                       static_cast<uint32_t>(b * wq::ACC_COLS + h * wq::BN + 32 * c),
                                   v);
                tmem_ld_wait();
                const int col0 = n0 + 32 * c;
                if (!row_ok || col0 >= p.d_out) continue;
                const int64_t off = static_cast<int64_t>(row) * p.d_out + col0;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (col0 + 8 * u >= p.d_out) break;
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * u + e]);
                    if (p.R) {
                        const uint4 rv = *reinterpret_cast<const uint4*>(p.R + off + 8 * u);
                        const __half2* rh = reinterpret_cast<const __half2*>(&rv);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 rf = __half22float2(rh[e]);
                            f[2 * e] += rf.x;
                            f[2 * e + 1] += rf.y;
                        }
                    }
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __half2 hv = __floats2half2_rn(f[2 * e], f[2 * e + 1]);
                        o[e] = *reinterpret_cast<const uint32_t*>(&hv);
                    }
                    *reinterpret_cast<uint4*>(p.Y + off + 8 * u) = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
            ++lt;
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, wq::TMEM_COLS);
}

// packed[r][p/2] holds codes[r][perm[p]] (identity without perm), even p in the low nibble
__global__ void w4a16_pack_kernel(const uint8_t* __restrict__ codes, int d_out, int d_in,
                                  const int32_t* __restrict__ perm, uint8_t* __restrict__ packed) {
    const int half = d_in / 2;
    const int64_t n = static_cast<int64_t>(d_out) * half;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = e / half;
        const int p = 2 * static_cast<int>(e - r * half);
        const uint8_t* row = codes + r * d_in;
        const int c0 = perm ? perm[p] : p, c1 = perm ? perm[p + 1] : p + 1;
        packed[e] = static_cast<uint8_t>((row[c0] & 0xF) | ((row[c1] & 0xF) << 4));
    }
}

// Xg[t][p] = X[t][perm[p]] (fp16), one row per block iteration
__global__ void gather_cols_kernel(const __half* __restrict__ X, int64_t n, int d,
                                   const int32_t* __restrict__ perm, __half* __restrict__ Xg) {
    for (int64_t t = blockIdx.x; t < n; t += gridDim.x) {
        const __half* src = X + t * d;
        __half* dst = Xg + t * d;
        for (int p = threadIdx.x; p < d; p += blockDim.x) dst[p] = src[perm[p]];
    }
}

// A[t][j] = fp16(silu(g) * u) with g = GU[t][j], u = GU[t][d_ff + j] (the gate and up halves of
// a row-stacked gate/up projection's output), silu(g) = g / (1 + e^-g) in fp32. Eight outputs
// per thread: 16-byte loads and stores (d_ff is a multiple of 8).
__global__ void __launch_bounds__(256) silu_mul_kernel(const __half* __restrict__ GU, int64_t n,
                                                       int d_ff, __half* __restrict__ A) {
    const int per_row = d_ff / 8;
    const int64_t total = n * per_row;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = e / per_row;
        const int j = static_cast<int>(e - t * per_row) * 8;
        const __half* row = GU + t * 2 * static_cast<int64_t>(d_ff);
        const uint4 gv = __ldcs(reinterpret_cast<const uint4*>(row + j));
        const uint4 uv = __ldcs(reinterpret_cast<const uint4*>(row + d_ff + j));
        const __half2* g2 = reinterpret_cast<const __half2*>(&gv);
        const __half2* u2 = reinterpret_cast<const __half2*>(&uv);
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 g = __half22float2(g2[i]);
            const float2 u = __half22float2(u2[i]);
            const float a0 = g.x / (1.0f + expf(-g.x)) * u.x;
            const float a1 = g.y / (1.0f + expf(-g.y)) * u.y;
            const __half2 h = __floats2half2_rn(a0, a1);
            o[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(A + t * d_ff + j) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Y[t] = fp16(X[t] / sqrt(mean(X[t]^2) + eps)) per row (the unit-weight RMS pre-norm of a
// block): one warp per row, fp32 sum of squares over 16-byte chunks, IEEE sqrt and division.
__global__ void __launch_bounds__(256) rms_norm_kernel(const __half* __restrict__ X, int64_t n,
                                                       int d, float eps, __half* __restrict__ Y) {
    const int lane = threadIdx.x & 31;
    const int64_t wstride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         t < n; t += wstride) {
        const uint4* row = reinterpret_cast<const uint4*>(X + t * d);
        float ss = 0.0f;
        for (int c = lane; c < d / 8; c += 32) {
            const uint4 v = row[c];
            const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __half22float2(h[i]);
                ss = fmaf(f.x, f.x, ss);
                ss = fmaf(f.y, f.y, ss);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float r = sqrtf(ss / static_cast<float>(d) + eps);
        uint4* out = reinterpret_cast<uint4*>(Y + t * d);
        for (int c = lane; c < d / 8; c += 32) {
            const uint4 v = row[c];
            const __half2* h = reinterpret_cast<const __half2*>(&v);
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __half22float2(h[i]);
                const __half2 q = __floats2half2_rn(f.x / r, f.y / r);
                o[i] = *reinterpret_cast<const uint32_t*>(&q);
            }
            out[c] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

static int g_wq_attr = 0;

gptq_status w4a16_launch(const __half* X, int64_t n, int d_in, const uint8_t* packed,
                         const uint16_t* scales, const uint16_t* zeros, int g, int d_out,
                         const int32_t* perm, const __half* R, __half* Y, __half* Xg,
                         int* status, cudaStream_t s) {
    if (!g_wq_attr) {
        GPTQ_CUDA_TRY(cudaFuncSetAttribute(w4a16_gemm_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, wq::SMEM));
        g_wq_attr = 1;
    }
    const __half* A = X;
    if (perm) {
        const int blocks = static_cast<int>(std::min<int64_t>(n, static_cast<int64_t>(num_sms()) * 16));
        gather_cols_kernel<<<blocks, 256, 0, s>>>(X, n, d_in, perm, Xg);
        GPTQ_LAUNCHED();
        A = Xg;
    }
    CUtensorMap xmap, cmap;
    GPTQ_TRY(encode_tensor_map_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, const_cast<__half*>(A),
                                  d_in, n, static_cast<uint64_t>(d_in) * 2, wq::BK, wq::MS,
                                  CU_TENSOR_MAP_SWIZZLE_128B));
    GPTQ_TRY(encode_tensor_map_2d(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8,
                                  const_cast<uint8_t*>(packed), d_in / 2, d_out,
                                  static_cast<uint64_t>(d_in) / 2, wq::BK / 2, wq::BN,
                                  CU_TENSOR_MAP_SWIZZLE_NONE));
    WqParams p;
    p.n_tok = static_cast<int>(n);
    p.d_in = d_in;
    p.d_out = d_out;
    p.g = g;
    p.ng = d_in / g;
    p.g_shift = -1;
    for (int sft = 3; sft < 17; ++sft)
        if ((1 << sft) == g) p.g_shift = sft;
    p.n_mt = static_cast<int>((n + wq::BM - 1) / wq::BM);
    p.n_nt = (d_out + wq::BN - 1) / wq::BN;
    p.n_kb = d_in / wq::BK;
    const int n_bands = (p.n_mt + wq::BAND - 1) / wq::BAND;
    p.n_tiles = static_cast<long long>(n_bands) * wq::BAND * p.n_nt;
    p.scales = scales;
    p.zeros = zeros;
    p.R = R;
    p.Y = Y;
    p.status = status;
    const long long useful = static_cast<long long>(p.n_mt) * p.n_nt;
    const int grid = static_cast<int>(std::max<long long>(1, std::min<long long>(useful, num_sms())));
    w4a16_gemm_kernel<<<grid, wq::THREADS, wq::SMEM, s>>>(xmap, cmap, p);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

gptq_status w4a16_pack_launch(const uint8_t* codes, int d_out, int d_in, const int32_t* perm,
                              uint8_t* packed, cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(d_out) * (d_in / 2);
    const int blocks = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>((n + 255) / 256, static_cast<int64_t>(num_sms()) * 16)));
    w4a16_pack_kernel<<<blocks, 256, 0, s>>>(codes, d_out, d_in, perm, packed);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

gptq_status rms_norm_launch(const __half* X, int64_t n, int d, float eps, __half* Y,
                            cudaStream_t s) {
    const int blocks = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>((n + 7) / 8, static_cast<int64_t>(num_sms()) * 16)));
    rms_norm_kernel<<<blocks, 256, 0, s>>>(X, n, d, eps, Y);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

gptq_status silu_mul_launch(const __half* GU, int64_t n, int d_ff, __half* A, cudaStream_t s) {
    const int64_t total = n * (d_ff / 8);
    const int blocks = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(num_sms()) * 8)));
    silu_mul_kernel<<<blocks, 256, 0, s>>>(GU, n, d_ff, A);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

}  // namespace gq

extern "C" {

gptq_status gptq_silu_mul(const void* GU, int64_t n_tokens, int d_ff, void* A, void* stream) {
    if (!GU || !A || n_tokens < 1 || d_ff < 8 || d_ff % 8) return GPTQ_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(GU) & 15) || (reinterpret_cast<uintptr_t>(A) & 15))
        return GPTQ_ERR_ARG;
    GPTQ_TRY(gq::check_device());
    return gq::silu_mul_launch(static_cast<const __half*>(GU), n_tokens, d_ff,
                               static_cast<__half*>(A), static_cast<cudaStream_t>(stream));
}

gptq_status gptq_rms_norm(const void* X, int64_t n_tokens, int d, float eps, void* Y,
                          void* stream) {
    if (!X || !Y || n_tokens < 1 || d < 8 || d % 8 || !(eps >= 0.0f)) return GPTQ_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(X) & 15) || (reinterpret_cast<uintptr_t>(Y) & 15))
        return GPTQ_ERR_ARG;
    GPTQ_TRY(gq::check_device());
    return gq::rms_norm_launch(static_cast<const __half*>(X), n_tokens, d, eps,
                               static_cast<__half*>(Y), static_cast<cudaStream_t>(stream));
}

size_t w4a16_linear_workspace(int64_t n_tokens, int d_in, int has_perm) {
    if (n_tokens < 0 || d_in < 1) return 0;
    return has_perm ? static_cast<size_t>(n_tokens) * d_in * 2 : 0;
}

gptq_status w4a16_pack(const uint8_t* codes, int d_out, int d_in, const int32_t* perm,
                       uint8_t* packed, void* stream) {
    if (!codes || !packed || d_out < 1 || d_in < 2 || d_in % 2) return GPTQ_ERR_ARG;
    GPTQ_TRY(gq::check_device());
    return gq::w4a16_pack_launch(codes, d_out, d_in, perm, packed,
                                 static_cast<cudaStream_t>(stream));
}

gptq_status w4a16_linear(const void* X, int64_t n_tokens, int d_in, const uint8_t* packed,
                         const uint16_t* scales, const uint16_t* zeros, int group_size,
                         int d_out, const int32_t* perm, const void* R, void* Y,
                         void* workspace, size_t workspace_bytes, int* status_dev,
                         void* stream) {
    if (!X || !packed || !scales || !zeros || !Y) return GPTQ_ERR_ARG;
    if (n_tokens < 1 || n_tokens >= (int64_t(1) << 31)) return GPTQ_ERR_ARG;
    if (d_in < 64 || d_in % 64 || d_in > 65536 || d_out < 8 || d_out % 8) return GPTQ_ERR_ARG;
    if (group_size < 8 || group_size % 8 || d_in % group_size) return GPTQ_ERR_ARG;
    auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    if (!al16(X) || !al16(packed) || !al16(Y) || (R && !al16(R))) return GPTQ_ERR_ARG;
    if (perm) {
        if (!workspace || !al16(workspace) ||
            workspace_bytes < w4a16_linear_workspace(n_tokens, d_in, 1))
            return workspace ? GPTQ_ERR_WORKSPACE : GPTQ_ERR_ARG;
    }
    GPTQ_TRY(gq::check_device());
    return gq::w4a16_launch(static_cast<const __half*>(X), n_tokens, d_in, packed, scales, zeros,
                            group_size, d_out, perm, static_cast<const __half*>(R),
                            static_cast<__half*>(Y), static_cast<__half*>(workspace), status_dev,
                            static_cast<cudaStream_t>(stream));
}

}  // extern "C"
