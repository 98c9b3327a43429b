// Calibration Hessian H += 2 * X^T X on the 5th-generation tensor cores.
//
// GPTQ deep-dive (hncyxsy.com/news/243429) §3.1 step 1: from the layer inputs X form
// H = 2XX^T (+ lambda*I, added later by the quantizer); gtnt.cn/news/115337 §4: collect each
// layer's Hessian from calibration forward passes. X here is [n_tokens x d_in] fp16, so the
// contraction runs over tokens and both MMA operands are read "MN-major" straight from X's
// row-major layout: a token row holds consecutive channels.
//
// Kernel design (one CTA per SM, persistent):
//   * output tiles of 128 x 256 (rows i, columns j) covering the upper triangle only;
//     work unit = (tile, token slice); units are ordered slice-major so CTAs running at the
//     same time stream the same token rows (L2 reuse of X);
//   * warp 0: TMA producer — per 64-token k-block it loads X[k:k+64, i0:i0+128] (2 boxes) and
//     X[k:k+64, j0:j0+256] (4 boxes) of 64 channels x 64 tokens with 128-byte swizzle into a
//     4-stage ring;
//   * warp 1: TMEM allocator and single-thread MMA issuer — 4 x tcgen05.mma (M128 N256 K16,
//     fp16 in, fp32 accumulate) per k-block into one of two 256-column TMEM accumulators,
//     switching accumulator every CHUNK_KB k-blocks (256 tokens);
//   * warps 2-17: promotion epilogue — each warp owns 32 rows x 64 columns of the tile in 64
//     fp32 registers per thread. When a 256-token chunk is complete it reads its slice from
//     TMEM (tcgen05.ld) and adds it to the registers, then hands the accumulator back. At the
//     end of a unit it adds 2x the registers into H with vector atomics (fp32 add in L2), so
//     token slices of the same tile and successive calls accumulate in place.
// Why promote: the tensor cores' fp32 accumulation truncates, so a long accumulation drifts
// low (about -4e-5 relative over 8192 tokens, measured on B200); 256-token partial sums keep
// that drift near 1e-6 and the register sums round to nearest.
// Every mbarrier wait is bounded; on timeout the kernel records GPTQ_ERR_TIMEOUT, drains its
// own copies and MMAs, frees TMEM and returns.
#include <algorithm>

#include "common.cuh"

namespace gq {

namespace hs {
constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int CHUNK_KB = 4;                         // k-blocks per tensor-core partial sum
constexpr int BOX_BYTES = 64 * BK * 2;              // 64 channels x 64 tokens fp16 = 8 KB
constexpr int A_BYTES = BM * BK * 2;                // 16 KB
constexpr int B_BYTES = BN * BK * 2;                // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;      // 48 KB
constexpr int EPI_WARPS = 16;                       // 4 lane quadrants x 4 column slices of 64
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
constexpr int THREADS = (2 + EPI_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = umma_idesc_f16_mn_mn(BM, BN);
// canonical MN-major SW128 operand: 64-element (128 B) chunks along M/N are one TMA box apart,
// groups of 8 tokens are 8 x 128 B apart
constexpr uint32_t LBO = BOX_BYTES;
constexpr uint32_t SBO = 1024;
}  // namespace hs

struct HessianParams {
    float* H;
    int d;
    int n_tj;
    int n_tiles;
    int n_kblocks;
    int kblocks_per_unit;
    long long n_units;
    int* status;
};

// tile t (row-major over the upper-triangle tile list) -> (ti, tj); row ti holds
// tj in [ti/2, n_tj)
__device__ __forceinline__ void hessian_tile(int t, int n_tj, int& ti, int& tj) {
    int r = 0;
    while (true) {
        const int cnt = n_tj - r / 2;
        if (t < cnt) {
            ti = r;
            tj = r / 2 + t;
            return;
        }
        t -= cnt;
        ++r;
    }
}

__device__ __forceinline__ bool unit_range(const HessianParams& p, long long u, int& i0, int& j0,
                                           int& kb0, int& kb1) {
    const int split = static_cast<int>(u / p.n_tiles);
    const int t = static_cast<int>(u % p.n_tiles);
    int ti, tj;
    hessian_tile(t, p.n_tj, ti, tj);
    i0 = ti * hs::BM;
    j0 = tj * hs::BN;
    kb0 = split * p.kblocks_per_unit;
    kb1 = min(kb0 + p.kblocks_per_unit, p.n_kblocks);
    return kb0 < kb1;
}

__global__ void __launch_bounds__(hs::THREADS, 1)
    hessian_tc_kernel(const __grid_constant__ CUtensorMap xmap, const HessianParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* stages = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + hs::STAGES * hs::STAGE_BYTES);
    uint64_t* full = bars;                      // [STAGES]
    uint64_t* empty = bars + hs::STAGES;        // [STAGES]
    uint64_t* acc_full = bars + 2 * hs::STAGES; // [2]
    uint64_t* acc_empty = acc_full + 2;         // [2]
    uint64_t* drained = acc_empty + 2;          // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < hs::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], hs::EPI_WARPS);
        }
        mbar_init(drained, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&xmap);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, hs::TMEM_COLS);
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
            for (long long u = blockIdx.x; u < p.n_units && !*abort_flag; u += gridDim.x) {
                int i0, j0, kb0, kb1;
                if (!unit_range(p, u, i0, j0, kb0, kb1)) continue;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int st = it % hs::STAGES;
                    const uint32_t ph = (it / hs::STAGES) & 1;
                    if (!mbar_wait(&empty[st], ph ^ 1)) {
                        set_status(p.status, GPTQ_ERR_TIMEOUT);
                        *abort_flag = 1;
                        break;
                    }
                    uint8_t* sa = stages + st * hs::STAGE_BYTES;
                    uint8_t* sb = sa + hs::A_BYTES;
                    const int y = kb * hs::BK;
                    mbar_arrive_expect_tx(&full[st], hs::STAGE_BYTES);
                    tma_load_2d(sa, &xmap, &full[st], i0, y);
                    tma_load_2d(sa + hs::BOX_BYTES, &xmap, &full[st], i0 + 64, y);
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        tma_load_2d(sb + m * hs::BOX_BYTES, &xmap, &full[st], j0 + 64 * m, y);
                }
            }
            // no copy may still be writing this CTA's shared memory when it exits
            const int n_tail = it < hs::STAGES ? it : hs::STAGES;
            for (int k = it - n_tail; k < it; ++k) {
                if (!mbar_wait(&full[k % hs::STAGES], (k / hs::STAGES) & 1)) {
                    set_status(p.status, GPTQ_ERR_TIMEOUT);
                    *abort_flag = 1;
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int it = 0, ch = 0;
            bool ok = true;
            for (long long u = blockIdx.x; ok && u < p.n_units && !*abort_flag; u += gridDim.x) {
                int i0, j0, kb0, kb1;
                if (!unit_range(p, u, i0, j0, kb0, kb1)) continue;
                for (int c0 = kb0; ok && c0 < kb1; c0 += hs::CHUNK_KB, ++ch) {
                    const int c1 = min(c0 + hs::CHUNK_KB, kb1);
                    const int b = ch & 1;
                    if (!mbar_wait(&acc_empty[b], ((ch >> 1) & 1) ^ 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * hs::BN);
                    for (int kb = c0; kb < c1; ++kb, ++it) {
                        const int st = it % hs::STAGES;
                        if (!mbar_wait(&full[st], (it / hs::STAGES) & 1)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a0 = smem_u32(stages + st * hs::STAGE_BYTES);
                        const uint32_t b0 = a0 + hs::A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < hs::BK / 16; ++kk) {
                            const uint64_t ad = umma_desc_sw128(a0 + kk * 2048, hs::LBO, hs::SBO);
                            const uint64_t bd = umma_desc_sw128(b0 + kk * 2048, hs::LBO, hs::SBO);
                            umma_f16(d_tmem, ad, bd, hs::IDESC, (kb > c0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit(&empty[st]);
                    }
                    if (!ok) break;
                    umma_commit(&acc_full[b]);
                }
            }
            if (!ok) {
                set_status(p.status, GPTQ_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            // every MMA must have finished before TMEM is released
            umma_commit(drained);
            if (!mbar_wait(drained, 0)) set_status(p.status, GPTQ_ERR_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ---------------- promotion epilogue ----------------
        // control flow stays warp-uniform: tcgen05.ld below is a .sync.aligned instruction
        const int q = warp & 3;                // TMEM lane quadrant this warp may access
        const int cs = (warp - 2) >> 2;        // column slice [64*cs, 64*cs + 64)
        const uint32_t t_lane = static_cast<uint32_t>(32 * q) << 16;
        float acc[64];
#pragma unroll
        for (int k = 0; k < 64; ++k) acc[k] = 0.0f;
        int ch = 0;
        bool stop = false;
        for (long long u = blockIdx.x; u < p.n_units && !stop; u += gridDim.x) {
            int i0, j0, kb0, kb1;
            if (!unit_range(p, u, i0, j0, kb0, kb1)) continue;
            for (int c0 = kb0; c0 < kb1; c0 += hs::CHUNK_KB, ++ch) {
                const int b = ch & 1;
                int ok = 1;
                if (lane == 0) ok = mbar_wait(&acc_full[b], (ch >> 1) & 1) ? 1 : 0;
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok || __shfl_sync(0xffffffffu, *abort_flag, 0)) {
                    if (lane == 0 && !ok) {
                        set_status(p.status, GPTQ_ERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    stop = true;
                    break;
                }
                tc_fence_after();
                const uint32_t t_col = static_cast<uint32_t>(b * hs::BN + 64 * cs);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t r[16];
                    tmem_ld_32x32b_x16(tmem_base + t_lane + t_col + 16 * j, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < 16; ++k) acc[16 * j + k] += __uint_as_float(r[k]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[b]);
            }
            if (stop) break;
            // unit complete: H[row][cols] += 2 * acc
            const int row = i0 + 32 * q + lane;
            const int col0 = j0 + 64 * cs;
            if (row < p.d) {
                float* hrow = p.H + static_cast<int64_t>(row) * p.d;
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int col = col0 + 4 * k;
                    if (col < p.d) {
                        atomicAdd(reinterpret_cast<float4*>(hrow + col),
                                  make_float4(2.0f * acc[4 * k], 2.0f * acc[4 * k + 1],
                                              2.0f * acc[4 * k + 2], 2.0f * acc[4 * k + 3]));
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < 64; ++k) acc[k] = 0.0f;
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, hs::TMEM_COLS);
}

// H_out[i][j] = H[min(i,j)][max(i,j)]
__global__ void mirror_upper_kernel(const float* __restrict__ H, float* __restrict__ out, int d) {
    __shared__ float tile[32][33];
    const int bi = blockIdx.y * 32, bj = blockIdx.x * 32;
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    if (bi <= bj) {
        for (int k = ty; k < 32; k += 8) {
            const int i = bi + k, j = bj + tx;
            if (i < d && j < d) out[static_cast<int64_t>(i) * d + j] =
                (j >= i) ? H[static_cast<int64_t>(i) * d + j] : H[static_cast<int64_t>(j) * d + i];
        }
    } else {
        // strictly below the diagonal: transpose the upper tile (bj, bi) through shared memory
        for (int k = ty; k < 32; k += 8) {
            const int i = bj + k, j = bi + tx;
            tile[k][tx] = (i < d && j < d) ? H[static_cast<int64_t>(i) * d + j] : 0.0f;
        }
        __syncthreads();
        for (int k = ty; k < 32; k += 8) {
            const int i = bi + k, j = bj + tx;
            if (i < d && j < d) out[static_cast<int64_t>(i) * d + j] = tile[tx][k];
        }
    }
}

static bool g_hessian_attr_set = false;

gptq_status hessian_launch(float* H, int d, const void* X, int64_t n, int unit_tokens,
                           int* status, cudaStream_t s) {
    if (n <= 0) return GPTQ_OK;
    if (!g_hessian_attr_set) {
        GPTQ_CUDA_TRY(cudaFuncSetAttribute(hessian_tc_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           hs::SMEM_BYTES));
        g_hessian_attr_set = true;
    }
    const int sms = num_sms();
    const int n_ti = (d + hs::BM - 1) / hs::BM;
    const int n_tj = (d + hs::BN - 1) / hs::BN;
    int n_tiles = 0;
    for (int ti = 0; ti < n_ti; ++ti) n_tiles += std::max(0, n_tj - ti / 2);

    // token coordinates are 32-bit: feed very long inputs in slices
    const int64_t kMaxTokens = int64_t(1) << 30;
    for (int64_t t0 = 0; t0 < n; t0 += kMaxTokens) {
        const int64_t nt = std::min(kMaxTokens, n - t0);
        const void* Xs = static_cast<const uint8_t*>(X) + t0 * static_cast<int64_t>(d) * 2;
        CUtensorMap xmap;
        GPTQ_TRY(encode_tensor_map_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                                      const_cast<void*>(Xs), d, nt,
                                      static_cast<uint64_t>(d) * 2, 64, 64,
                                      CU_TENSOR_MAP_SWIZZLE_128B));
        const int n_kblocks = static_cast<int>((nt + hs::BK - 1) / hs::BK);
        int kpu;
        if (unit_tokens > 0) {
            kpu = std::max(1, unit_tokens / hs::BK);
        } else {
            // token slices per tile: the count (up to 64) that fills the last wave of SMs best,
            // keeping >= 32 k-blocks (2048 tokens) per unit when there are enough tokens
            int best_s = 1;
            double best_eff = -1.0;
            for (int sp = 1; sp <= 64; ++sp) {
                const int k = (n_kblocks + sp - 1) / sp;
                if (sp > 1 && k < 32) break;
                const int sp_eff = (n_kblocks + k - 1) / k;
                const long long units = static_cast<long long>(n_tiles) * sp_eff;
                const long long waves = (units + sms - 1) / sms;
                const double eff = static_cast<double>(units) / static_cast<double>(waves * sms);
                if (eff > best_eff + 1e-3) {
                    best_eff = eff;
                    best_s = sp_eff;
                }
            }
            kpu = (n_kblocks + best_s - 1) / best_s;
        }
        HessianParams p;
        p.H = H;
        p.d = d;
        p.n_tj = n_tj;
        p.n_tiles = n_tiles;
        p.n_kblocks = n_kblocks;
        p.kblocks_per_unit = kpu;
        p.n_units = static_cast<long long>(n_tiles) * ((n_kblocks + kpu - 1) / kpu);
        p.status = status;
        const int grid = static_cast<int>(std::min<long long>(p.n_units, sms));
        hessian_tc_kernel<<<grid, hs::THREADS, hs::SMEM_BYTES, s>>>(xmap, p);
        GPTQ_LAUNCHED();
    }
    return GPTQ_OK;
}

gptq_status mirror_upper_launch(const float* H, float* out, int d, cudaStream_t s) {
    const dim3 grid((d + 31) / 32, (d + 31) / 32), block(32, 8);
    mirror_upper_kernel<<<grid, block, 0, s>>>(H, out, d);
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

}  // namespace gq
