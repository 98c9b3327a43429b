// Calibration Hessian H += 2 * X^T X on the 5th-generation tensor cores.
//
// GPTQ deep-dive (hncyxsy.com/news/243429) §3.1 step 1: from the layer inputs X form
// H = 2XX^T (+ lambda*I, added later by the quantizer); gtnt.cn/news/115337 §4: collect each
// layer's Hessian from calibration forward passes. X here is [n_tokens x d_in] fp16, so the
// contraction runs over tokens and both MMA operands are read "MN-major" straight from X's
// row-major layout: a token row holds consecutive channels.
//
// Kernel design (clusters of two CTAs, one CTA per SM, persistent):
//   * output tiles of 256 x 256 (rows i, columns j) covering the upper triangle only, one per
//     CTA pair; work unit = (tile, token slice); units are ordered slice-major so pairs running
//     at the same time stream the same token rows (L2 reuse of X);
//   * warp 0 of each CTA: TMA producer - per 64-token k-block it loads its CTA's 128 rows
//     (2 boxes of 64 channels x 64 tokens, 128-byte swizzle) and its 128 of the tile's 256
//     columns (2 boxes) into a 6-stage ring;
//   * warp 1: TMEM allocation in both CTAs; in the leader CTA the single-thread issuer of
//     4 x tcgen05.mma.cta_group::2 (M256 N256 K16, fp16 in, fp32 accumulate) per k-block into
//     one of two 256-column TMEM accumulators, switching every CHUNK_KB k-blocks (512 tokens);
//   * warps 2-17 of each CTA: promotion epilogue - each warp owns 32 of its CTA's rows x 64
//     columns in 64 fp32 registers per thread. When a 512-token chunk is complete it reads its
//     slice from TMEM (tcgen05.ld) and adds it to the registers, then hands the accumulator
//     back. At the end of a unit it adds 2x the registers into H with vector atomics (fp32 add
//     in L2), so token slices of the same tile and successive calls accumulate in place.
// Why promote: the tensor cores' fp32 accumulation truncates, so a long accumulation drifts
// low (about -4e-5 relative over 8192 tokens, measured on B200); 512-token partial sums keep
// that drift near 2e-6 over 262144 tokens (1024-token sums: 5e-6) and the register sums round
// to nearest.
// Every mbarrier wait is bounded; on timeout the kernel records GPTQ_ERR_TIMEOUT, drains its
// own copies and MMAs, frees TMEM and returns.
#include <algorithm>

#include "common.cuh"

namespace gq {

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

// ---------------------------------------------------------------------------------------
// Pair kernel: two CTAs of a cluster share one 256 x 256 MMA tile (tcgen05 cta_group::2).
// CTA r of the pair loads only its halves: X[k:k+64, i0+128r : +128] (its 128 rows of the
// tile) and X[k:k+64, j0+128r : +128] (its 128 of the tile's 256 columns), 32 KB per k-block
// instead of the 48 KB a single-CTA 128 x 256 tile needs for the same flops per SM. The
// leader CTA (rank 0) issues M256 N256 K16 MMAs that read A by rows and B by columns from both
// CTAs' shared memory; each CTA's TMEM receives its 128 rows x 256 columns, and each CTA's
// warps promote and flush their own rows.
// Synchronisation: both CTAs' TMA loads complete on the leader's stage barrier (the leader
// expects both halves); the leader's MMA commits arrive, multicast, on the stage-free and
// accumulator-full barriers of both CTAs; both CTAs' promotion warps release an accumulator on
// the leader's barrier. No load is multicast: each CTA loads its own shared memory. A cluster
// barrier after set-up and another before exit keep either CTA from touching a CTA that has
// not initialised or has already left.
// ---------------------------------------------------------------------------------------
namespace hp2 {
constexpr int PT = 256;                             // pair tile edge
constexpr int BM = 128;                             // rows per CTA
constexpr int BNC = 128;                            // B columns loaded per CTA
constexpr int BN = 256;                             // accumulator columns
constexpr int BK = 64, STAGES = 6;
constexpr int CHUNK_KB = 8;                         // k-blocks per tensor-core partial sum
constexpr int BOX_BYTES = 64 * BK * 2;              // 64 channels x 64 tokens fp16 = 8 KB
constexpr int A_BYTES = BM * BK * 2;                // 16 KB
constexpr int B_BYTES = BNC * BK * 2;               // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;      // 32 KB per CTA
constexpr int EPI_WARPS = 16;
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
constexpr int THREADS = (2 + EPI_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = umma_idesc_f16_mn_mn(2 * BM, BN);
constexpr uint32_t LBO = BOX_BYTES;
constexpr uint32_t SBO = 1024;
}  // namespace hp2

// pair tile t (row-major over the upper triangle of an n_t x n_t grid) -> (ti, tj), ti <= tj
__device__ __forceinline__ void pair_tile(int t, int n_t, int& ti, int& tj) {
    int r = 0;
    while (t >= n_t - r) {
        t -= n_t - r;
        ++r;
    }
    ti = r;
    tj = r + t;
}

__device__ __forceinline__ bool pair_unit(const HessianParams& p, long long u, int& i0, int& j0,
                                          int& kb0, int& kb1) {
    const int split = static_cast<int>(u / p.n_tiles);
    const int t = static_cast<int>(u % p.n_tiles);
    int ti, tj;
    pair_tile(t, p.n_tj, ti, tj);
    i0 = ti * hp2::PT;
    j0 = tj * hp2::PT;
    kb0 = split * p.kblocks_per_unit;
    kb1 = min(kb0 + p.kblocks_per_unit, p.n_kblocks);
    return kb0 < kb1;
}

__global__ void __launch_bounds__(hp2::THREADS, 1)
    hessian_pair_kernel(const __grid_constant__ CUtensorMap xmap, const HessianParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* stages = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + hp2::STAGES * hp2::STAGE_BYTES);
    uint64_t* full = bars;                        // [STAGES] leader: both CTAs' bytes
    uint64_t* empty = bars + hp2::STAGES;         // [STAGES] each CTA: its stage is free again
    uint64_t* acc_full = bars + 2 * hp2::STAGES;  // [2] each CTA: a partial sum is ready
    uint64_t* acc_empty = acc_full + 2;           // [2] leader: both CTAs read the partial sum
    uint64_t* drained = acc_empty + 2;            // [1] leader
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = warp_id(), lane = lane_id();
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const long long cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < hp2::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2 * hp2::EPI_WARPS);
        }
        mbar_init(drained, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&xmap);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, hp2::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();     // both CTAs' barriers exist before either CTA signals the other's
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        if (lane == 0) {
            int it = 0;
            for (long long u = cluster; u < p.n_units && !*abort_flag; u += n_clusters) {
                int i0, j0, kb0, kb1;
                if (!pair_unit(p, u, i0, j0, kb0, kb1)) continue;
                const int ri = i0 + hp2::BM * static_cast<int>(rank);
                const int rj = j0 + hp2::BNC * static_cast<int>(rank);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int st = it % hp2::STAGES;
                    const uint32_t ph = (it / hp2::STAGES) & 1;
                    if (!mbar_wait(&empty[st], ph ^ 1)) {
                        set_status(p.status, GPTQ_ERR_TIMEOUT);
                        *abort_flag = 1;
                        break;
                    }
                    uint8_t* sa = stages + st * hp2::STAGE_BYTES;
                    uint8_t* sb = sa + hp2::A_BYTES;
                    const int y = kb * hp2::BK;
                    if (leader) mbar_arrive_expect_tx(&full[st], 2 * hp2::STAGE_BYTES);
                    const uint32_t fb = mapa_shared(smem_u32(&full[st]), 0);
                    tma_load_2d_pair(sa, &xmap, fb, ri, y);
                    tma_load_2d_pair(sa + hp2::BOX_BYTES, &xmap, fb, ri + 64, y);
                    tma_load_2d_pair(sb, &xmap, fb, rj, y);
                    tma_load_2d_pair(sb + hp2::BOX_BYTES, &xmap, fb, rj + 64, y);
                }
            }
            // the leader's stage barriers count both CTAs' bytes: once it has seen the last
            // stages complete, no copy of either CTA is still writing shared memory
            if (leader) {
                const int n_tail = it < hp2::STAGES ? it : hp2::STAGES;
                for (int k = it - n_tail; k < it; ++k) {
                    if (!mbar_wait(&full[k % hp2::STAGES], (k / hp2::STAGES) & 1)) {
                        set_status(p.status, GPTQ_ERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader) ----------------
        if (leader && lane == 0) {
            int it = 0, ch = 0;
            bool ok = true;
            for (long long u = cluster; ok && u < p.n_units && !*abort_flag; u += n_clusters) {
                int i0, j0, kb0, kb1;
                if (!pair_unit(p, u, i0, j0, kb0, kb1)) continue;
                for (int c0 = kb0; ok && c0 < kb1; c0 += hp2::CHUNK_KB, ++ch) {
                    const int c1 = min(c0 + hp2::CHUNK_KB, kb1);
                    const int b = ch & 1;
                    if (!mbar_wait(&acc_empty[b], ((ch >> 1) & 1) ^ 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * hp2::BN);
                    for (int kb = c0; kb < c1; ++kb, ++it) {
                        const int st = it % hp2::STAGES;
                        if (!mbar_wait(&full[st], (it / hp2::STAGES) & 1)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a0 = smem_u32(stages + st * hp2::STAGE_BYTES);
                        const uint32_t b0 = a0 + hp2::A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < hp2::BK / 16; ++kk) {
                            const uint64_t ad = umma_desc_sw128(a0 + kk * 2048, hp2::LBO, hp2::SBO);
                            const uint64_t bd = umma_desc_sw128(b0 + kk * 2048, hp2::LBO, hp2::SBO);
                            umma_f16_pair(d_tmem, ad, bd, hp2::IDESC, (kb > c0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit_pair_mc(&empty[st], 0x3);
                    }
                    if (!ok) break;
                    umma_commit_pair_mc(&acc_full[b], 0x3);
                }
            }
            if (!ok) {
                set_status(p.status, GPTQ_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            // every MMA must have finished before either CTA releases TMEM or leaves
            umma_commit_pair_mc(drained, 0x1);
            if (!mbar_wait(drained, 0)) set_status(p.status, GPTQ_ERR_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ---------------- promotion epilogue (both CTAs, their own rows) ----------------
        const int q = warp & 3;
        const int cs = (warp - 2) >> 2;
        const uint32_t t_lane = static_cast<uint32_t>(32 * q) << 16;
        float acc[64];
#pragma unroll
        for (int k = 0; k < 64; ++k) acc[k] = 0.0f;
        int ch = 0;
        bool stop = false;
        for (long long u = cluster; u < p.n_units && !stop; u += n_clusters) {
            int i0, j0, kb0, kb1;
            if (!pair_unit(p, u, i0, j0, kb0, kb1)) continue;
            for (int c0 = kb0; c0 < kb1; c0 += hp2::CHUNK_KB, ++ch) {
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
                const uint32_t t_col = static_cast<uint32_t>(b * hp2::BN + 64 * cs);
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
                if (lane == 0) {
                    // the leader's barrier: a local arrive for the leader's warps, a cluster-scope
                    // remote one for the peer's
                    if (leader) mbar_arrive(&acc_empty[b]);
                    else mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[b]), 0));
                }
            }
            if (stop) break;
            // unit complete: H[row][cols] += 2 * acc for this CTA's rows of the pair tile
            const int row = i0 + hp2::BM * static_cast<int>(rank) + 32 * q + lane;
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
    cluster_sync();     // neither CTA leaves while the pair's MMAs, copies or arrivals may touch it
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, hp2::TMEM_COLS);
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

static int g_pair_clusters = 0;   // co-resident clusters of two CTAs (one CTA per SM)

static gptq_status pair_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute& attr, int grid,
                               cudaStream_t s) {
    cfg = cudaLaunchConfig_t{};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(hp2::THREADS);
    cfg.dynamicSmemBytes = hp2::SMEM_BYTES;
    cfg.stream = s;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return GPTQ_OK;
}

gptq_status hessian_launch(float* H, int d, const void* X, int64_t n, int unit_tokens,
                           int* status, cudaStream_t s) {
    if (n <= 0) return GPTQ_OK;
    if (!g_hessian_attr_set) {
        GPTQ_CUDA_TRY(cudaFuncSetAttribute(hessian_pair_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           hp2::SMEM_BYTES));
        cudaLaunchConfig_t cfg;
        cudaLaunchAttribute attr;
        pair_config(cfg, attr, 2 * num_sms(), s);
        int nc = 0;
        GPTQ_CUDA_TRY(cudaOccupancyMaxActiveClusters(&nc, hessian_pair_kernel, &cfg));
        if (nc < 1) return GPTQ_ERR_UNSUPPORTED;
        g_pair_clusters = nc;
        g_hessian_attr_set = true;
    }
    const int slots = g_pair_clusters;
    const int n_t = (d + hp2::PT - 1) / hp2::PT;
    const int n_tiles = n_t * (n_t + 1) / 2;

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
        const int n_kblocks = static_cast<int>((nt + hp2::BK - 1) / hp2::BK);
        int kpu;
        if (unit_tokens > 0) {
            kpu = std::max(1, unit_tokens / hp2::BK);
        } else {
            // token slices per pair tile: the count (up to 64) that fills the last wave of
            // cluster slots best, keeping >= 32 k-blocks (2048 tokens) per unit when there are
            // enough tokens
            int best_s = 1;
            double best_eff = -1.0;
            for (int sp = 1; sp <= 64; ++sp) {
                const int k = (n_kblocks + sp - 1) / sp;
                if (sp > 1 && k < 32) break;
                const int sp_eff = (n_kblocks + k - 1) / k;
                const long long units = static_cast<long long>(n_tiles) * sp_eff;
                const long long waves = (units + slots - 1) / slots;
                const double eff = static_cast<double>(units) / static_cast<double>(waves * slots);
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
        p.n_tj = n_t;
        p.n_tiles = n_tiles;
        p.n_kblocks = n_kblocks;
        p.kblocks_per_unit = kpu;
        p.n_units = static_cast<long long>(n_tiles) * ((n_kblocks + kpu - 1) / kpu);
        p.status = status;
        const int clusters = static_cast<int>(std::min<long long>(p.n_units, slots));
        cudaLaunchConfig_t cfg;
        cudaLaunchAttribute attr;
        pair_config(cfg, attr, 2 * clusters, s);
        GPTQ_CUDA_TRY(cudaLaunchKernelEx(&cfg, hessian_pair_kernel, xmap, p));
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
