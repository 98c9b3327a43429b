// fp32-accurate GEMM on the 5th-generation tensor cores (tcgen05.mma kind::tf32).
//
// tf32 keeps 10 explicit mantissa bits. An fp32 operand x is written as hi + lo with
// hi = tf32(x) and lo = tf32(x - hi); the product a*b is taken as hi_a*hi_b + hi_a*lo_b +
// lo_a*hi_b, dropping lo_a*lo_b (about 2^-22 relative). Each partial product is exact in the
// tensor core and accumulates in fp32 in TMEM, so the result carries fp32-level error, at
// three tf32 MMAs per step instead of one. An operand that is already exact in tf32 (for
// example fp16 weights) is not split, and its pass is skipped.
//
// Kernel (persistent, one CTA per SM; output tiles of 128 x 128, k-blocks of 32):
//   warp 0      TMA producer: A tile 128 x 32 (K-major, 128-byte swizzle); B tile either
//               K-major 128 x 32, or MN-major as four 32 x 32 boxes (128-byte swizzle with
//               32-byte atoms, the layout the MMA needs for MN-major tf32); 3-stage ring.
//   warps 2-9   converters: split the fp32 tiles in shared memory into hi (in place) and lo,
//               then make the writes visible to the tensor core (proxy fence).
//   warp 1      TMEM allocator and MMA issuer: per k-block 4 k-steps x (1..3) MMAs
//               M128 N128 K8 into one of two 128-column TMEM accumulators.
//   warps 10-13 epilogue: tcgen05.ld, scale by alpha, stage 32 x 32 pieces in swizzled shared
//               memory and let TMA write them: a tensor reduce-add (C += alpha*A*B, the add
//               happens in L2) when beta = 1, a tensor store when beta = 0; or a dot with D.
// Every mbarrier wait is bounded; on timeout the kernel records GPTQ_ERR_TIMEOUT, drains its
// copies and MMAs, frees TMEM and returns.
#include <algorithm>

#include "tcgemm.cuh"

namespace gq {

namespace tg {
constexpr int BM = 128, BN = 128, BK = 32, STAGES = 3;
constexpr int TILE_A = BM * BK * 4;                  // 16 KB
constexpr int TILE_B = BN * BK * 4;                  // 16 KB
constexpr int OFF_A_LO = TILE_A;
constexpr int OFF_B = 2 * TILE_A;
constexpr int OFF_B_LO = 2 * TILE_A + TILE_B;
constexpr int STAGE = 2 * TILE_A + 2 * TILE_B;       // 64 KB
constexpr int CONV_WARPS = 8;
constexpr int EPI_WARP0 = 2 + CONV_WARPS;            // warps 10..13
constexpr int THREADS = (EPI_WARP0 + 4) * 32;        // 448
constexpr int EPI_BUF = 32 * 32 * 4;                // 4 KB: 32 rows x 32 fp32
constexpr int EPI_BYTES = 4 * 2 * EPI_BUF;           // 4 warps, double-buffered
constexpr int BAR_BYTES = 256;
constexpr int SMEM = 1024 + STAGES * STAGE + EPI_BYTES + BAR_BYTES;
constexpr uint32_t TMEM_COLS = 512;                  // two chunk accumulators + the sum
constexpr int BAND = 16;                             // m-tiles per raster band (L2 reuse)
// Promoted accumulation: the tensor cores' fp32 accumulation truncates, so a long K-chain
// drifts; K is cut into chunks of PROMO_KB k-blocks (128), each accumulated in TMEM from zero,
// and the chunks are summed with round-to-nearest fp32 additions by the epilogue: into a
// third TMEM region for the store epilogue (read, add, store back, 32 columns at a time), and
// straight into the dot for the dot epilogue.
constexpr int PROMO_KB = 4;
constexpr uint32_t SUM_COL = 2 * BN;                 // the running sum's TMEM columns
}  // namespace tg

// kind::tf32 instruction descriptor: A, B tf32 (format 2), D f32, A K-major, B K- or MN-major
__host__ __device__ constexpr uint32_t umma_idesc_tf32(int M, int N, bool b_mn) {
    return (1u << 4) | (2u << 7) | (2u << 10) | (0u << 15) | ((b_mn ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

struct TcParams {
    TcGemmArgs a;
    int beta_one;
    int n_mt, n_nt, n_kb;
    long long n_tiles;
};

__device__ __forceinline__ bool tc_tile(const TcParams& p, long long t, int& m0, int& n0) {
    // bands of BAND m-tiles; inside a band the m-tile varies fastest
    const long long per_band = static_cast<long long>(tg::BAND) * p.n_nt;
    const int band = static_cast<int>(t / per_band);
    const int rem = static_cast<int>(t % per_band);
    const int band_m = min(tg::BAND, p.n_mt - band * tg::BAND);
    const int mt = band * tg::BAND + rem % band_m;
    const int nt = rem / band_m;
    m0 = mt * tg::BM;
    n0 = nt * tg::BN;
    if (nt >= p.n_nt) return false;
    if (p.a.lower_only && m0 + tg::BM - 1 < n0) return false;
    return true;
}

template <bool B_K, int EPI, bool SPLIT_A, bool SPLIT_B, bool PRE>
__global__ void __launch_bounds__(tg::THREADS, 1)
    tcgemm_kernel(const __grid_constant__ CUtensorMap amap,
                  const __grid_constant__ CUtensorMap bmap,
                  const __grid_constant__ CUtensorMap cmap,
                  const __grid_constant__ CUtensorMap alomap,
                  const __grid_constant__ CUtensorMap blomap, const TcParams p) {
    pdl_wait();
    static_assert(!PRE || (SPLIT_A && SPLIT_B), "pre-split operands come in hi/lo pairs");
    // pre-split operands need no converter warps: the epilogue warps follow warp 1 directly
    // (warps 2..5 take TMEM lane quarters 2, 3, 0, 1, as warps 10..13 do)
    constexpr int EPI0 = PRE ? 2 : tg::EPI_WARP0;
    // accumulation chunks of the tile's K (a K of at most 128 is one chunk)
    const int ckb = tg::PROMO_KB;
    const int n_chunks = (p.n_kb + ckb - 1) / ckb;
    if (status_bad(p.a.status)) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float* epi_smem = reinterpret_cast<float*>(smem + tg::STAGES * tg::STAGE);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + tg::STAGES * tg::STAGE + tg::EPI_BYTES);
    uint64_t* full = bars;                          // [STAGES] TMA landed
    uint64_t* conv = bars + tg::STAGES;             // [STAGES] split done
    uint64_t* empty = bars + 2 * tg::STAGES;        // [STAGES] MMAs done reading
    uint64_t* acc_full = bars + 3 * tg::STAGES;     // [2]
    uint64_t* acc_empty = acc_full + 2;             // [2]
    uint64_t* drained = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* status = const_cast<int*>(p.a.status);

    const int warp = warp_id(), lane = lane_id();
    if (threadIdx.x == 0) {
        for (int s = 0; s < tg::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&conv[s], tg::CONV_WARPS);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(drained, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&bmap);
        if (EPI == TC_EPI_STORE) tma_prefetch_desc(&cmap);
        if (PRE) {
            tma_prefetch_desc(&alomap);
            tma_prefetch_desc(&blomap);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, tg::TMEM_COLS);
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
                if (!tc_tile(p, t, m0, n0)) continue;
                for (int kb = 0; kb < p.n_kb; ++kb, ++it) {
                    const int st = it % tg::STAGES;
                    if (!mbar_wait(&empty[st], ((it / tg::STAGES) & 1) ^ 1)) {
                        set_status(status, GPTQ_ERR_TIMEOUT);
                        *abort_flag = 1;
                        break;
                    }
                    uint8_t* sa = smem + st * tg::STAGE;
                    const int k0 = kb * tg::BK;
                    mbar_arrive_expect_tx(&full[st], (PRE ? 2 : 1) * (tg::TILE_A + tg::TILE_B));
                    tma_load_2d(sa, &amap, &full[st], k0, m0);
                    if (PRE) tma_load_2d(sa + tg::OFF_A_LO, &alomap, &full[st], k0, m0);
                    if (B_K) {
                        tma_load_2d(sa + tg::OFF_B, &bmap, &full[st], k0, n0);
                        if (PRE) tma_load_2d(sa + tg::OFF_B_LO, &blomap, &full[st], k0, n0);
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            tma_load_2d(sa + tg::OFF_B + c * 4096, &bmap, &full[st], n0 + 32 * c, k0);
                            if (PRE)
                                tma_load_2d(sa + tg::OFF_B_LO + c * 4096, &blomap, &full[st],
                                            n0 + 32 * c, k0);
                        }
                    }
                }
            }
            const int n_tail = it < tg::STAGES ? it : tg::STAGES;
            for (int k = it - n_tail; k < it; ++k) {
                if (!mbar_wait(&full[k % tg::STAGES], (k / tg::STAGES) & 1)) {
                    set_status(status, GPTQ_ERR_TIMEOUT);
                    *abort_flag = 1;
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t IDESC = umma_idesc_tf32(tg::BM, tg::BN, !B_K);
            int it = 0, lt = 0;   // lt counts accumulation chunks
            bool ok = true;
            for (long long t = blockIdx.x; ok && t < p.n_tiles && !*abort_flag; t += gridDim.x) {
                int m0, n0;
                if (!tc_tile(p, t, m0, n0)) continue;
              for (int ch = 0; ok && ch < n_chunks; ++ch) {
                const int b = lt & 1;
                if (!mbar_wait(&acc_empty[b], ((lt >> 1) & 1) ^ 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * tg::BN);
                const int kb_first = ch * ckb, kb_end = min(p.n_kb, kb_first + ckb);
                for (int kb = kb_first; kb < kb_end; ++kb, ++it) {
                    const int st = it % tg::STAGES;
                    if (!mbar_wait(PRE ? &full[st] : &conv[st], (it / tg::STAGES) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t s0 = smem_u32(smem + st * tg::STAGE);
#pragma unroll
                    for (int kk = 0; kk < tg::BK / 8; ++kk) {
                        // A: K-major rows of 128 B; a k-step of 8 tf32 is 32 B along the row
                        const uint64_t a_hi = umma_desc_sw128(s0 + kk * 32, 16, 1024);
                        const uint64_t a_lo = umma_desc_sw128(s0 + tg::OFF_A_LO + kk * 32, 16, 1024);
                        uint64_t b_hi, b_lo;
                        if (B_K) {
                            b_hi = umma_desc_sw128(s0 + tg::OFF_B + kk * 32, 16, 1024);
                            b_lo = umma_desc_sw128(s0 + tg::OFF_B_LO + kk * 32, 16, 1024);
                        } else {
                            // MN-major tf32: 128-byte swizzle with 32-byte atoms; 32-column
                            // chunks 4 KB apart, 4-row swizzle atoms 512 B apart, a k-step is
                            // 8 rows (1 KB)
                            b_hi = umma_desc_sw128_32b(s0 + tg::OFF_B + kk * 1024, 4096, 512);
                            b_lo = umma_desc_sw128_32b(s0 + tg::OFF_B_LO + kk * 1024, 4096, 512);
                        }
                        umma_tf32(d_tmem, a_hi, b_hi, IDESC, (kb > kb_first || kk > 0) ? 1u : 0u);
                        if (SPLIT_B) umma_tf32(d_tmem, a_hi, b_lo, IDESC, 1u);
                        if (SPLIT_A) umma_tf32(d_tmem, a_lo, b_hi, IDESC, 1u);
                    }
                    umma_commit(&empty[st]);
                }
                if (!ok) break;
                umma_commit(&acc_full[b]);
                ++lt;
              }
            }
            if (!ok) {
                set_status(status, GPTQ_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            umma_commit(drained);
            if (!mbar_wait(drained, 0)) set_status(status, GPTQ_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp < EPI0) {
        // ---------------- converters: fp32 -> tf32 hi (in place) + lo ----------------
        if constexpr (!PRE) {   // (pre-split operands arrive ready for the MMA)
            const int ct = (warp - 2) * 32 + lane;   // 0..255
            int it = 0;
            bool stop = false;
            for (long long t = blockIdx.x; t < p.n_tiles && !stop; t += gridDim.x) {
                int m0, n0;
                if (!tc_tile(p, t, m0, n0)) continue;
                for (int kb = 0; kb < p.n_kb; ++kb, ++it) {
                    const int st = it % tg::STAGES;
                    int ok = 1;
                    if (lane == 0) ok = mbar_wait(&full[st], (it / tg::STAGES) & 1) ? 1 : 0;
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok || __shfl_sync(0xffffffffu, *abort_flag, 0)) {
                        if (lane == 0 && !ok) {
                            set_status(status, GPTQ_ERR_TIMEOUT);
                            *abort_flag = 1;
                        }
                        stop = true;
                        break;
                    }
                    uint8_t* sa = smem + st * tg::STAGE;
                    if (SPLIT_A) {
                        float4* hi = reinterpret_cast<float4*>(sa);
                        float4* lo = reinterpret_cast<float4*>(sa + tg::OFF_A_LO);
    #pragma unroll
                        for (int j = 0; j < tg::TILE_A / 16 / 256; ++j) {
                            const int i = ct + 256 * j;
                            const float4 x = hi[i];
                            float4 h, l;
                            h.x = tf32_rna(x.x); l.x = tf32_rna(x.x - h.x);
                            h.y = tf32_rna(x.y); l.y = tf32_rna(x.y - h.y);
                            h.z = tf32_rna(x.z); l.z = tf32_rna(x.z - h.z);
                            h.w = tf32_rna(x.w); l.w = tf32_rna(x.w - h.w);
                            hi[i] = h;
                            lo[i] = l;
                        }
                    }
                    if (SPLIT_B) {
                        float4* hi = reinterpret_cast<float4*>(sa + tg::OFF_B);
                        float4* lo = reinterpret_cast<float4*>(sa + tg::OFF_B_LO);
    #pragma unroll
                        for (int j = 0; j < tg::TILE_B / 16 / 256; ++j) {
                            const int i = ct + 256 * j;
                            const float4 x = hi[i];
                            float4 h, l;
                            h.x = tf32_rna(x.x); l.x = tf32_rna(x.x - h.x);
                            h.y = tf32_rna(x.y); l.y = tf32_rna(x.y - h.y);
                            h.z = tf32_rna(x.z); l.z = tf32_rna(x.z - h.z);
                            h.w = tf32_rna(x.w); l.w = tf32_rna(x.w - h.w);
                            hi[i] = h;
                            lo[i] = l;
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&conv[st]);
                }
            }
            __syncwarp();
        }
    } else {
        // ---------------- epilogue ----------------
        const int q = warp & 3;
        const uint32_t t_lane = static_cast<uint32_t>(32 * q) << 16;
        float* stage_buf = epi_smem + (warp - EPI0) * 2 * (tg::EPI_BUF / 4);
        double dot = 0.0;
        int lt = 0, nbulk = 0;
        bool stop = false;
        // stage one 32 x 32 piece (this warp's rows, 32 columns) with the 128-byte swizzle of
        // the C map and send it out with a TMA store or reduce-add
        auto store_piece = [&](const float* v, int col0, int row0) {
            float* buf = stage_buf + (nbulk & 1) * (tg::EPI_BUF / 4);
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
            float4* rowp = reinterpret_cast<float4*>(buf + lane * 32);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                rowp[j ^ (lane & 7)] = make_float4(p.a.alpha * v[4 * j], p.a.alpha * v[4 * j + 1],
                                                   p.a.alpha * v[4 * j + 2], p.a.alpha * v[4 * j + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                if (p.beta_one) tma_reduce_add_2d(&cmap, buf, col0, row0);
                else tma_store_2d(&cmap, buf, col0, row0);
                bulk_commit();
            }
            ++nbulk;
        };
        for (long long t = blockIdx.x; t < p.n_tiles && !stop; t += gridDim.x) {
            int m0, n0;
            if (!tc_tile(p, t, m0, n0)) continue;
            const int row0 = m0 + 32 * q;
            const int row = row0 + lane;
          for (int ch = 0; ch < n_chunks && !stop; ++ch) {
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
            if constexpr (EPI == TC_EPI_STORE) {
                if (n_chunks > 1) {
                    const bool last = ch == n_chunks - 1;
                    // sum += this chunk, 32 columns at a time; the last chunk goes out instead
#pragma unroll 1
                    for (int c = 0; c < tg::BN / 32; ++c) {
                        const uint32_t cc = static_cast<uint32_t>(32 * c);
                        uint32_t r[32], a[32];
                        tmem_ld_32x32b_x32(tmem_base + t_lane + static_cast<uint32_t>(b * tg::BN) + cc, r);
                        if (ch > 0) tmem_ld_32x32b_x32(tmem_base + t_lane + tg::SUM_COL + cc, a);
                        tmem_ld_wait();
                        if (ch > 0) {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                r[i] = __float_as_uint(__uint_as_float(a[i]) + __uint_as_float(r[i]));
                        }
                        if (!last) {
                            tmem_st_32x32b_x32(tmem_base + t_lane + tg::SUM_COL + cc, r);
                        } else if (row0 < p.a.M && n0 + 32 * c < p.a.N) {   // warp-uniform
                            float v[32];
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
                            store_piece(v, n0 + 32 * c, row0);
                        }
                    }
                    if (!last) tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acc_empty[b]);
                    ++lt;
                    continue;
                }
            }
#pragma unroll 1
            for (int c = 0; c < tg::BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + t_lane + static_cast<uint32_t>(b * tg::BN + 32 * c), r);
                tmem_ld_wait();
                const int col0 = n0 + 32 * c;
                if (row0 >= p.a.M || col0 >= p.a.N) continue;       // warp-uniform
                if (EPI == TC_EPI_STORE) {
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
                    store_piece(v, col0, row0);
                } else if (row < p.a.M) {
                    const float* dp = p.a.D + static_cast<int64_t>(row) * p.a.ldd + col0;
                    float part = 0.0f;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        if (col0 + 4 * k < p.a.N) {
                            const float4 dv = *reinterpret_cast<const float4*>(dp + 4 * k);
                            part = fmaf(__uint_as_float(r[4 * k]), dv.x, part);
                            part = fmaf(__uint_as_float(r[4 * k + 1]), dv.y, part);
                            part = fmaf(__uint_as_float(r[4 * k + 2]), dv.z, part);
                            part = fmaf(__uint_as_float(r[4 * k + 3]), dv.w, part);
                        }
                    }
                    dot += static_cast<double>(part);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
            ++lt;
          }
        }
        if (EPI == TC_EPI_STORE) {
            if (lane == 0) bulk_wait_all();
        } else {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
            if (lane == 0 && dot != 0.0) atomicAdd(p.a.dot, static_cast<double>(p.a.alpha) * dot);
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, tg::TMEM_COLS);
}

template <bool B_K, int EPI, bool SA, bool SB, bool PRE>
static gptq_status launch_variant(const CUtensorMap& am, const CUtensorMap& bm,
                                  const CUtensorMap& cm, const CUtensorMap& alom,
                                  const CUtensorMap& blom, const TcParams& p, int grid,
                                  cudaStream_t s) {
    static bool attr = false;
    if (!attr) {
        GPTQ_CUDA_TRY(cudaFuncSetAttribute(tcgemm_kernel<B_K, EPI, SA, SB, PRE>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, tg::SMEM));
        attr = true;
    }
    constexpr int threads = PRE ? 6 * 32 : tg::THREADS;
    GPTQ_CUDA_TRY(launch_pdl(tcgemm_kernel<B_K, EPI, SA, SB, PRE>, dim3(grid), dim3(threads),
                             tg::SMEM, s, am, bm, cm, alom, blom, p));
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

template <bool B_K, int EPI>
static gptq_status launch_split(const CUtensorMap& am, const CUtensorMap& bm,
                                const CUtensorMap& cm, const TcParams& p, int grid, bool sa,
                                bool sb, cudaStream_t s) {
    if (sa && sb) return launch_variant<B_K, EPI, true, true, false>(am, bm, cm, am, bm, p, grid, s);
    if (sa) return launch_variant<B_K, EPI, true, false, false>(am, bm, cm, am, bm, p, grid, s);
    if (sb) return launch_variant<B_K, EPI, false, true, false>(am, bm, cm, am, bm, p, grid, s);
    return launch_variant<B_K, EPI, false, false, false>(am, bm, cm, am, bm, p, grid, s);
}

static gptq_status check_args(const TcGemmArgs& a, int epi) {
    if (a.lda % 4 || a.ldb % 4 || a.N % 4 || (epi == TC_EPI_STORE && a.ldc % 4) ||
        (epi == TC_EPI_DOT && a.ldd % 4))
        return GPTQ_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(a.A) & 15) || (reinterpret_cast<uintptr_t>(a.B) & 15))
        return GPTQ_ERR_ARG;
    // the stored result goes out through TMA: beta must be 0 (store) or 1 (reduce-add)
    if (epi == TC_EPI_STORE &&
        ((a.beta != 0.0f && a.beta != 1.0f) || (reinterpret_cast<uintptr_t>(a.C) & 15)))
        return GPTQ_ERR_ARG;
    return GPTQ_OK;
}

static gptq_status encode_a(CUtensorMap* m, const float* A, const TcGemmArgs& a, int lda) {
    return encode_tensor_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, const_cast<float*>(A), a.K,
                                a.M, static_cast<uint64_t>(lda) * 4, 32, 128,
                                CU_TENSOR_MAP_SWIZZLE_128B);
}
static gptq_status encode_a(CUtensorMap* m, const float* A, const TcGemmArgs& a) {
    return encode_a(m, A, a, a.lda);
}

static gptq_status encode_b(CUtensorMap* m, const float* B, const TcGemmArgs& a, bool b_kmajor,
                            int ldb) {
    if (b_kmajor)
        return encode_tensor_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, const_cast<float*>(B),
                                    a.K, a.N, static_cast<uint64_t>(ldb) * 4, 32, 128,
                                    CU_TENSOR_MAP_SWIZZLE_128B);
    return encode_tensor_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, const_cast<float*>(B), a.N,
                                a.K, static_cast<uint64_t>(ldb) * 4, 32, 32,
                                CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B);
}
static gptq_status encode_b(CUtensorMap* m, const float* B, const TcGemmArgs& a, bool b_kmajor) {
    return encode_b(m, B, a, b_kmajor, a.ldb);
}

static gptq_status encode_c(CUtensorMap* m, const TcGemmArgs& a) {
    return encode_tensor_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.C, a.N, a.M,
                                static_cast<uint64_t>(a.ldc) * 4, 32, 32,
                                CU_TENSOR_MAP_SWIZZLE_128B);
}

static TcParams make_params(const TcGemmArgs& a, int& grid) {
    TcParams p;
    p.a = a;
    p.beta_one = (a.beta == 1.0f) ? 1 : 0;
    p.n_mt = (a.M + tg::BM - 1) / tg::BM;
    p.n_nt = (a.N + tg::BN - 1) / tg::BN;
    p.n_kb = (a.K + tg::BK - 1) / tg::BK;
    const int n_bands = (p.n_mt + tg::BAND - 1) / tg::BAND;
    p.n_tiles = static_cast<long long>(n_bands) * tg::BAND * p.n_nt;
    long long useful = static_cast<long long>(p.n_mt) * p.n_nt;
    if (a.lower_only) useful = useful / 2 + p.n_mt;
    long long cap = num_sms();
    if (a.max_ctas > 0) cap = std::min<long long>(cap, a.max_ctas);
    grid = static_cast<int>(std::max<long long>(1, std::min<long long>(useful, cap)));
    return p;
}

gptq_status tcgemm_launch(const TcGemmArgs& a, bool b_kmajor, int epi, bool split_a, bool split_b,
                          cudaStream_t s) {
    if (a.M <= 0 || a.N <= 0 || a.K <= 0) return GPTQ_OK;
    GPTQ_TRY(check_args(a, epi));
    CUtensorMap am, bm, cm;
    GPTQ_TRY(encode_a(&am, a.A, a));
    GPTQ_TRY(encode_b(&bm, a.B, a, b_kmajor));
    if (epi == TC_EPI_STORE) GPTQ_TRY(encode_c(&cm, a));
    else cm = am;   // unused by the dot epilogue
    int grid;
    const TcParams p = make_params(a, grid);
    if (b_kmajor) {
        return epi == TC_EPI_STORE
                   ? launch_split<true, TC_EPI_STORE>(am, bm, cm, p, grid, split_a, split_b, s)
                   : launch_split<true, TC_EPI_DOT>(am, bm, cm, p, grid, split_a, split_b, s);
    }
    return epi == TC_EPI_STORE
               ? launch_split<false, TC_EPI_STORE>(am, bm, cm, p, grid, split_a, split_b, s)
               : launch_split<false, TC_EPI_DOT>(am, bm, cm, p, grid, split_a, split_b, s);
}

gptq_status tcgemm_presplit_launch(const TcGemmArgs& a, cudaStream_t s, bool b_kmajor) {
    if (a.M <= 0 || a.N <= 0 || a.K <= 0) return GPTQ_OK;
    GPTQ_TRY(check_args(a, TC_EPI_STORE));
    const int lda_lo = a.lda_lo > 0 ? a.lda_lo : a.lda;
    const int ldb_lo = a.ldb_lo > 0 ? a.ldb_lo : a.ldb;
    if (!a.A_lo || !a.B_lo || (reinterpret_cast<uintptr_t>(a.A_lo) & 15) ||
        (reinterpret_cast<uintptr_t>(a.B_lo) & 15) || lda_lo % 4 || ldb_lo % 4)
        return GPTQ_ERR_ARG;
    CUtensorMap am, bm, cm, alom, blom;
    GPTQ_TRY(encode_a(&am, a.A, a));
    GPTQ_TRY(encode_a(&alom, a.A_lo, a, lda_lo));
    GPTQ_TRY(encode_b(&bm, a.B, a, b_kmajor));
    GPTQ_TRY(encode_b(&blom, a.B_lo, a, b_kmajor, ldb_lo));
    GPTQ_TRY(encode_c(&cm, a));
    int grid;
    const TcParams p = make_params(a, grid);
    if (b_kmajor)
        return launch_variant<true, TC_EPI_STORE, true, true, true>(am, bm, cm, alom, blom, p,
                                                                    grid, s);
    return launch_variant<false, TC_EPI_STORE, true, true, true>(am, bm, cm, alom, blom, p, grid, s);
}

__global__ void tf32_split_kernel(const float* src, float* hi, float* __restrict__ lo, int rows,
                                  int cols, int ld, int ld_hi, int ld_lo, int upper) {
    pdl_wait();
    for (int r = blockIdx.x; r < rows; r += gridDim.x) {
        const int64_t row = static_cast<int64_t>(r) * ld;
        const int64_t row_hi = static_cast<int64_t>(r) * ld_hi;
        const int64_t row_lo = static_cast<int64_t>(r) * ld_lo;
        for (int c = (upper ? (r & ~3) : 0) + 4 * static_cast<int>(threadIdx.x); c < cols;
             c += 4 * blockDim.x) {
            const float4 x = *reinterpret_cast<const float4*>(src + row + c);
            float4 h, l;
            h.x = tf32_rna(x.x); l.x = tf32_rna(x.x - h.x);
            h.y = tf32_rna(x.y); l.y = tf32_rna(x.y - h.y);
            h.z = tf32_rna(x.z); l.z = tf32_rna(x.z - h.z);
            h.w = tf32_rna(x.w); l.w = tf32_rna(x.w - h.w);
            *reinterpret_cast<float4*>(hi + row_hi + c) = h;
            *reinterpret_cast<float4*>(lo + row_lo + c) = l;
        }
    }
}

gptq_status tcgemm_split_launch(const float* src, float* hi, float* lo, int rows, int cols, int ld,
                                bool upper, cudaStream_t s, int ld_hi, int ld_lo) {
    if (rows <= 0 || cols <= 0) return GPTQ_OK;
    if (ld_hi <= 0) ld_hi = ld;
    if (ld_lo <= 0) ld_lo = ld;
    if (cols % 4 || ld % 4 || ld_hi % 4 || ld_lo % 4 || (upper && (ld_lo != ld || ld_hi != ld)))
        return GPTQ_ERR_ARG;
    const int blocks = std::min(rows, num_sms() * 8);
    GPTQ_CUDA_TRY(launch_pdl(tf32_split_kernel, dim3(blocks), dim3(256), 0, s, src, hi, lo, rows,
                             cols, ld, ld_hi, ld_lo, upper ? 1 : 0));
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

}  // namespace gq
