// C ABI of the library: argument checks, workspace layout, stage orchestration, stage timing
// and the Hessian handle. Every numeric step runs in this library's kernels.
#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "internal.cuh"
#include "tcgemm.cuh"

namespace gq {

// ---------------------------------------------------------------------------------------
// host helpers
// ---------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

gptq_status encode_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, void* base,
                                 uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                                 uint32_t box_inner, uint32_t box_outer,
                                 CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return GPTQ_ERR_CUDA;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, dtype, 2, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GPTQ_OK : GPTQ_ERR_CUDA;
}

gptq_status check_device() {
    int dev = 0;
    GPTQ_CUDA_TRY(cudaGetDevice(&dev));
    int major = 0, minor = 0;
    GPTQ_CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    GPTQ_CUDA_TRY(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    return (major == 10 && minor == 0) ? GPTQ_OK : GPTQ_ERR_UNSUPPORTED;
}

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

static std::atomic<unsigned long long> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
static inline size_t round256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

// ---------------------------------------------------------------------------------------
// stage timing
// ---------------------------------------------------------------------------------------
constexpr int kStages = 7;
struct Profiler {
    bool on = false;
    std::vector<cudaEvent_t> pool;
    std::vector<int> stage_of;  // one entry per recorded (start, stop) pair
    size_t used = 0;
    float last[kStages] = {0};
    std::mutex mu;

    cudaEvent_t ev() {
        if (used == pool.size()) {
            cudaEvent_t e;
            cudaEventCreate(&e);
            pool.push_back(e);
        }
        return pool[used++];
    }
};
static Profiler g_prof;

struct StageTimer {
    cudaStream_t s;
    int stage = -1;
    explicit StageTimer(cudaStream_t st) : s(st) {}
    void begin(int stg) {
        if (!g_prof.on) return;
        stage = stg;
        cudaEventRecord(g_prof.ev(), s);
    }
    void end() {
        if (!g_prof.on || stage < 0) return;
        cudaEventRecord(g_prof.ev(), s);
        g_prof.stage_of.push_back(stage);
        stage = -1;
    }
};

static void profile_reset() {
    g_prof.used = 0;
    g_prof.stage_of.clear();
}

static void profile_collect() {
    if (!g_prof.on) return;
    float acc[kStages] = {0};
    for (size_t k = 0; k < g_prof.stage_of.size(); ++k) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, g_prof.pool[2 * k], g_prof.pool[2 * k + 1]) == cudaSuccess)
            acc[g_prof.stage_of[k]] += ms;
    }
    for (int i = 0; i < kStages; ++i) g_prof.last[i] = acc[i];
}

// ---------------------------------------------------------------------------------------
// quantizer workspace layout
// ---------------------------------------------------------------------------------------
struct Workspace {
    DevState* st;
    float* A;        // d^2: damped, permuted, reversed H -> Cholesky factor; later undamped Hp
    float* X;        // d^2: L^-1, then U
    float* Wk;       // d_out x d_in working weights (processing order)
    float* Err[2];   // d_out x kSuperCols errors of a super-block (tf32 hi part), two buffers:
    float* ErrLo[2]; // a super-block's far update may still read one while the next fills the other
    uint8_t* codes_p;// d_out x d_in codes in processing order
    float* P;        // d x 128: the column loop's images of U's diagonal blocks
    float* Dinv;     // ceil(d/128) x 128 x 128 inverses of the Cholesky diagonal blocks
    float* F;        // 4 x d x 128 (512 from kOuterMinD on): the factorisation's split panels
    int* perm;
    int* invperm;
    size_t bytes;
};

static Workspace layout(void* base, int d_out, int d_in) {
    Workspace w{};
    size_t off = 0;
    auto take = [&](size_t b) {
        const size_t o = off;
        off += round256(b);
        return static_cast<uint8_t*>(base) + o;
    };
    const size_t d = static_cast<size_t>(d_in);
    const size_t nbl = (d + kCholBlock - 1) / kCholBlock;
    w.st = reinterpret_cast<DevState*>(take(sizeof(DevState)));
    w.A = reinterpret_cast<float*>(take(d * d * 4));
    w.X = reinterpret_cast<float*>(take(d * d * 4));
    w.Wk = reinterpret_cast<float*>(take(static_cast<size_t>(d_out) * d * 4));
    for (int b = 0; b < 2; ++b) {
        w.Err[b] = reinterpret_cast<float*>(take(static_cast<size_t>(d_out) * kSuperCols * 4));
        w.ErrLo[b] = reinterpret_cast<float*>(take(static_cast<size_t>(d_out) * kSuperCols * 4));
    }
    w.codes_p = take(static_cast<size_t>(d_out) * d);
    w.P = reinterpret_cast<float*>(take(d * kCholBlock * 4));
    w.Dinv = reinterpret_cast<float*>(take(nbl * kCholBlock * kCholBlock * 4));
    w.F = reinterpret_cast<float*>(
        take(4 * d * static_cast<size_t>(factor_panel_cols(static_cast<int>(d))) * 4));
    w.perm = reinterpret_cast<int*>(take(d * 4));
    w.invperm = reinterpret_cast<int*>(take(d * 4));
    w.bytes = off;
    return w;
}

}  // namespace gq

using namespace gq;

// =========================================================================================
// C ABI
// =========================================================================================
extern "C" {

const char* gptq_status_string(int status) {
    switch (status) {
        case GPTQ_OK: return "GPTQ_OK";
        case GPTQ_ERR_ARG: return "GPTQ_ERR_ARG: invalid argument";
        case GPTQ_ERR_NOT_PD: return "GPTQ_ERR_NOT_PD: damped Hessian is not positive definite";
        case GPTQ_ERR_NONFINITE: return "GPTQ_ERR_NONFINITE: NaN or Inf in H or W";
        case GPTQ_ERR_CUDA: return "GPTQ_ERR_CUDA: CUDA call failed";
        case GPTQ_ERR_OOM: return "GPTQ_ERR_OOM: device allocation failed";
        case GPTQ_ERR_TIMEOUT: return "GPTQ_ERR_TIMEOUT: a bounded device wait gave up";
        case GPTQ_ERR_WORKSPACE: return "GPTQ_ERR_WORKSPACE: workspace too small";
        case GPTQ_ERR_UNSUPPORTED: return "GPTQ_ERR_UNSUPPORTED: device is not sm_100";
        default: return "unknown gptq status";
    }
}

// ------------------------------- Hessian --------------------------------------------------
struct gptq_hessian {
    int d;
    int64_t tokens;
    float* H;
    int* status;
};

gptq_status gptq_hessian_accumulate_into(float* H, int d_in, const void* X, int64_t n_tokens,
                                         int unit_tokens, int* status_dev, void* stream) {
    if (!H || d_in < 8 || d_in > 65536 || d_in % 8 || n_tokens < 0) return GPTQ_ERR_ARG;
    if (n_tokens > 0 && (!X || !aligned16(X))) return GPTQ_ERR_ARG;
    if (!aligned16(H) || unit_tokens < 0 || unit_tokens % 64) return GPTQ_ERR_ARG;
    GPTQ_TRY(check_device());
    return hessian_launch(H, d_in, X, n_tokens, unit_tokens, status_dev,
                          static_cast<cudaStream_t>(stream));
}

gptq_status gptq_hessian_create(int d_in, gptq_hessian** out) {
    if (!out || d_in < 8 || d_in > 65536 || d_in % 8) return GPTQ_ERR_ARG;
    *out = nullptr;
    GPTQ_TRY(check_device());
    gptq_hessian* h = new gptq_hessian{};
    h->d = d_in;
    const size_t bytes = static_cast<size_t>(d_in) * d_in * 4;
    if (cudaMalloc(&h->H, bytes) != cudaSuccess) {
        cudaGetLastError();
        delete h;
        return GPTQ_ERR_OOM;
    }
    if (cudaMalloc(&h->status, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(h->H);
        delete h;
        return GPTQ_ERR_OOM;
    }
    if (cudaMemset(h->H, 0, bytes) != cudaSuccess || cudaMemset(h->status, 0, sizeof(int)) != cudaSuccess) {
        cudaFree(h->H);
        cudaFree(h->status);
        delete h;
        return GPTQ_ERR_CUDA;
    }
    *out = h;
    return GPTQ_OK;
}

gptq_status gptq_hessian_accumulate(gptq_hessian* h, const void* X, int64_t n_tokens,
                                    void* stream) {
    if (!h) return GPTQ_ERR_ARG;
    GPTQ_TRY(gptq_hessian_accumulate_into(h->H, h->d, X, n_tokens, 0, h->status, stream));
    h->tokens += n_tokens;
    return GPTQ_OK;
}

gptq_status gptq_hessian_get(const gptq_hessian* h, float* H_out, void* stream) {
    if (!h || !H_out) return GPTQ_ERR_ARG;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    GPTQ_TRY(mirror_upper_launch(h->H, H_out, h->d, s));
    int st = 0;
    GPTQ_CUDA_TRY(cudaMemcpyAsync(&st, h->status, sizeof(int), cudaMemcpyDeviceToHost, s));
    GPTQ_CUDA_TRY(cudaStreamSynchronize(s));
    return st ? static_cast<gptq_status>(st) : GPTQ_OK;
}

const float* gptq_hessian_data(const gptq_hessian* h) { return h ? h->H : nullptr; }
int64_t gptq_hessian_tokens(const gptq_hessian* h) { return h ? h->tokens : -1; }
int gptq_hessian_dim(const gptq_hessian* h) { return h ? h->d : -1; }

gptq_status gptq_hessian_reset(gptq_hessian* h, void* stream) {
    if (!h) return GPTQ_ERR_ARG;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    GPTQ_CUDA_TRY(cudaMemsetAsync(h->H, 0, static_cast<size_t>(h->d) * h->d * 4, s));
    GPTQ_CUDA_TRY(cudaMemsetAsync(h->status, 0, sizeof(int), s));
    h->tokens = 0;
    return GPTQ_OK;
}

gptq_status gptq_hessian_destroy(gptq_hessian* h) {
    if (!h) return GPTQ_OK;
    cudaFree(h->H);
    cudaFree(h->status);
    delete h;
    return GPTQ_OK;
}

// ------------------------------- GPTQ layer -----------------------------------------------
size_t gptq_quantize_layer_workspace(int d_out, int d_in, int block_size) {
    (void)block_size;
    if (d_out < 1 || d_in < 8) return 0;
    return layout(nullptr, d_out, d_in).bytes;
}

gptq_status gptq_quantize_layer(const void* W, int w_dtype, int d_out, int d_in,
                                const float* H, int bits, int group_size, int block_size,
                                float percdamp, int act_order, uint8_t* codes, uint16_t* scales,
                                uint16_t* zeros, int32_t* g_idx, int32_t* perm, float* loss,
                                void* workspace, size_t workspace_bytes, void* stream) {
    return gptq_quantize_layer_ex(W, w_dtype, d_out, d_in, H, bits, group_size, block_size,
                                  percdamp, act_order, 0, 0, codes, scales, zeros, g_idx, perm,
                                  loss, workspace, workspace_bytes, stream);
}

gptq_status gptq_quantize_layer_ex(const void* W, int w_dtype, int d_out, int d_in,
                                   const float* H, int bits, int group_size, int block_size,
                                   float percdamp, int act_order, int sym, int static_groups,
                                   uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                                   int32_t* g_idx, int32_t* perm, float* loss, void* workspace,
                                   size_t workspace_bytes, void* stream) {
    // ---- argument checks (no launch on failure) ----
    if (!W || !H || !codes || !scales || !zeros || !g_idx || !workspace) return GPTQ_ERR_ARG;
    if (w_dtype != GPTQ_DTYPE_F16 && w_dtype != GPTQ_DTYPE_F32) return GPTQ_ERR_ARG;
    if (d_out < 1 || d_in < 8 || d_in > 65536 || d_in % 8) return GPTQ_ERR_ARG;
    if (bits < 2 || bits > 8) return GPTQ_ERR_ARG;
    if (group_size < 1 || d_in % group_size) return GPTQ_ERR_ARG;
    const bool per_channel = group_size == d_in;
    if (block_size < 8 || block_size > 128 || block_size % 8 ||
        (block_size % group_size && !per_channel))
        return GPTQ_ERR_ARG;
    if (!(percdamp >= 0.0f) || act_order < 0 || act_order > 1) return GPTQ_ERR_ARG;
    if (sym < 0 || sym > 1 || static_groups < 0 || static_groups > 1) return GPTQ_ERR_ARG;
    // grids fixed before the column loop: every group of the original weights (static
    // groups), or the whole row (per-channel)
    const int preset = (static_groups || per_channel) ? 1 : 0;
    if (!aligned16(W) || !aligned16(H) || !aligned16(codes) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255))
        return GPTQ_ERR_ARG;
    if (static_cast<int64_t>(d_out) * d_in / group_size > (int64_t(1) << 40)) return GPTQ_ERR_ARG;
    const Workspace ws = layout(workspace, d_out, d_in);
    if (workspace_bytes < ws.bytes) return GPTQ_ERR_WORKSPACE;
    GPTQ_TRY(check_device());

    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    int* status = &ws.st->status;
    std::lock_guard<std::mutex> lock(g_prof.mu);
    profile_reset();
    StageTimer tm(s);

    GPTQ_CUDA_TRY(cudaMemsetAsync(ws.st, 0, sizeof(DevState), s));
    // ---- stage 0: damping, processing order, gathers ----
    tm.begin(0);
    GPTQ_TRY(diag_stats_launch(H, d_in, static_cast<double>(percdamp), ws.st, s));
    GPTQ_TRY(act_order_launch(H, d_in, act_order, ws.perm, ws.invperm, s));
    GPTQ_TRY(gather_h_launch(H, d_in, ws.perm, ws.st, 1, ws.A, status, s));
    GPTQ_TRY(gather_w_launch(W, w_dtype, d_out, d_in, ws.perm, ws.Wk, status, s));
    if (preset)
        GPTQ_TRY(group_grid_launch(W, w_dtype, d_out, d_in, group_size, bits, sym, scales, zeros,
                                   s));
    tm.end();
    // ---- stage 1: U with U^T U = H_d^-1 (factor and inverse overlap on two streams) ----
    tm.begin(1);
    GPTQ_TRY(factor_inverse_launch(ws.A, d_in, ws.Dinv, ws.X, ws.F, status, s));
    tm.end();
    // ---- stage 2: the forms of U that the column loop and the lazy updates read ----
    uint8_t* codes_p = act_order ? ws.codes_p : codes;
    // the block inverses are free after the triangular inverse: they take 1/U_ii, and P the
    // column loop's images of U's diagonal blocks
    tm.begin(2);
    GPTQ_TRY(column_images_launch(ws.X, d_in, block_size, ws.P, ws.Dinv, s));
    // U as tf32 hi (in place) and lo (into the factor's buffer, free now) for the lazy updates
    GPTQ_TRY(tcgemm_split_launch(ws.X, ws.X, ws.A, d_in, d_in, d_in, true, s));
    tm.end();
    // ---- stage 3-4: column loop and lazy batch updates ----
    // Lazy batch updates on two levels: the errors of a super-block of whole blocks (about
    // kSuperCols columns) are kept; after each block only the rest of its super-block is
    // updated, and the columns beyond the super-block get one update per super-block. Every
    // column still receives the compensation of all earlier columns before it is quantized.
    // The far update of super-block S is split in two: the next super-block's columns on the
    // caller's stream (its column loop needs them next), and all later columns on the library's
    // second stream, where it runs on the SMs the next column loop leaves free. The main stream
    // waits for that rest before it next writes those columns; the errors alternate between
    // two buffers so the rest can read S's errors while S+1 records its own.
    const int super = block_size * std::max(1, kSuperCols / block_size);
    constexpr int kMinSideCtas = 64;
    const int side_ctas = num_sms() - gptq_rows_ctas(d_out);
    // (the 3xTF32 GEMM needs most of the GPU to pay: with fewer free SMs than this the far
    // update on the side would outlast the column loop it hides behind)
    const bool overlap = side_ctas >= kMinSideCtas && d_in > 2 * super;
    // while the overlap runs, the caller's stream keeps its GEMMs on the SMs the second stream
    // leaves free, so that every CTA of a persistent launch is resident at once
    const int main_ctas = overlap ? num_sms() - side_ctas : 0;
    std::unique_lock<std::mutex> side_lock(side_streams_mutex(), std::defer_lock);
    SideStreams* ss = nullptr;
    if (overlap) {
        side_lock.lock();
        GPTQ_TRY(side_streams(&ss));
        GPTQ_CUDA_TRY(cudaEventRecord(ss->aux1, s));
        GPTQ_CUDA_TRY(cudaStreamWaitEvent(ss->side, ss->aux1, 0));
    }
    auto column_stage = [&]() -> gptq_status {
        bool rest_pending = false;
        for (int s0 = 0, sb = 0; s0 < d_in; s0 += super, ++sb) {
            const int s1 = std::min(s0 + super, d_in);
            const int s2 = std::min(s1 + super, d_in);
            float* Eh = ws.Err[sb & 1];
            float* El = ws.ErrLo[sb & 1];
            for (int j0 = s0; j0 < s1; j0 += block_size) {
                const int bw = std::min(block_size, s1 - j0), j1 = j0 + bw;
                float* err_hi = Eh + (j0 - s0);
                float* err_lo = El + (j0 - s0);
                tm.begin(3);
                GPTQ_TRY(gptq_block_launch(ws.Wk, d_out, d_in, j0, bw, ws.P, ws.Dinv, group_size,
                                           bits, sym, preset ? ws.perm : nullptr, codes_p,
                                           scales, zeros, err_hi, err_lo, kSuperCols,
                                           &ws.st->err_sq, status, s));
                tm.end();
                tm.begin(4);
                GPTQ_TRY(lazy_update_launch(ws.Wk, d_out, d_in, j0, j1, j1, s1, ws.X, ws.A,
                                            err_hi, err_lo, kSuperCols, status, s, main_ctas));
                tm.end();
            }
            tm.begin(4);
            if (rest_pending) GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, ss->aux2, 0));
            GPTQ_TRY(lazy_update_launch(ws.Wk, d_out, d_in, s0, s1, s1, overlap ? s2 : d_in,
                                        ws.X, ws.A, Eh, El, kSuperCols, status, s, main_ctas));
            tm.end();
            if (overlap && s2 < d_in) {
                GPTQ_CUDA_TRY(cudaEventRecord(ss->aux1, s));      // S's errors are complete
                GPTQ_CUDA_TRY(cudaStreamWaitEvent(ss->side, ss->aux1, 0));
                GPTQ_TRY(lazy_update_launch(ws.Wk, d_out, d_in, s0, s1, s2, d_in, ws.X, ws.A, Eh,
                                            El, kSuperCols, status, ss->side, side_ctas));
                GPTQ_CUDA_TRY(cudaEventRecord(ss->aux2, ss->side));
                rest_pending = true;
            }
        }
        return GPTQ_OK;
    };
    const gptq_status crc = column_stage();
    if (overlap) {
        // join the second stream back, also after an error, so a capture of `s` stays formed
        const cudaError_t e1 = cudaEventRecord(ss->join, ss->side);
        const cudaError_t e2 = cudaStreamWaitEvent(s, ss->join, 0);
        side_lock.unlock();
        if (crc == GPTQ_OK && (e1 != cudaSuccess || e2 != cudaSuccess)) return GPTQ_ERR_CUDA;
    }
    GPTQ_TRY(crc);
    // ---- stage 5: outputs in the original column order ----
    tm.begin(5);
    GPTQ_TRY(assemble_launch(codes_p, d_out, d_in, ws.perm, ws.invperm, group_size, act_order,
                             preset, codes, g_idx, perm, s));
    tm.end();
    // ---- stage 6: reconstruction loss ----
    if (loss) {
        tm.begin(6);
        GPTQ_TRY(loss_launch(W, w_dtype, d_out, d_in, H, ws.perm, codes_p, scales, zeros,
                             group_size, preset, ws.Wk, ws.A, ws.st, s));
        tm.end();
    }
    DevState host{};
    GPTQ_CUDA_TRY(cudaMemcpyAsync(&host, ws.st, sizeof(DevState), cudaMemcpyDeviceToHost, s));
    GPTQ_CUDA_TRY(cudaStreamSynchronize(s));
    profile_collect();
    if (host.status) return static_cast<gptq_status>(host.status);
    if (loss) *loss = static_cast<float>((host.err_sq - host.lam * host.delta_sq) / host.loss_den);
    return GPTQ_OK;
}

// ------------------------------- inverse factor -------------------------------------------
size_t gptq_inverse_factor_workspace(int d_in) {
    if (d_in < 8) return 0;
    return layout(nullptr, 1, d_in).bytes;
}

gptq_status gptq_inverse_factor(const float* H, int d_in, float percdamp, int act_order,
                                float* U, int32_t* perm, void* workspace,
                                size_t workspace_bytes, void* stream) {
    if (!H || !U || !workspace) return GPTQ_ERR_ARG;
    if (d_in < 8 || d_in > 65536 || d_in % 8) return GPTQ_ERR_ARG;
    if (!(percdamp >= 0.0f) || act_order < 0 || act_order > 1) return GPTQ_ERR_ARG;
    if (!aligned16(H) || !aligned16(U) || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return GPTQ_ERR_ARG;
    const Workspace ws = layout(workspace, 1, d_in);
    if (workspace_bytes < ws.bytes) return GPTQ_ERR_WORKSPACE;
    GPTQ_TRY(check_device());
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    int* status = &ws.st->status;
    GPTQ_CUDA_TRY(cudaMemsetAsync(ws.st, 0, sizeof(DevState), s));
    GPTQ_TRY(diag_stats_launch(H, d_in, static_cast<double>(percdamp), ws.st, s));
    GPTQ_TRY(act_order_launch(H, d_in, act_order, ws.perm, ws.invperm, s));
    GPTQ_TRY(gather_h_launch(H, d_in, ws.perm, ws.st, 1, ws.A, status, s));
    GPTQ_TRY(factor_inverse_launch(ws.A, d_in, ws.Dinv, ws.X, ws.F, status, s));
    GPTQ_CUDA_TRY(cudaMemcpyAsync(U, ws.X, static_cast<size_t>(d_in) * d_in * 4,
                                  cudaMemcpyDeviceToDevice, s));
    if (perm)
        GPTQ_CUDA_TRY(cudaMemcpyAsync(perm, ws.perm, static_cast<size_t>(d_in) * 4,
                                      cudaMemcpyDeviceToDevice, s));
    DevState host{};
    GPTQ_CUDA_TRY(cudaMemcpyAsync(&host, ws.st, sizeof(DevState), cudaMemcpyDeviceToHost, s));
    GPTQ_CUDA_TRY(cudaStreamSynchronize(s));
    return host.status ? static_cast<gptq_status>(host.status) : GPTQ_OK;
}

// ------------------------------- RTN ------------------------------------------------------
gptq_status rtn_minmax_quantize(const void* W, int w_dtype, int d_out, int d_in, int bits,
                                int group_size, uint8_t* packed, uint16_t* scales,
                                uint16_t* zeros, void* stream) {
    return rtn_quantize_ex(W, w_dtype, d_out, d_in, bits, group_size, 0, packed, scales, zeros,
                           stream);
}

gptq_status rtn_quantize_ex(const void* W, int w_dtype, int d_out, int d_in, int bits,
                            int group_size, int sym, uint8_t* packed, uint16_t* scales,
                            uint16_t* zeros, void* stream) {
    if (!W || !packed || !scales || !zeros) return GPTQ_ERR_ARG;
    if (w_dtype != GPTQ_DTYPE_F16 && w_dtype != GPTQ_DTYPE_F32) return GPTQ_ERR_ARG;
    if (d_out < 1 || d_in < 8 || d_in % 8 || bits < 2 || bits > 8) return GPTQ_ERR_ARG;
    if (group_size < 1 || d_in % group_size || sym < 0 || sym > 1) return GPTQ_ERR_ARG;
    if (!aligned16(W) || !aligned16(packed)) return GPTQ_ERR_ARG;
    GPTQ_TRY(check_device());
    return rtn_launch(W, w_dtype, d_out, d_in, bits, group_size, sym, packed, scales, zeros,
                      static_cast<cudaStream_t>(stream));
}

// ------------------------------- profiling ------------------------------------------------
void gptq_profile_enable(int on) {
    std::lock_guard<std::mutex> lock(g_prof.mu);
    g_prof.on = on != 0;
}

unsigned long long gptq_launch_count(void) { return g_launches.load(); }

gptq_status gptq_test_stall_factor(int on) {
    GPTQ_TRY(check_device());
    return factor_stall_set(on);
}

int gptq_profile_read(float* ms_out, int max_stages) {
    std::lock_guard<std::mutex> lock(g_prof.mu);
    const int n = max_stages < kStages ? max_stages : kStages;
    for (int i = 0; i < n; ++i) ms_out[i] = g_prof.last[i];
    return n;
}

}  // extern "C"
