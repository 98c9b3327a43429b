// gptq_quantize_layer_noalloc: the GPTQ layer quantizer for callers that cannot allocate.
//
// Some callers of this library are not allowed to allocate device memory at the point where
// they quantize a layer. Examples are a runtime that reserved nearly all of the GPU for its
// own pools at start-up (a serving engine's KV cache, a framework's caching allocator), so
// that an extra cudaMalloc of tens of MB fails or fragments the pool, and a deployment that
// forbids device allocation after initialisation. Such callers also cannot hand over a
// workspace. This entry point takes its scratch from a fixed array that is reserved when the
// library's device code is loaded, and it calls no allocator at all.
//
// The array lives in this file. Host code only knows its symbol, so the device address is
// looked up with cudaGetSymbolAddress once per device (with that device current) and then
// passed to the unchanged gptq_quantize_layer path as its workspace.
#include <mutex>

#include "internal.cuh"

namespace gq {

// Largest workspace this entry point can serve: 32 MiB. The array is part of the library's
// device code: it takes device memory when that code is loaded onto a GPU and keeps it until
// the process exits. With CUDA's lazy module loading (the default) the load happens at the
// first use on each device, which for this array is the address lookup in the first call of
// gptq_quantize_layer_noalloc there; a caller that reserves its pools at start-up should make
// that first call before reserving them.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
static std::mutex g_scratch_mu;
static void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device, resolved on first use.
static gptq_status static_scratch(void** out) {
    int dev = 0;
    GPTQ_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return GPTQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();   // do not leave the failure for an unrelated later check
            return GPTQ_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return GPTQ_OK;
}

}  // namespace gq

extern "C" gptq_status gptq_quantize_layer_noalloc(
    const void* W, int w_dtype, int d_out, int d_in, const float* H, int bits, int group_size,
    int block_size, float percdamp, int act_order, uint8_t* codes, uint16_t* scales,
    uint16_t* zeros, int32_t* g_idx, int32_t* perm, float* loss, void* stream) {
    if (d_out < 1 || d_in < 8) return GPTQ_ERR_ARG;
    const size_t need = gptq_quantize_layer_workspace(d_out, d_in, block_size);
    if (need == 0 || need > gq::kStaticScratchBytes) return GPTQ_ERR_WORKSPACE;
    GPTQ_TRY(gq::check_device());
    void* ws = nullptr;
    GPTQ_TRY(gq::static_scratch(&ws));
    // gptq_quantize_layer clears the status block at the head of the workspace itself and
    // writes every other scratch byte before reading it, so leftovers of a previous call do
    // not leak into this one.
    return gptq_quantize_layer(W, w_dtype, d_out, d_in, H, bits, group_size, block_size,
                               percdamp, act_order, codes, scales, zeros, g_idx, perm, loss, ws,
                               gq::kStaticScratchBytes, stream);
}
