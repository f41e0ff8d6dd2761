// gdn_prefill_noalloc.cu -- gdn_prefill for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain device scratch at call time: a plugin
// hosted by a framework that owns all of the GPU's memory and hands it only
// the input and output buffers, or a latency-critical loop that must never
// call cudaMalloc/cudaFree, which can synchronise the whole device.  For them
// this file keeps the prefill scratch in one fixed, file-scope device array,
// so that the entry point below allocates nothing.
//
// Set-up: the first call on each device (with that device current) looks up
// the array's device address with cudaGetSymbolAddress and caches it; every
// later call on that device reuses it.  In host code the array's name is only
// a host-side stand-in, never a device address, so the looked-up address is
// what reaches the kernels.  Because the first call on a device does this
// set-up, make that first call before any stream capture.
#include <mutex>

#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace {

constexpr size_t kScratchBytes = GDN_NOALLOC_SCRATCH_BYTES;

// The shared scratch: normalised q|k and convolved v of one call, as in the
// caller-provided workspace of gdn_prefill.  Every GPU that loads the library
// holds it until the process exits.
static __device__ __align__(256) unsigned char g_prefill_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices]; // device address of g_prefill_scratch, per device

// Device address of the scratch on the current device (looked up once).
gdn_status scratch_on_current_device(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0)
        return GDN_ERR_CUDA;
    if (dev >= kMaxDevices)
        return GDN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_prefill_scratch);
        if (e != cudaSuccess || p == nullptr)
            return GDN_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return GDN_OK;
}

} // namespace

extern "C" gdn_status gdn_prefill_noalloc(const gdn_config *cfg, const gdn_params *params,
                                          const void *qkv, const void *a, const void *b,
                                          const void *z, const int32_t *cu_seqlens, int32_t batch,
                                          int64_t total_tokens, const float *initial_state,
                                          const void *initial_conv, void *y, float *final_state,
                                          void *final_conv, float *o_raw, void *stream) {
    // The argument checks of gdn_prefill first (same codes, same order), then
    // the size check: a call that needs more than the fixed array is rejected
    // before any CUDA call.
    size_t need = 0;
    gdn_status st = gdn::validate_prefill(cfg, params, qkv, a, b, z, cu_seqlens, batch,
                                          total_tokens, initial_state, initial_conv, y,
                                          final_state, final_conv, o_raw, &need);
    if (st != GDN_OK)
        return st;
    if (need > kScratchBytes)
        return GDN_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (need > 0 && (st = scratch_on_current_device(&scratch)) != GDN_OK)
        return st;
    // Nothing in the scratch has to start at zero: the first kernel of the
    // call clears the status words, and the front-end kernels write every
    // element the recurrence later reads, so the previous call's contents
    // never leak into this one.
    // every kernel on the caller's stream: no second stream is created here
    return gdn::prefill_impl(cfg, params, qkv, a, b, z, cu_seqlens, batch, total_tokens,
                             initial_state, initial_conv, y, final_state, final_conv, o_raw,
                             scratch, scratch ? kScratchBytes : 0, stream, false);
}

extern "C" gdn_status gdn_prefill_noalloc_status(uint32_t *detail, void *stream) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0)
        return GDN_ERR_CUDA;
    void *addr = nullptr;
    if (dev < kMaxDevices) {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        addr = g_scratch_addr[dev];
    }
    if (detail != nullptr)
        *detail = 0u;
    if (addr == nullptr) // no gdn_prefill_noalloc call has used the array on this device
        return GDN_OK;
    return gdn::read_status_words(addr, detail, (cudaStream_t)stream);
}
