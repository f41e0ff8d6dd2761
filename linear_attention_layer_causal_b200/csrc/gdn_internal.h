// gdn_internal.h -- argument bundles passed from the C ABI layer to the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn {

struct PrefillArgs {
    int Hk, Hv, D, G;
    bool bf16;
    float rms_eps, l2_eps, q_scale;
    const void *qkv, *a, *b, *z;
    const int32_t *cu;
    int batch;
    int64_t N;
    const float *init_state;
    const void *init_conv;
    void *y;
    float *final_state;
    void *final_conv;
    float *o_raw;
    const float *conv_w, *A_log, *dt_bias, *norm_w;
    bool chunked;            // tensor-core chunked path (head_dim 128) or token-serial
    // workspace carve-up
    unsigned int *ws_err;    // device status word (0 = ok; bit 0: a bounded wait timed out)
    void *ws_qk;             // [N, 2*Hk*D] float32: normalised q | k
    void *ws_v;              // [N, Hv*D]   float32: convolved v
    void *ws_kq;             // [N, Hk, 2, 64] float32: chunk Gram rows (chunked path)
    int32_t *ws_offs;        // [batch + 1] chunk offsets per sequence (chunked path)
};

struct DecodeArgs {
    int Hk, Hv, D, G;
    bool bf16;
    float rms_eps, l2_eps, q_scale;
    const void *qkv, *a, *b, *z;
    float *state;
    void *conv_cache;
    int batch;
    void *y;
    const float *conv_w, *A_log, *dt_bias, *norm_w;
};

// One-shot events around the main kernel of the next call on this host thread.
struct ProfileHook {
    cudaEvent_t begin = nullptr, end = nullptr;
};
ProfileHook take_profile_hook(); // returns the armed events and disarms

// Records `ev` on `s` when it is non-null.
inline cudaError_t record_if(cudaEvent_t ev, cudaStream_t s) {
    return ev ? cudaEventRecord(ev, s) : cudaSuccess;
}

// Workspace bytes for the prefill path (each region 256-byte aligned).
size_t prefill_workspace_bytes(int Hk, int Hv, int D, bool bf16, int64_t N, int batch);
constexpr size_t kWorkspaceHeader = 256; // holds the device status word

cudaError_t launch_conv_prep(const PrefillArgs &p, cudaStream_t s);
cudaError_t launch_final_conv(const PrefillArgs &p, cudaStream_t s);
cudaError_t launch_recurrent_prefill(const PrefillArgs &p, cudaStream_t s);
cudaError_t launch_chunk_offsets(const PrefillArgs &p, cudaStream_t s);
cudaError_t launch_kq_prep(const PrefillArgs &p, cudaStream_t s);
cudaError_t launch_chunk_prefill(const PrefillArgs &p, cudaStream_t s);
size_t kq_workspace_bytes(int Hk, int64_t N);
cudaError_t launch_decode(const DecodeArgs &p, cudaStream_t s);

} // namespace gdn
