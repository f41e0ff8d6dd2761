// gdn_internal.h -- argument bundles passed from the C ABI layer to the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gdn.h"

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
    const void *kda_zdec = nullptr; // KDA: per-channel decay inputs [N, H, d] (a, dt_bias unused)
    float *ws_o = nullptr;          // KDA: [N, H, d] float32 raw output before the gated norm
    long long wait_limit;    // SM cycles a wait between warps may take before the call aborts
    // workspace carve-up
    unsigned int *ws_err;    // device status word (0 = ok; bit 0: a bounded wait timed out)
    void *ws_qk;             // [N, 2*Hk*D] float32: normalised q | k
    void *ws_v;              // [N, Hv*D]   float32: convolved v (nullptr where the chunk kernel convolves v)
    void *ws_kq;             // [N, Hk, 64] float32: chunk Q K^T rows (chunked path)
    void *ws_kk;             // [chunks, Hk, 3072] float32: K K^T triangular tiles (chunked path)
    void *ws_tb;             // [chunks, Hv, 2, 96, 32] float32: T diag(beta), -T diag(beta gamma) tiles (chunked path)
    float *ws_gt;            // [chunks, Hv, 3, 64] float32: per chunk G, gamma_C / gamma, gamma (chunked path)
    int32_t *ws_offs;        // [batch + 1] chunk offsets per sequence (chunked path)
    // sequence split of the chunked path (segments > 1)
    int segments = 1;        // P: segments per sequence
    int seg_pass = 0;        // chunk kernel launch: 0 = output pass, 1 = summary pass
    float *ws_seg = nullptr; // R, M [batch, P-1, Hv, 128, 128] each, then the segment start states
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
    const void *kda_zdec = nullptr;    // KDA: per-channel decay inputs [batch, H, d]
    int k = 1;                         // tokens per sequence (multi-token decode)
    const int32_t *accepted = nullptr; // [batch] tokens to take (commit mode)
};

// Multi-token decode: modes and the most tokens per sequence one call takes.
constexpr int kDecodeMulti = 0, kDecodeVerify = 1, kDecodeCommit = 2;
constexpr int kDecodeMaxTokens = 8;
constexpr size_t kDecodeMaxSmem = 227 * 1024;

// One-shot events around the main kernel of the next call on this host thread.
struct ProfileHook {
    cudaEvent_t begin = nullptr, end = nullptr;
};
ProfileHook take_profile_hook(); // returns the armed events and disarms

// Default bound of a wait between the warps of a kernel (about one second of
// SM clock), and the one-shot override of the calling host thread (armed by
// gdn_wait_limit_next_call): returns the limit for this call and disarms.
constexpr long long kDefaultWaitLimit = 2000000000LL;
long long take_wait_limit();

// The argument checks of gdn_prefill, in its order, minus the workspace; on
// success *need holds the workspace bytes the call requires.
gdn_status validate_prefill(const gdn_config *cfg, const gdn_params *params, const void *qkv,
                            const void *a, const void *b, const void *z, const int32_t *cu_seqlens,
                            int32_t batch, int64_t total_tokens, const float *initial_state,
                            const void *initial_conv, const void *y, const float *final_state,
                            const void *final_conv, const float *o_raw, size_t *need);

// gdn_prefill itself; `side` allows the chunked path to run the v conv on a
// second stream of its own (gdn_prefill_noalloc passes false: it creates
// nothing, and runs every kernel on the caller's stream in order).
gdn_status prefill_impl(const gdn_config *cfg, const gdn_params *params, const void *qkv,
                        const void *a, const void *b, const void *z, const int32_t *cu_seqlens,
                        int32_t batch, int64_t total_tokens, const float *initial_state,
                        const void *initial_conv, void *y, float *final_state, void *final_conv,
                        float *o_raw, void *workspace, size_t workspace_bytes, void *stream,
                        bool side);

// Reads the two status words at `header` (device) after `stream` completes.
gdn_status read_status_words(const void *header, uint32_t *detail, cudaStream_t stream);

// Records `ev` on `s` when it is non-null.
inline cudaError_t record_if(cudaEvent_t ev, cudaStream_t s) {
    return ev ? cudaEventRecord(ev, s) : cudaSuccess;
}

// Workspace bytes for the prefill path (each region 256-byte aligned).
size_t prefill_workspace_bytes(const gdn_config *c, int64_t N, int batch);
// The chunk kernel convolves v itself from the 16-bit pre-conv rows; the
// front end then writes no convolved v.
inline bool v_conv_in_chunk(bool chunked, bool bf16) { return chunked && bf16; }
// Segments per sequence a chunked prefill of this config and size runs with
// (1 for the token-serial path and for calls without tokens).
int prefill_segments(const gdn_config *c, int batch, int64_t N);
constexpr int kMaxSegments = 16;
size_t seg_workspace_bytes(int Hv, int batch, int segments);
constexpr size_t kWorkspaceHeader = 256; // holds the device status word

// Which channels a conv launch covers: all, the channel blocks holding q or k
// (and the v channels of a block that straddles the boundary), or the rest.
enum class ConvPart { kAll, kQK, kV };
cudaError_t launch_conv_prep(const PrefillArgs &p, ConvPart part, cudaStream_t s);
cudaError_t launch_final_conv(const PrefillArgs &p, cudaStream_t s);
cudaError_t launch_recurrent_prefill(const PrefillArgs &p, cudaStream_t s);
cudaError_t launch_chunk_offsets(const PrefillArgs &p, cudaStream_t s);
cudaError_t launch_gram(const PrefillArgs &p, cudaStream_t s);
cudaError_t launch_tri(const PrefillArgs &p, cudaStream_t s);
cudaError_t launch_chunk_prefill(const PrefillArgs &p, cudaStream_t s);
size_t kq_workspace_bytes(int Hk, int64_t N);
size_t tb_workspace_bytes(int Hv, int64_t N, int batch);
size_t kk_workspace_bytes(int Hk, int64_t N, int batch);
size_t gt_workspace_bytes(int Hv, int64_t N, int batch);
constexpr int kGateRec = 192; // floats of one (chunk, value head) gate record: G, gamma_C / gamma, gamma
cudaError_t launch_decode(const DecodeArgs &p, cudaStream_t s);
cudaError_t launch_decode_multi(const DecodeArgs &p, int mode, cudaStream_t s);
cudaError_t launch_kda_prefill(const PrefillArgs &p, cudaStream_t s);
cudaError_t launch_kda_decode(const DecodeArgs &p, cudaStream_t s);
size_t decode_multi_smem_bytes(int G, int D, int k, int mode);

} // namespace gdn
