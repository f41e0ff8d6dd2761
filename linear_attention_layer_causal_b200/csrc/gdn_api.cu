// gdn_api.cu -- the C ABI declared in include/gdn.h: host-side argument
// checks, workspace carve-up and kernel launches.  Every check runs before the
// first CUDA call, so a rejected call launches nothing and touches no device.
#include <math.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gdn_status check_config(const gdn_config *c) {
    if (c == nullptr)
        return GDN_ERR_INVALID_ARG;
    if (c->num_qk_heads < 1 || c->num_v_heads < 1 || c->head_dim < 1 || c->conv_kernel < 1)
        return GDN_ERR_INVALID_ARG;
    if (c->num_v_heads % c->num_qk_heads != 0)
        return GDN_ERR_INVALID_ARG;
    if (c->act_dtype != GDN_F32 && c->act_dtype != GDN_BF16)
        return GDN_ERR_INVALID_ARG;
    if (!(c->rms_eps >= 0.f) || !(c->l2_eps >= 0.f) || !isfinite(c->rms_eps) ||
        !isfinite(c->l2_eps) || !isfinite(c->q_scale))
        return GDN_ERR_INVALID_ARG;
    if (c->head_dim != 32 && c->head_dim != 128)
        return GDN_ERR_UNSUPPORTED;
    if (c->conv_kernel != 4)
        return GDN_ERR_UNSUPPORTED;
    if (c->num_v_heads / c->num_qk_heads > 64)
        return GDN_ERR_UNSUPPORTED;
    if (c->algo < GDN_ALGO_AUTO || c->algo > GDN_ALGO_CHUNKED)
        return GDN_ERR_INVALID_ARG;
    if (c->algo == GDN_ALGO_CHUNKED && c->head_dim != 128)
        return GDN_ERR_UNSUPPORTED;
    if (c->segments < 0 || c->segments > kMaxSegments)
        return GDN_ERR_INVALID_ARG;
    if (c->segments > 1 && (c->head_dim != 128 || c->algo == GDN_ALGO_SERIAL))
        return GDN_ERR_UNSUPPORTED; // the split runs on the chunked path only
    // conv_dim * 16-byte channel groups must index in int
    const int64_t conv_dim = (int64_t)(2 * (int64_t)c->num_qk_heads + c->num_v_heads) * c->head_dim;
    if (conv_dim > (int64_t)1 << 26)
        return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

gdn_status check_params(const gdn_params *p) {
    if (p == nullptr || p->conv_w == nullptr || p->A_log == nullptr || p->dt_bias == nullptr ||
        p->norm_w == nullptr)
        return GDN_ERR_INVALID_ARG;
    if (!aligned16(p->conv_w) || !aligned16(p->norm_w))
        return GDN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(p->A_log) & 3u) || (reinterpret_cast<uintptr_t>(p->dt_bias) & 3u))
        return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

bool elem_aligned(const void *p, bool bf16) {
    return p == nullptr || (reinterpret_cast<uintptr_t>(p) & (bf16 ? 1u : 3u)) == 0;
}

gdn_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

thread_local ProfileHook tl_hook;

// A second stream per host thread and device, with a fork and a join event:
// the chunked prefill runs the (bandwidth-bound) conv of the v channels on it,
// beside the (latency-bound) q/k conv, Gram and inverse kernels on the
// caller's stream.  Created on the first chunked call of the thread on that
// device and kept until the process exits; thread-local, so calls from several
// host threads never share one.
struct SideStream {
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxSideDevices = 64;
thread_local SideStream tl_side[kMaxSideDevices];

cudaError_t side_stream(SideStream **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxSideDevices)
        return cudaErrorInvalidDevice;
    SideStream &ss = tl_side[dev];
    if (ss.stream == nullptr) {
        e = cudaStreamCreateWithFlags(&ss.stream, cudaStreamNonBlocking);
        if (e == cudaSuccess)
            e = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming);
        if (e == cudaSuccess)
            e = cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming);
        if (e != cudaSuccess)
            return e;
    }
    *out = &ss;
    return cudaSuccess;
}
thread_local long long tl_wait_limit = 0; // 0 = not armed

} // namespace

ProfileHook take_profile_hook() {
    ProfileHook h = tl_hook;
    tl_hook = ProfileHook{};
    return h;
}

long long take_wait_limit() {
    const long long w = tl_wait_limit;
    tl_wait_limit = 0;
    return w > 0 ? w : kDefaultWaitLimit;
}

gdn_status validate_prefill(const gdn_config *cfg, const gdn_params *params, const void *qkv,
                            const void *a, const void *b, const void *z, const int32_t *cu_seqlens,
                            int32_t batch, int64_t total_tokens, const float *initial_state,
                            const void *initial_conv, const void *y, const float *final_state,
                            const void *final_conv, const float *o_raw, size_t *need) {
    gdn_status st = check_config(cfg);
    if (st != GDN_OK)
        return st;
    if ((st = check_params(params)) != GDN_OK)
        return st;
    if (batch < 0 || total_tokens < 0 || batch > 65535)
        return batch > 65535 ? GDN_ERR_UNSUPPORTED : GDN_ERR_INVALID_ARG;
    if (batch == 0 && total_tokens > 0)
        return GDN_ERR_INVALID_ARG;
    if (batch > 0 && cu_seqlens == nullptr)
        return GDN_ERR_INVALID_ARG;
    const bool bf16 = cfg->act_dtype == GDN_BF16;
    if (total_tokens > 0 && (qkv == nullptr || a == nullptr || b == nullptr || z == nullptr ||
                             y == nullptr))
        return GDN_ERR_INVALID_ARG;
    if (!aligned16(qkv) || !aligned16(z) || !aligned16(y) || !aligned16(initial_state) ||
        !aligned16(initial_conv) || !aligned16(final_state) || !aligned16(final_conv) ||
        !aligned16(o_raw) || !elem_aligned(a, bf16) || !elem_aligned(b, bf16) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
        return GDN_ERR_INVALID_ARG;
    // the chunked path addresses its per-(chunk, value head) tiles by 32-bit TMA
    // row coordinates: 192 rows per (chunk, value head)
    const bool chunked = cfg->head_dim == 128 && cfg->algo != GDN_ALGO_SERIAL;
    if (chunked && ((total_tokens + 63) / 64 + (int64_t)batch) * cfg->num_v_heads * 192 > INT32_MAX)
        return GDN_ERR_UNSUPPORTED;
    *need = prefill_workspace_bytes(cfg, total_tokens, batch);
    return GDN_OK;
}

// The library's choice of segments per sequence.  Costs are in chunk steps of
// one chain: unsplit, the average sequence takes L = N / (64 batch) of them;
// split into P, the summary pass runs 2 (P - 1) CTAs per (sequence, value
// head) over L / P chunks at about kSummaryCost of an output step (no Q, O or
// P work, no z or y traffic), in ceil(2 (P - 1) batch H_v / 148) waves of one
// CTA per SM; the output pass runs P CTAs per unit in ceil(P batch H_v / 148)
// waves; the combine and the extra launches add about kSplitOverhead steps.
int prefill_segments(const gdn_config *c, int batch, int64_t N) {
    if (c->head_dim != 128 || c->algo == GDN_ALGO_SERIAL || batch <= 0 || N <= 0)
        return 1;
    if (c->segments > 0)
        return c->segments;
    constexpr int64_t kSMs = 148;
    constexpr double kSummaryCost = 0.6, kSplitOverhead = 8.0, kMinChunksPerSegment = 32.0;
    const int64_t units = (int64_t)batch * c->num_v_heads;
    if (2 * units > kSMs)
        return 1;
    const double L = (double)N / (64.0 * batch);
    int best = 1;
    double best_cost = L;
    for (int P = 2; P <= kMaxSegments && L / P >= kMinChunksPerSegment; ++P) {
        const double ws = (double)((2 * units * (P - 1) + kSMs - 1) / kSMs);
        const double wo = (double)((units * P + kSMs - 1) / kSMs);
        const double cost = (ws * kSummaryCost + wo) * L / P + kSplitOverhead;
        if (cost < best_cost) {
            best_cost = cost;
            best = P;
        }
    }
    return best;
}

// R and M of every segment but the last, and the start state of every segment
// but the first: 3 (P - 1) batch H_v states of 128 x 128 floats.
size_t seg_workspace_bytes(int Hv, int batch, int segments) {
    return segments <= 1 ? 0 : (size_t)3 * (segments - 1) * batch * Hv * 128 * 128 * sizeof(float);
}

gdn_status read_status_words(const void *header, uint32_t *detail, cudaStream_t stream) {
    uint32_t w[2] = {0u, 0u};
    cudaError_t e = cudaMemcpyAsync(w, header, sizeof(w), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess)
        return GDN_ERR_CUDA;
    if (detail != nullptr)
        *detail = w[1];
    if (w[0] & 1u)
        return GDN_ERR_TIMEOUT;
    return w[0] != 0u ? GDN_ERR_CUDA : GDN_OK;
}

// Header (status word), float32 normalised q|k, float32 convolved v (unless
// the chunk kernel convolves v itself: 16-bit activations) and, on the
// chunked path, the Q K^T rows, K K^T and T diag(beta) tiles, the gate
// records, the per-sequence chunk offsets and the split's states.
size_t prefill_workspace_bytes(const gdn_config *c, int64_t N, int batch) {
    if (N == 0)
        return 0;
    const int Hk = c->num_qk_heads, Hv = c->num_v_heads, D = c->head_dim;
    const bool chunked = D == 128 && c->algo != GDN_ALGO_SERIAL;
    size_t b = kWorkspaceHeader + round_up((size_t)N * 2 * Hk * D * 4);
    if (!v_conv_in_chunk(chunked, c->act_dtype == GDN_BF16))
        b += round_up((size_t)N * Hv * D * 4);
    if (chunked)
        b += round_up(kq_workspace_bytes(Hk, N)) + round_up(kk_workspace_bytes(Hk, N, batch)) +
             round_up(tb_workspace_bytes(Hv, N, batch)) + round_up(gt_workspace_bytes(Hv, N, batch)) +
             round_up(((size_t)batch + 1) * sizeof(int32_t)) + seg_workspace_bytes(Hv, batch, prefill_segments(c, batch, N));
    return b;
}

} // namespace gdn

using namespace gdn;

extern "C" {

int32_t gdn_abi_version(void) { return GDN_ABI_VERSION; }

gdn_status gdn_profile_next_call(void *begin_event, void *end_event) {
    if ((begin_event == nullptr) != (end_event == nullptr))
        return GDN_ERR_INVALID_ARG;
    tl_hook.begin = (cudaEvent_t)begin_event;
    tl_hook.end = (cudaEvent_t)end_event;
    return GDN_OK;
}

gdn_status gdn_wait_limit_next_call(int64_t cycles) {
    if (cycles < 0)
        return GDN_ERR_INVALID_ARG;
    tl_wait_limit = (long long)cycles;
    return GDN_OK;
}

gdn_status gdn_prefill_status(const void *workspace, size_t workspace_bytes, uint32_t *detail,
                              void *stream) {
    if (workspace == nullptr || workspace_bytes < 2 * sizeof(uint32_t))
        return GDN_ERR_INVALID_ARG;
    return read_status_words(workspace, detail, (cudaStream_t)stream);
}

const char *gdn_status_string(gdn_status s) {
    switch (s) {
    case GDN_OK: return "success";
    case GDN_ERR_INVALID_ARG: return "invalid argument (pointer, alignment, size or shape)";
    case GDN_ERR_UNSUPPORTED: return "configuration or size outside what the library supports";
    case GDN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case GDN_ERR_CUDA: return "CUDA launch or runtime error";
    case GDN_ERR_TIMEOUT: return "a bounded wait inside a kernel gave up; the outputs are invalid";
    }
    return "unknown status";
}

gdn_status gdn_prefill_workspace_size(const gdn_config *cfg, int32_t batch, int64_t total_tokens,
                                      size_t *bytes) {
    gdn_status st = check_config(cfg);
    if (st != GDN_OK)
        return st;
    if (bytes == nullptr || batch < 0 || total_tokens < 0)
        return GDN_ERR_INVALID_ARG;
    *bytes = prefill_workspace_bytes(cfg, total_tokens, batch);
    return GDN_OK;
}

gdn_status gdn_prefill_segments(const gdn_config *cfg, int32_t batch, int64_t total_tokens,
                                int32_t *segments) {
    gdn_status st = check_config(cfg);
    if (st != GDN_OK)
        return st;
    if (segments == nullptr || batch < 0 || total_tokens < 0)
        return GDN_ERR_INVALID_ARG;
    *segments = prefill_segments(cfg, batch, total_tokens);
    return GDN_OK;
}

gdn_status gdn_prefill(const gdn_config *cfg, const gdn_params *params, const void *qkv,
                       const void *a, const void *b, const void *z, const int32_t *cu_seqlens,
                       int32_t batch, int64_t total_tokens, const float *initial_state,
                       const void *initial_conv, void *y, float *final_state, void *final_conv,
                       float *o_raw, void *workspace, size_t workspace_bytes, void *stream) {
    return prefill_impl(cfg, params, qkv, a, b, z, cu_seqlens, batch, total_tokens, initial_state,
                        initial_conv, y, final_state, final_conv, o_raw, workspace, workspace_bytes,
                        stream, true);
}

} // extern "C"

namespace gdn {

gdn_status prefill_impl(const gdn_config *cfg, const gdn_params *params, const void *qkv,
                        const void *a, const void *b, const void *z, const int32_t *cu_seqlens,
                        int32_t batch, int64_t total_tokens, const float *initial_state,
                        const void *initial_conv, void *y, float *final_state, void *final_conv,
                        float *o_raw, void *workspace, size_t workspace_bytes, void *stream,
                        bool side) {
    size_t need = 0;
    gdn_status st = validate_prefill(cfg, params, qkv, a, b, z, cu_seqlens, batch, total_tokens,
                                     initial_state, initial_conv, y, final_state, final_conv,
                                     o_raw, &need);
    if (st != GDN_OK)
        return st;
    const bool bf16 = cfg->act_dtype == GDN_BF16;
    if (need > 0 && (workspace == nullptr || workspace_bytes < need ||
                     (reinterpret_cast<uintptr_t>(workspace) & 255u)))
        return GDN_ERR_WORKSPACE;

    PrefillArgs p{};
    p.Hk = cfg->num_qk_heads;
    p.Hv = cfg->num_v_heads;
    p.D = cfg->head_dim;
    p.G = p.Hv / p.Hk;
    p.bf16 = bf16;
    p.rms_eps = cfg->rms_eps;
    p.l2_eps = cfg->l2_eps;
    p.q_scale = cfg->q_scale;
    p.qkv = qkv; p.a = a; p.b = b; p.z = z;
    p.cu = cu_seqlens;
    p.batch = batch;
    p.N = total_tokens;
    p.init_state = initial_state;
    p.init_conv = initial_conv;
    p.y = y;
    p.final_state = final_state;
    p.final_conv = final_conv;
    p.o_raw = o_raw;
    p.conv_w = params->conv_w;
    p.A_log = params->A_log;
    p.dt_bias = params->dt_bias;
    p.norm_w = params->norm_w;
    p.chunked = p.D == 128 && cfg->algo != GDN_ALGO_SERIAL;
    const bool vconv = v_conv_in_chunk(p.chunked, bf16); // the chunk kernel convolves v
    if (need > 0) { // the regions of prefill_workspace_bytes, in its order
        char *w = (char *)workspace;
        p.ws_err = (unsigned int *)w;
        p.ws_qk = w + kWorkspaceHeader;
        w = (char *)p.ws_qk + round_up((size_t)total_tokens * 2 * p.Hk * p.D * 4);
        if (!vconv) {
            p.ws_v = w;
            w += round_up((size_t)total_tokens * p.Hv * p.D * 4);
        }
        if (p.chunked) {
            p.ws_kq = w;
            p.ws_kk = (char *)p.ws_kq + round_up(kq_workspace_bytes(p.Hk, total_tokens));
            p.ws_tb = (char *)p.ws_kk + round_up(kk_workspace_bytes(p.Hk, total_tokens, batch));
            p.ws_gt = (float *)((char *)p.ws_tb + round_up(tb_workspace_bytes(p.Hv, total_tokens, batch)));
            p.ws_offs = (int32_t *)((char *)p.ws_gt +
                                    round_up(gt_workspace_bytes(p.Hv, total_tokens, batch)));
            p.segments = prefill_segments(cfg, batch, total_tokens);
            if (p.segments > 1)
                p.ws_seg = (float *)((char *)p.ws_offs + round_up(((size_t)batch + 1) * sizeof(int32_t)));
        }
    }

    cudaStream_t s = (cudaStream_t)stream;
    const ProfileHook hook = take_profile_hook();
    p.wait_limit = take_wait_limit();
    if (batch == 0)
        return GDN_OK;
    // front end.  Token-serial path: conv, SiLU and q/k L2 norm of every
    // channel.  Chunked path: the chunk offsets (which also clear the status
    // words); then, on the side stream, the conv of the v channels, and on the
    // caller's stream the conv of q and k, the intra-chunk Gram rows and the
    // triangular inverses; the chunk kernel waits for both.
    cudaError_t e = cudaSuccess;
    if (!p.chunked) {
        e = launch_conv_prep(p, ConvPart::kAll, s);
    } else if (vconv || !side) { // everything on the caller's stream, in order
        // (16-bit activations: the conv of q and k only; the chunk kernel
        // convolves v from the pre-conv rows)
        e = launch_chunk_offsets(p, s);
        if (e == cudaSuccess)
            e = launch_conv_prep(p, vconv ? ConvPart::kQK : ConvPart::kAll, s);
        if (e == cudaSuccess)
            e = launch_gram(p, s);
        if (e == cudaSuccess)
            e = launch_tri(p, s);
    } else {
        SideStream *ss = nullptr;
        e = launch_chunk_offsets(p, s);
        if (e == cudaSuccess)
            e = side_stream(&ss);
        if (e == cudaSuccess)
            e = cudaEventRecord(ss->fork, s);
        if (e == cudaSuccess)
            e = cudaStreamWaitEvent(ss->stream, ss->fork, 0);
        if (e == cudaSuccess) {
            e = launch_conv_prep(p, ConvPart::kV, ss->stream);
            // the join is recorded (and waited for) whatever the launch did, so
            // that the caller's stream never runs ahead of the side stream
            const cudaError_t e2 = cudaEventRecord(ss->join, ss->stream);
            if (e == cudaSuccess)
                e = e2;
            if (e == cudaSuccess)
                e = launch_conv_prep(p, ConvPart::kQK, s);
            if (e == cudaSuccess)
                e = launch_gram(p, s);
            if (e == cudaSuccess)
                e = launch_tri(p, s);
            const cudaError_t e3 = e2 == cudaSuccess ? cudaStreamWaitEvent(s, ss->join, 0) : e2;
            if (e == cudaSuccess)
                e = e3;
        }
    }
    if (e == cudaSuccess)
        e = record_if(hook.begin, s);
    if (e == cudaSuccess)
        e = p.chunked ? launch_chunk_prefill(p, s) : launch_recurrent_prefill(p, s);
    if (e == cudaSuccess)
        e = record_if(hook.end, s);
    if (e == cudaSuccess)
        e = launch_final_conv(p, s);
    return cuda_status(e);
}

} // namespace gdn

namespace gdn {
namespace {

// The checks and launch shared by the decode entry points.  mode < 0: the
// one-token kernel; otherwise a multi-token mode with `k` tokens per sequence.
gdn_status decode_call(const gdn_config *cfg, const gdn_params *params, const void *qkv,
                       const void *a, const void *b, const void *z, const float *state,
                       const void *conv_cache, int32_t batch, int32_t k, const int32_t *accepted,
                       void *y, void *stream, int mode) {
    gdn_status st = check_config(cfg);
    if (st != GDN_OK)
        return st;
    if ((st = check_params(params)) != GDN_OK)
        return st;
    if (batch < 0 || k < 1)
        return GDN_ERR_INVALID_ARG;
    if (batch > 65535 || k > kDecodeMaxTokens)
        return GDN_ERR_UNSUPPORTED;
    const int G = cfg->num_v_heads / cfg->num_qk_heads;
    if (mode >= 0 && decode_multi_smem_bytes(G, cfg->head_dim, k, mode) > kDecodeMaxSmem)
        return GDN_ERR_UNSUPPORTED;
    if (batch == 0) {
        take_profile_hook();
        return GDN_OK;
    }
    const bool bf16 = cfg->act_dtype == GDN_BF16;
    const bool want_y = mode != kDecodeCommit;
    const bool want_z = want_y;
    if (qkv == nullptr || a == nullptr || b == nullptr || (want_z && z == nullptr) ||
        state == nullptr || conv_cache == nullptr || (want_y && y == nullptr) ||
        (mode == kDecodeCommit && accepted == nullptr))
        return GDN_ERR_INVALID_ARG;
    if (!aligned16(qkv) || !aligned16(z) || !aligned16(y) || !aligned16(state) ||
        !aligned16(conv_cache) || !elem_aligned(a, bf16) || !elem_aligned(b, bf16) ||
        (reinterpret_cast<uintptr_t>(accepted) & 3u))
        return GDN_ERR_INVALID_ARG;
    DecodeArgs p{};
    p.Hk = cfg->num_qk_heads;
    p.Hv = cfg->num_v_heads;
    p.D = cfg->head_dim;
    p.G = G;
    p.bf16 = bf16;
    p.rms_eps = cfg->rms_eps;
    p.l2_eps = cfg->l2_eps;
    p.q_scale = cfg->q_scale;
    p.qkv = qkv; p.a = a; p.b = b; p.z = z;
    p.state = const_cast<float *>(state); // written only by the updating modes
    p.conv_cache = const_cast<void *>(conv_cache);
    p.batch = batch;
    p.y = y;
    p.conv_w = params->conv_w;
    p.A_log = params->A_log;
    p.dt_bias = params->dt_bias;
    p.norm_w = params->norm_w;
    p.k = k;
    p.accepted = accepted;
    cudaStream_t s = (cudaStream_t)stream;
    const ProfileHook hook = take_profile_hook();
    cudaError_t e = record_if(hook.begin, s);
    if (e == cudaSuccess)
        e = mode < 0 ? launch_decode(p, s) : launch_decode_multi(p, mode, s);
    if (e == cudaSuccess)
        e = record_if(hook.end, s);
    return cuda_status(e);
}

} // namespace
} // namespace gdn

extern "C" {

gdn_status gdn_decode(const gdn_config *cfg, const gdn_params *params, const void *qkv,
                      const void *a, const void *b, const void *z, float *state,
                      void *conv_cache, int32_t batch, void *y, void *stream) {
    return decode_call(cfg, params, qkv, a, b, z, state, conv_cache, batch, 1, nullptr, y, stream,
                       -1);
}

gdn_status gdn_decode_multi(const gdn_config *cfg, const gdn_params *params, const void *qkv,
                            const void *a, const void *b, const void *z, float *state,
                            void *conv_cache, int32_t batch, int32_t num_tokens, void *y,
                            void *stream) {
    return decode_call(cfg, params, qkv, a, b, z, state, conv_cache, batch, num_tokens, nullptr, y,
                       stream, kDecodeMulti);
}

gdn_status gdn_decode_verify(const gdn_config *cfg, const gdn_params *params, const void *qkv,
                             const void *a, const void *b, const void *z, const float *state,
                             const void *conv_cache, int32_t batch, int32_t num_tokens, void *y,
                             void *stream) {
    return decode_call(cfg, params, qkv, a, b, z, state, conv_cache, batch, num_tokens, nullptr, y,
                       stream, kDecodeVerify);
}

gdn_status gdn_decode_commit(const gdn_config *cfg, const gdn_params *params, const void *qkv,
                             const void *a, const void *b, float *state, void *conv_cache,
                             int32_t batch, int32_t num_tokens, const int32_t *accepted,
                             void *stream) {
    return decode_call(cfg, params, qkv, a, b, nullptr, state, conv_cache, batch, num_tokens,
                       accepted, nullptr, stream, kDecodeCommit);
}

// ------------------------------------------------------------------- KDA

namespace {

gdn_status kda_check(const gdn_config *cfg, const gdn_kda_params *params) {
    gdn_status st = check_config(cfg);
    if (st != GDN_OK)
        return st;
    if (cfg->num_qk_heads != cfg->num_v_heads) // one q and one k per head
        return GDN_ERR_INVALID_ARG;
    if (cfg->segments > 1) // token-serial: no sequence split
        return GDN_ERR_UNSUPPORTED;
    if (params == nullptr || params->conv_w == nullptr || params->A_log == nullptr ||
        params->norm_w == nullptr || !aligned16(params->conv_w) || !aligned16(params->norm_w) ||
        (reinterpret_cast<uintptr_t>(params->A_log) & 3u))
        return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

} // namespace

gdn_status gdn_kda_prefill_workspace_size(const gdn_config *cfg, int32_t batch, int64_t total_tokens,
                                          size_t *bytes) {
    gdn_status st = check_config(cfg);
    if (st != GDN_OK)
        return st;
    if (cfg->num_qk_heads != cfg->num_v_heads)
        return GDN_ERR_INVALID_ARG;
    if (cfg->segments > 1)
        return GDN_ERR_UNSUPPORTED;
    if (bytes == nullptr || batch < 0 || total_tokens < 0)
        return GDN_ERR_INVALID_ARG;
    // header, normalised q|k, convolved v, and the raw output before the gated norm
    const size_t hd = (size_t)total_tokens * cfg->num_v_heads * cfg->head_dim * 4;
    *bytes = total_tokens == 0 ? 0
                               : kWorkspaceHeader + round_up((size_t)total_tokens * 2 * cfg->num_qk_heads * cfg->head_dim * 4) +
                                     round_up(hd) + round_up(hd);
    return GDN_OK;
}

gdn_status gdn_kda_prefill(const gdn_config *cfg, const gdn_kda_params *params, const void *qkv,
                           const void *zdec, const void *b, const void *gate,
                           const int32_t *cu_seqlens, int32_t batch, int64_t total_tokens,
                           const float *initial_state, const void *initial_conv, void *y,
                           float *final_state, void *final_conv, float *o_raw, void *workspace,
                           size_t workspace_bytes, void *stream) {
    gdn_status st = kda_check(cfg, params);
    if (st != GDN_OK)
        return st;
    if (batch < 0 || total_tokens < 0 || batch > 65535)
        return batch > 65535 ? GDN_ERR_UNSUPPORTED : GDN_ERR_INVALID_ARG;
    if ((batch == 0 && total_tokens > 0) || (batch > 0 && cu_seqlens == nullptr))
        return GDN_ERR_INVALID_ARG;
    const bool bf16 = cfg->act_dtype == GDN_BF16;
    if (total_tokens > 0 && (qkv == nullptr || zdec == nullptr || b == nullptr || gate == nullptr ||
                             y == nullptr))
        return GDN_ERR_INVALID_ARG;
    if (!aligned16(qkv) || !aligned16(zdec) || !aligned16(gate) || !aligned16(y) ||
        !aligned16(initial_state) || !aligned16(initial_conv) || !aligned16(final_state) ||
        !aligned16(final_conv) || !aligned16(o_raw) || !elem_aligned(b, bf16) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
        return GDN_ERR_INVALID_ARG;
    size_t need = 0;
    gdn_kda_prefill_workspace_size(cfg, batch, total_tokens, &need);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need ||
                     (reinterpret_cast<uintptr_t>(workspace) & 255u)))
        return GDN_ERR_WORKSPACE;
    PrefillArgs p{};
    p.Hk = cfg->num_qk_heads;
    p.Hv = cfg->num_v_heads;
    p.D = cfg->head_dim;
    p.G = 1;
    p.bf16 = bf16;
    p.rms_eps = cfg->rms_eps;
    p.l2_eps = cfg->l2_eps;
    p.q_scale = cfg->q_scale;
    p.qkv = qkv; p.b = b; p.z = gate;
    p.kda_zdec = zdec;
    p.cu = cu_seqlens;
    p.batch = batch;
    p.N = total_tokens;
    p.init_state = initial_state;
    p.init_conv = initial_conv;
    p.y = y;
    p.final_state = final_state;
    p.final_conv = final_conv;
    p.o_raw = o_raw;
    p.conv_w = params->conv_w;
    p.A_log = params->A_log;
    p.norm_w = params->norm_w;
    p.chunked = false;
    p.wait_limit = kDefaultWaitLimit;
    if (need > 0) {
        char *w = (char *)workspace;
        p.ws_err = (unsigned int *)w;
        p.ws_qk = w + kWorkspaceHeader;
        p.ws_v = (char *)p.ws_qk + round_up((size_t)total_tokens * 2 * p.Hk * p.D * 4);
        p.ws_o = (float *)((char *)p.ws_v + round_up((size_t)total_tokens * p.Hv * p.D * 4));
    }
    cudaStream_t s = (cudaStream_t)stream;
    const ProfileHook hook = take_profile_hook();
    if (batch == 0)
        return GDN_OK;
    cudaError_t e = launch_conv_prep(p, ConvPart::kAll, s);
    if (e == cudaSuccess)
        e = record_if(hook.begin, s);
    if (e == cudaSuccess)
        e = launch_kda_prefill(p, s);
    if (e == cudaSuccess)
        e = record_if(hook.end, s);
    if (e == cudaSuccess)
        e = launch_final_conv(p, s);
    return cuda_status(e);
}

gdn_status gdn_kda_decode(const gdn_config *cfg, const gdn_kda_params *params, const void *qkv,
                          const void *zdec, const void *b, const void *gate, float *state,
                          void *conv_cache, int32_t batch, void *y, void *stream) {
    gdn_status st = kda_check(cfg, params);
    if (st != GDN_OK)
        return st;
    if (batch < 0)
        return GDN_ERR_INVALID_ARG;
    if (batch > 65535)
        return GDN_ERR_UNSUPPORTED;
    if (batch == 0) {
        take_profile_hook();
        return GDN_OK;
    }
    const bool bf16 = cfg->act_dtype == GDN_BF16;
    if (qkv == nullptr || zdec == nullptr || b == nullptr || gate == nullptr || state == nullptr ||
        conv_cache == nullptr || y == nullptr)
        return GDN_ERR_INVALID_ARG;
    if (!aligned16(qkv) || !aligned16(zdec) || !aligned16(gate) || !aligned16(y) ||
        !aligned16(state) || !aligned16(conv_cache) || !elem_aligned(b, bf16))
        return GDN_ERR_INVALID_ARG;
    DecodeArgs p{};
    p.Hk = cfg->num_qk_heads;
    p.Hv = cfg->num_v_heads;
    p.D = cfg->head_dim;
    p.G = 1;
    p.bf16 = bf16;
    p.rms_eps = cfg->rms_eps;
    p.l2_eps = cfg->l2_eps;
    p.q_scale = cfg->q_scale;
    p.qkv = qkv; p.b = b; p.z = gate;
    p.kda_zdec = zdec;
    p.state = state;
    p.conv_cache = conv_cache;
    p.batch = batch;
    p.y = y;
    p.conv_w = params->conv_w;
    p.A_log = params->A_log;
    p.norm_w = params->norm_w;
    cudaStream_t s = (cudaStream_t)stream;
    const ProfileHook hook = take_profile_hook();
    cudaError_t e = record_if(hook.begin, s);
    if (e == cudaSuccess)
        e = launch_kda_decode(p, s);
    if (e == cudaSuccess)
        e = record_if(hook.end, s);
    return cuda_status(e);
}

} // extern "C"
