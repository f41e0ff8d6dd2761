/*
 * gdn.h -- C ABI of the B200 (sm_100a) Gated DeltaNet token mixer.
 *
 * The layer is the linear-attention mixer that fills 69 of the 92 layers of
 * Qwen3.8-2.4T-A95B ("Qwen3.8-2.4T-A95B vs Inkling", component table, Gated
 * DeltaNet row; "Qwen3.8 2.4T A95B", key facts, layer stack "Linear x69").
 * Per token it
 *   1. runs a depthwise causal convolution of kernel 4 (no bias) + SiLU over
 *      the q, k and v channels (Gated DeltaNet row; raw config field
 *      linear_conv_kernel_dim = 4),
 *   2. L2-normalises q and k per q/k head,
 *   3. forms per value head the decay g = -exp(A_log) * softplus(a + dt_bias)
 *      and the write strength beta = sigmoid(b) (Gated DeltaNet row),
 *   4. applies the gated delta rule to an FP32 d_v x d_k state per value head
 *      (raw config field mamba_ssm_dtype = float32),
 *         S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *         o_t = S_t q_t,
 *      where value head h reads q/k head h / (H_v / H_k) (Gated DeltaNet row:
 *      16 q/k heads serve 128 value heads, 8 each),
 *   5. normalises o per value head by RMS (eps = rms_norm_eps = 1e-6, raw
 *      config fields) and multiplies by a weight and by SiLU(z) ("Qwen3.8-
 *      2.4T-A95B vs Inkling", component table, output-gate row:
 *      output_gate_type swish after a per-head RMSNorm).
 * The in- and out-projections that produce qkv, a, b, z and consume y are
 * not part of this library.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers (cudaMalloc'd or equivalent) on
 *     the current device, except the gdn_config / gdn_params structs and the
 *     `bytes` out-parameter, which are host memory.  The caller owns every
 *     buffer; the library allocates nothing.
 *   - Tensors are row-major and contiguous; every tensor pointer must be
 *     16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued on it; no entry point synchronises the host.
 *   - Argument errors are detected on the host before anything is launched
 *     and return GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED or
 *     GDN_ERR_WORKSPACE; launch failures return GDN_ERR_CUDA.  Nothing traps
 *     and no C++ exception crosses the ABI.  Entry points are stateless and
 *     may be called from several host threads at once.
 *   - Channel layout of a pre-conv qkv row (conv_dim = (2 H_k + H_v) d):
 *     q of q/k head j at [j d, (j+1) d), k of head j at [H_k d + j d, ...),
 *     v of value head h at [2 H_k d + h d, ...).
 *   - The state of one value head is stored [d_v][d_k] (row = value channel).
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_ABI_VERSION 3

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

typedef enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1, /* NULL/misaligned pointer, bad size or inconsistent shape */
    GDN_ERR_UNSUPPORTED = 2, /* well-formed, but no kernel for this shape (head_dim, kernel) */
    GDN_ERR_WORKSPACE = 3,   /* workspace NULL, misaligned or smaller than the size query says */
    GDN_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed */
    GDN_ERR_TIMEOUT = 5      /* a bounded wait inside a kernel gave up (device status word);
                                returned only by the status queries below */
} gdn_status;

typedef enum gdn_dtype {
    GDN_F32 = 0, /* float32 activations */
    GDN_BF16 = 1 /* bfloat16 activations */
} gdn_dtype;

/* Head layout and scalar settings of one layer. */
typedef struct gdn_config {
    int32_t num_qk_heads; /* H_k >= 1 */
    int32_t num_v_heads;  /* H_v, a multiple of H_k (G = H_v / H_k value heads per q/k head) */
    int32_t head_dim;     /* d = d_k = d_v; the library supports 32 and 128 */
    int32_t conv_kernel;  /* causal conv width; the library supports 4 */
    float rms_eps;        /* epsilon of the gated RMSNorm (1e-6 for Qwen3.8) */
    float l2_eps;         /* epsilon inside the q/k L2 norm: x / sqrt(sum x^2 + l2_eps) */
    float q_scale;        /* extra factor on normalised q (1.0 = none) */
    int32_t act_dtype;    /* gdn_dtype of qkv, a, b, z, y and the conv caches */
    int32_t algo;         /* gdn_algo: prefill algorithm (GDN_ALGO_AUTO = 0 is right for most callers) */
    int32_t segments;     /* chunked prefill: segments per sequence (see below); 0 = the library's choice */
} gdn_config;

/*
 * Sequence split of the chunked prefill (gdn_config.segments).
 *
 * The state map of a stretch of tokens is affine in the state entering it,
 * S_end = S_0 M + R, with M the product of the per-token factors
 * exp(g_t) (I - beta_t k_t k_t^T) and R the state the stretch reaches from
 * S_0 = 0 (the Gated DeltaNet update of "Qwen3.8-2.4T-A95B vs Inkling",
 * component table; "Qwen3.8 2.4T A95B", key facts: a 262,144-token context).
 * With segments = P >= 2 every sequence is cut at chunk boundaries into P
 * segments of equal chunk count.  A summary pass computes (M, R) of the first
 * P - 1 segments of every (sequence, value head) in parallel, a short FP32
 * pass chains them into the state entering each segment, and the output pass
 * then scans all P segments in parallel.  The results are those of P = 1 up to
 * rounding.  It pays when batch * H_v is small against the GPU's 148 SMs and
 * the sequences are long.
 *   0      the library's choice: 1 unless batch * H_v <= 74, else the P in
 *          2..16 that a cost model of the two passes favours, with at least
 *          32 chunks (2,048 tokens) per segment on average
 *   1      no split: one chain per (sequence, value head)
 *   2..16  that many segments (a sequence shorter than P chunks leaves some
 *          segments empty)
 * The token-serial path and the KDA entry points take 0 or 1 only
 * (GDN_ERR_UNSUPPORTED otherwise); decode ignores the field.  The workspace
 * size query counts the split's workspace: 3 (P - 1) batch H_v d^2 floats.
 */

/* Prefill algorithm.  Both compute the same recurrence; decode ignores it. */
typedef enum gdn_algo {
    GDN_ALGO_AUTO = 0,    /* chunked for head_dim 128, token-serial otherwise */
    GDN_ALGO_SERIAL = 1,  /* token-serial FP32 recurrence on CUDA cores (any head_dim) */
    GDN_ALGO_CHUNKED = 2  /* 64-token chunks on the tensor cores (head_dim 128 only) */
} gdn_algo;

/* Layer parameters, all float32 device arrays. */
typedef struct gdn_params {
    const float *conv_w;  /* [conv_dim, conv_kernel]; tap conv_kernel-1 multiplies the current token */
    const float *A_log;   /* [H_v] */
    const float *dt_bias; /* [H_v] */
    const float *norm_w;  /* [d], shared by all value heads */
} gdn_params;

/*
 * Bytes of device workspace gdn_prefill needs for `total_tokens` packed
 * tokens in `batch` sequences.  Writes *bytes; returns GDN_ERR_INVALID_ARG for
 * a bad config or negative sizes, GDN_ERR_UNSUPPORTED for an unsupported one.
 */
GDN_API gdn_status gdn_prefill_workspace_size(const gdn_config *cfg, int32_t batch, int64_t total_tokens,
                                      size_t *bytes);

/*
 * Segments per sequence (see gdn_config.segments) that gdn_prefill runs with
 * for `total_tokens` packed tokens in `batch` sequences: cfg->segments when
 * it is nonzero on the chunked path, the library's choice when it is 0, and 1
 * on the token-serial path or without tokens.  Writes *segments; errors as
 * gdn_prefill_workspace_size.
 */
GDN_API gdn_status gdn_prefill_segments(const gdn_config *cfg, int32_t batch, int64_t total_tokens,
                                        int32_t *segments);

/*
 * Prefill over a packed varlen batch: sequence n owns token rows
 * cu_seqlens[n] .. cu_seqlens[n+1]-1 of every [N, ...] tensor, N = total_tokens.
 *
 *   qkv           [N, conv_dim]      act_dtype   pre-conv q|k|v rows
 *   a, b          [N, H_v]           act_dtype   gate inputs
 *   z             [N, H_v, d]        act_dtype   output-gate input
 *   cu_seqlens    [batch+1]          int32, DEVICE; cu_seqlens[0] = 0,
 *                                    non-decreasing, cu_seqlens[batch] = N
 *                                    (zero-length sequences are allowed: their
 *                                    state and conv window pass through)
 *   initial_state [batch, H_v, d, d] float32, or NULL for zero states
 *   initial_conv  [batch, K-1, conv_dim] act_dtype: the K-1 pre-conv rows
 *                                    before each sequence, oldest first; NULL = zeros
 *   y             [N, H_v, d]        act_dtype   output (gated RMSNorm of o)
 *   final_state   [batch, H_v, d, d] float32, or NULL to skip; may equal
 *                                    initial_state (in-place update)
 *   final_conv    [batch, K-1, conv_dim] act_dtype, or NULL to skip: the last
 *                                    K-1 pre-conv rows of [initial_conv; sequence];
 *                                    may equal initial_conv
 *   o_raw         [N, H_v, d]        float32 pre-norm recurrence output, or NULL
 *   workspace     device scratch of at least gdn_prefill_workspace_size bytes,
 *                 256-byte aligned; its contents on entry do not matter.  Its
 *                 first 4 bytes become a status word: 0 after a successful
 *                 call; nonzero if a wait inside a kernel gave up (the call's
 *                 outputs are then invalid).  gdn_prefill_status reads it.
 * The values of cu_seqlens are read on the device only; a cu_seqlens array
 * that breaks the rules above gives unspecified output (never an
 * out-of-bounds access outside [0, N) rows).
 */
GDN_API gdn_status gdn_prefill(const gdn_config *cfg, const gdn_params *params, const void *qkv,
                       const void *a, const void *b, const void *z, const int32_t *cu_seqlens,
                       int32_t batch, int64_t total_tokens, const float *initial_state,
                       const void *initial_conv, void *y, float *final_state, void *final_conv,
                       float *o_raw, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Device-side outcome of the last gdn_prefill that used `workspace`.
 *
 * The chunked kernels hand work between warps through barriers whose waits
 * are bounded (about one second of SM clock); a wait that gives up makes the
 * whole call abort cleanly (no fault, no hang) and leaves bits in the status
 * word at the start of the workspace.  This call waits for `stream` (the
 * stream the prefill ran on) to finish, then reads that word:
 *   GDN_OK           the call completed normally,
 *   GDN_ERR_TIMEOUT  a bounded wait gave up; the call's outputs are invalid,
 *   GDN_ERR_CUDA     the stream reported an error, or a kernel found its
 *                    shared-memory window misaligned,
 *   GDN_ERR_INVALID_ARG  workspace NULL or shorter than the 8-byte header.
 * `detail` (host, may be NULL) receives the second word of the header: 0, or
 * where the first timed-out wait gave up (0x80000000 | warp << 24 | barrier
 * index << 16 | waits that warp had completed).  A workspace that no prefill
 * has used holds unspecified bytes.  Synchronises the host with `stream`.
 */
GDN_API gdn_status gdn_prefill_status(const void *workspace, size_t workspace_bytes,
                                      uint32_t *detail, void *stream);

/*
 * Testing hook for the bounded waits above.  Arms a one-shot on the calling
 * host thread: the next gdn_prefill or gdn_prefill_noalloc call made by this
 * thread gives each wait between the warps of its chunked kernel `cycles` SM
 * cycles instead of the default of 2e9 (about one second), so that a test can
 * make a wait run out and check the abort path and gdn_prefill_status.  The
 * waits that let a kernel's own in-flight copies and tensor-core work finish
 * before it exits keep the default.  cycles = 0 disarms.  Returns
 * GDN_ERR_INVALID_ARG for a negative value.
 */
GDN_API gdn_status gdn_wait_limit_next_call(int64_t cycles);

/*
 * Decode: one new token for each of `batch` sequences against their resident
 * states, updated in place.
 *
 *   qkv        [batch, conv_dim]      act_dtype   the new tokens' pre-conv rows
 *   a, b       [batch, H_v]           act_dtype
 *   z          [batch, H_v, d]        act_dtype
 *   state      [batch, H_v, d, d]     float32, in/out
 *   conv_cache [batch, K-1, conv_dim] act_dtype, in/out: the last K-1 pre-conv
 *                                     rows, oldest first; on return the oldest
 *                                     row is dropped and the new row appended
 *   y          [batch, H_v, d]        act_dtype   output
 * Needs no workspace.
 */
GDN_API gdn_status gdn_decode(const gdn_config *cfg, const gdn_params *params, const void *qkv,
                      const void *a, const void *b, const void *z, float *state,
                      void *conv_cache, int32_t batch, void *y, void *stream);

/*
 * Multi-token decode: num_tokens (k, 1..8) new tokens for each of `batch`
 * sequences against their resident states, applied in order; state and conv
 * cache advance by all k tokens, in place.  This is what decoding several
 * tokens per step needs, e.g. the draft tokens of the multi-token-prediction
 * layer of Qwen3.8 ("Qwen3.8 2.4T A95B", key facts: one extra MTP layer used
 * to accelerate decoding; raw config field mtp_num_hidden_layers 1) once they
 * are all accepted.  Each state row is read once and written once for the k
 * tokens.  The result equals k calls of gdn_decode, and a prefill of the same
 * k tokens continuing the sequence.
 *
 *   qkv        [batch, k, conv_dim]   act_dtype
 *   a, b       [batch, k, H_v]        act_dtype
 *   z          [batch, k, H_v, d]     act_dtype
 *   state      [batch, H_v, d, d]     float32, in/out
 *   conv_cache [batch, K-1, conv_dim] act_dtype, in/out
 *   y          [batch, k, H_v, d]     act_dtype   output of every token
 * Returns GDN_ERR_UNSUPPORTED for k > 8, or when k tokens of one q/k head
 * group do not fit the kernel's shared memory (k * G * d * 8 bytes and a
 * little more; every G <= 16 at d = 128 fits k = 8).  Needs no workspace.
 */
GDN_API gdn_status gdn_decode_multi(const gdn_config *cfg, const gdn_params *params,
                                    const void *qkv, const void *a, const void *b, const void *z,
                                    float *state, void *conv_cache, int32_t batch,
                                    int32_t num_tokens, void *y, void *stream);

/*
 * Speculative decoding, step 1 of 2: the outputs y of k draft tokens per
 * sequence (layout as gdn_decode_multi), computed against the resident state
 * and conv cache WITHOUT changing either (both are only read).  The state is
 * read once for all k tokens.  After the caller has decided how many leading
 * tokens of each sequence it keeps, gdn_decode_commit takes exactly those.
 */
GDN_API gdn_status gdn_decode_verify(const gdn_config *cfg, const gdn_params *params,
                                     const void *qkv, const void *a, const void *b, const void *z,
                                     const float *state, const void *conv_cache, int32_t batch,
                                     int32_t num_tokens, void *y, void *stream);

/*
 * Speculative decoding, step 2 of 2: advance each sequence's state and conv
 * cache, in place, by its first accepted[n] of the num_tokens tokens given
 * (the same qkv, a, b as the verify call; z is not needed).  accepted is a
 * DEVICE int32 array [batch]; values are clamped to [0, num_tokens], and a
 * sequence with 0 is left untouched.  Rejected draft tokens never reach the
 * state, so nothing has to be rolled back.  The result equals gdn_decode_multi
 * over the accepted tokens.
 */
GDN_API gdn_status gdn_decode_commit(const gdn_config *cfg, const gdn_params *params,
                                     const void *qkv, const void *a, const void *b, float *state,
                                     void *conv_cache, int32_t batch, int32_t num_tokens,
                                     const int32_t *accepted, void *stream);

/*
 * Kimi Delta Attention (KDA), the per-channel-decay variant of the mixer
 * ("Inkling vs Kimi K3", component table, linear-attention row: 96 heads of
 * dimension 128, kernel-4 conv + SiLU on q, k and v, L2-normalised q and k,
 * per-channel log-decay g = -5 sigmoid(exp(A) z); output-gate row: the
 * head-wise RMSNorm of the recurrent output times a full-rank channel-wise
 * sigmoid gate).  Per head (one q, k and v head each: cfg->num_qk_heads must
 * equal cfg->num_v_heads) and token, with alpha = exp(g) in R^{d_k}:
 *     S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = S_t q_t,   beta_t = sigmoid(b_t),
 *     y_t = o_t / sqrt(mean(o_t^2) + rms_eps) * norm_w * sigmoid(gate_t).
 * Arithmetic is FP32 on CUDA cores: the prefill takes two tokens per step (an
 * exact refactoring of the recurrence above), the decode one token.
 */
typedef struct gdn_kda_params {
    const float *conv_w; /* [3 H d, conv_kernel] (q heads, k heads, v heads) */
    const float *A_log;  /* [H]: the decay scale exp(A_log[h]) of head h */
    const float *norm_w; /* [d], shared by all heads */
} gdn_kda_params;

/*
 * Workspace bytes of gdn_kda_prefill (as gdn_prefill_workspace_size): a
 * 256-byte header, float32 normalised q|k [N, 2 H d], float32 convolved v
 * [N, H d] and the float32 raw output [N, H, d] before the gated norm, each
 * region rounded up to 256 bytes; 0 when total_tokens is 0.  Requires
 * num_qk_heads == num_v_heads (GDN_ERR_INVALID_ARG otherwise) and segments
 * 0 or 1 (GDN_ERR_UNSUPPORTED otherwise).
 */
GDN_API gdn_status gdn_kda_prefill_workspace_size(const gdn_config *cfg, int32_t batch,
                                                  int64_t total_tokens, size_t *bytes);

/*
 * KDA prefill over a packed varlen batch; conventions, cu_seqlens, states,
 * conv windows, o_raw and workspace as in gdn_prefill.
 *   qkv   [N, 3 H d]  act_dtype   pre-conv q|k|v rows
 *   zdec  [N, H, d]   act_dtype   per-channel decay inputs z
 *   b     [N, H]      act_dtype   write-strength inputs
 *   gate  [N, H, d]   act_dtype   output-gate inputs (sigmoid applied here)
 *   y     [N, H, d]   act_dtype   output
 */
GDN_API gdn_status gdn_kda_prefill(const gdn_config *cfg, const gdn_kda_params *params,
                                   const void *qkv, const void *zdec, const void *b,
                                   const void *gate, const int32_t *cu_seqlens, int32_t batch,
                                   int64_t total_tokens, const float *initial_state,
                                   const void *initial_conv, void *y, float *final_state,
                                   void *final_conv, float *o_raw, void *workspace,
                                   size_t workspace_bytes, void *stream);

/*
 * KDA decode: one token per sequence against resident states, which are
 * updated in place, as is the conv cache (layouts as gdn_decode, with zdec
 * [batch, H, d], b [batch, H] and gate [batch, H, d]).  Needs no workspace.
 */
GDN_API gdn_status gdn_kda_decode(const gdn_config *cfg, const gdn_kda_params *params,
                                  const void *qkv, const void *zdec, const void *b,
                                  const void *gate, float *state, void *conv_cache, int32_t batch,
                                  void *y, void *stream);

/*
 * Size of the fixed device scratch array used by gdn_prefill_noalloc:
 * 64 MiB, held on every GPU that loads the library until the process exits.
 */
#define GDN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * gdn_prefill for callers that cannot allocate device memory.  (The pages
 * have no counterpart of this entry point; it exists for integration.)
 *
 * Some callers cannot obtain device scratch at call time: a plugin hosted by
 * a framework that owns all of the GPU's memory and hands it only the input
 * and output buffers, or a latency-critical loop that must never call
 * cudaMalloc/cudaFree, which can synchronise the whole device.  This entry
 * point takes the same arguments as gdn_prefill minus the workspace; its
 * scratch is one fixed array of GDN_NOALLOC_SCRATCH_BYTES inside the library,
 * and it allocates nothing.
 *
 *   - Limit: a call whose gdn_prefill_workspace_size exceeds
 *     GDN_NOALLOC_SCRATCH_BYTES returns GDN_ERR_WORKSPACE before any CUDA
 *     call (at the Qwen3.8 layer shape with 16-bit activations, about
 *     72.5 KiB per token plus 3.3 MiB per sequence: up to 832 tokens of one
 *     sequence).
 *   - Set-up: the first call on a device, with that device current, looks up
 *     the array's device address (cudaGetSymbolAddress) and caches it; make
 *     that first call before any stream capture.
 *   - Sharing: every call on a device uses the same array, which keeps the
 *     last call's contents.  Nothing in it needs to start at zero.  Calls
 *     whose work overlaps on the GPU (different streams or host threads on
 *     the same device) race on the array and give wrong results: order them.
 *   - Device status: the status word that gdn_prefill leaves in its
 *     workspace lives here in the fixed array, out of the caller's reach;
 *     read it with gdn_prefill_noalloc_status.
 *   - A device reset (cudaDeviceReset) after the first call on that device
 *     is not supported: the cached address would be stale.
 * Validates its arguments exactly as gdn_prefill does (same codes, same
 * order); only then a call that needs more than the fixed array returns
 * GDN_ERR_WORKSPACE.  Nothing is launched by a rejected call.  Returns
 * GDN_ERR_CUDA if the address look-up fails.
 */
GDN_API gdn_status gdn_prefill_noalloc(const gdn_config *cfg, const gdn_params *params,
                                       const void *qkv, const void *a, const void *b,
                                       const void *z, const int32_t *cu_seqlens, int32_t batch,
                                       int64_t total_tokens, const float *initial_state,
                                       const void *initial_conv, void *y, float *final_state,
                                       void *final_conv, float *o_raw, void *stream);

/*
 * gdn_prefill_status for gdn_prefill_noalloc: waits for `stream`, then reads
 * the status word of the fixed scratch array on the current device (the
 * outcome of the last gdn_prefill_noalloc call there).  Returns GDN_OK when
 * no such call has been made on this device.  Allocates nothing.
 */
GDN_API gdn_status gdn_prefill_noalloc_status(uint32_t *detail, void *stream);

/*
 * Timing hook for benchmarks.  Arms a one-shot on the calling host thread:
 * the next gdn_prefill or gdn_decode call made by this thread records
 * `begin_event` on its stream immediately before launching its main kernel
 * (the recurrence) and `end_event` immediately after it, so that
 * cudaEventElapsedTime gives that kernel's device time alone.  Both are
 * cudaEvent_t handles created by the caller; pass NULL, NULL to disarm.  A
 * call that fails argument checks leaves the hook armed.  Returns
 * GDN_ERR_INVALID_ARG if exactly one event is NULL.
 */
GDN_API gdn_status gdn_profile_next_call(void *begin_event, void *end_event);

/* Static English text for a status code (never NULL). */
GDN_API const char *gdn_status_string(gdn_status status);

/* GDN_ABI_VERSION of the loaded library. */
GDN_API int32_t gdn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
