// gdn_conv.cuh -- the per-thread body of the prefill front end: depthwise causal
// conv (kernel 4) + SiLU over one vector of q|k|v channels (8 or 16 bytes) for
// up to 8 tokens, L2 normalisation of q and k per q/k head, FP32 results into
// the workspace.
//
// The conv, its kernel size and the SiLU follow the Gated DeltaNet row of the
// component table on "Qwen3.8-2.4T-A95B vs Inkling" (and linear_conv_kernel_dim
// in the raw config fields of "Qwen3.8 2.4T A95B"); the q/k normalisation is
// the L2 norm the layer applies before its recurrence.
#pragma once

#include "gdn_common.cuh"

namespace gdn {

constexpr int kConvTokens = 8; // tokens per thread

// float32 -> tf32, round to nearest with ties away from zero (the same rule
// as tf32_rna of gdn_sm100.cuh, without needing that header here)
__device__ __forceinline__ float round_tf32(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xffffe000u);
}

// Loads of one thread's channel vector: Vec16<T> (16 bytes) or Vec8bf (8 bytes of bf16).
template <typename VecT, typename T> struct VecIO;
template <typename T> struct VecIO<Vec16<T>, T> {
    static __device__ __forceinline__ Vec16<T> load(const T *p) { return ld16_nc(p); }
    static __device__ __forceinline__ Vec16<T> zero() { return zero16<T>(); }
};
template <> struct VecIO<Vec8bf, __nv_bfloat16> {
    static __device__ __forceinline__ Vec8bf load(const __nv_bfloat16 *p) {
        Vec8bf v;
        v.raw = __ldg(reinterpret_cast<const uint2 *>(p));
        return v;
    }
    static __device__ __forceinline__ Vec8bf zero() {
        Vec8bf v;
        v.raw = make_uint2(0u, 0u);
        return v;
    }
};

template <typename T> struct ConvIO {
    const T *qkv;          // [N, C] pre-conv q|k|v rows
    const int32_t *cu;     // [batch + 1] sequence offsets
    int batch;
    int64_t N;
    const T *init_conv;    // [batch, 3, C] or null (zeros)
    const float *conv_w;   // [C, 4]
    int Hk, Hv;
    float l2_eps, q_scale;
    float *qk_out;         // [N, 2 Hk D] normalised q | k
    float *v_out;          // [N, Hv D] convolved v (nullptr: v is not written; the chunk kernel
                           // of 16-bit activations convolves v itself)
    bool round_v;          // v to its tf32 operand (tensor-core path)
    int block_y0;          // channel block of blockIdx.y = 0 (skips the q/k-only blocks)
};

// One thread: channels cc .. cc + V - 1 (V = the vector's elements) for the tokens
// t0 .. tend - 1 (at most kConvTokens; tend <= N), n = the sequence of t0,
// given rows[k] = the pre-conv row t0 - 3 + k of those channels (zero outside
// [0, N)).  Tokens whose taps reach before the start of their sequence read
// the initial conv window (or zeros) from global memory instead.
// The lanes holding one q/k head must be an aligned group of D / V lanes of
// the warp, and t0 / tend must be uniform over the warp (the norm shuffles).
// Inactive lanes (active = false, cc any valid channel) join the shuffles only.
// V_ONLY: the caller guarantees that every lane of the warp holds v channels
// (no norm, no reduction).
template <typename T, int D, bool V_ONLY = false, typename VecT = Vec16<T>>
__device__ __forceinline__ void conv_emit(const ConvIO<T> &io, int cc, bool active, int64_t t0,
                                          int64_t tend, int n, const VecT (&rows)[kConvTokens + 3]) {
    constexpr int V = VecT::N;
    constexpr int LANES = D / V; // lanes per head
    static_assert(LANES >= 1 && LANES <= 32 && (32 % LANES) == 0, "head must tile a warp");
    const int C = (2 * io.Hk + io.Hv) * D;
    const int region = V_ONLY ? 2 : (cc < io.Hk * D ? 0 : (cc < 2 * io.Hk * D ? 1 : 2)); // q, k, v
    float w[V][4];
#pragma unroll
    for (int i = 0; i < V; ++i) {
        float4 wv = __ldg(reinterpret_cast<const float4 *>(io.conv_w) + (cc + i));
        w[i][0] = wv.x; w[i][1] = wv.y; w[i][2] = wv.z; w[i][3] = wv.w;
    }
    int64_t start = __ldg(io.cu + n), next = __ldg(io.cu + n + 1);
    // q and k leave L2-normalised (the warp reduces only if some lane holds q
    // or k), v as is; all in float32 so that no rounding is added before the
    // recurrence, except that v, when only the tensor-core path reads it, is
    // rounded to its tf32 operand here
    const bool norm_warp = V_ONLY ? false : __any_sync(0xffffffffu, region < 2);
    auto emit = [&](int64_t t, float (&acc)[V]) {
        if (V_ONLY) {
            if (!active || io.v_out == nullptr)
                return;
            float *dst = io.v_out + t * ((int64_t)io.Hv * D) + (cc - 2 * io.Hk * D);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                acc[i] = siluf_(acc[i]);
                if (io.round_v) {
                    acc[i] = round_tf32(acc[i]);
                }
            }
#pragma unroll
            for (int i = 0; i < V; i += 4)
                *reinterpret_cast<float4 *>(dst + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
            return;
        }
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            acc[i] = siluf_(acc[i]);
            ss = fmaf(acc[i], acc[i], ss);
        }
        if (norm_warp)
            ss = group_sum<LANES>(ss);
        if (!active || (region == 2 && io.v_out == nullptr))
            return;
        const float f = region == 2 ? 1.0f : rsqrtf(ss + io.l2_eps) * (region == 0 ? io.q_scale : 1.0f);
        if (region == 2 && io.round_v) {
#pragma unroll
            for (int i = 0; i < V; ++i) {
                acc[i] = round_tf32(acc[i]);
            }
        }
        float *dst = region < 2 ? io.qk_out + t * (2 * io.Hk * D) + cc
                                : io.v_out + t * ((int64_t)io.Hv * D) + (cc - 2 * io.Hk * D);
#pragma unroll
        for (int i = 0; i < V; i += 4)
            *reinterpret_cast<float4 *>(dst + i) =
                make_float4(acc[i] * f, acc[i + 1] * f, acc[i + 2] * f, acc[i + 3] * f);
    };
    if (start <= t0 - 3 && next >= tend) {
        // one sequence covers every tap of every token (the usual case)
#pragma unroll
        for (int tt = 0; tt < kConvTokens; ++tt) {
            if (t0 + tt >= tend)
                break; // uniform over the warp
            float acc[V];
#pragma unroll
            for (int i = 0; i < V; ++i)
                acc[i] = w[i][0] * rows[tt].get(i);
#pragma unroll
            for (int tap = 1; tap < 4; ++tap)
#pragma unroll
                for (int i = 0; i < V; ++i)
                    acc[i] = fmaf(w[i][tap], rows[tt + tap].get(i), acc[i]);
            emit(t0 + tt, acc);
        }
        return;
    }
#pragma unroll 1
    for (int tt = 0; tt < kConvTokens; ++tt) {
        const int64_t t = t0 + tt;
        if (t >= tend)
            break; // uniform over the warp
        while (t >= next && n + 1 < io.batch) { // t starts a new sequence (after any empty ones)
            ++n;
            start = next;
            next = __ldg(io.cu + n + 1);
        }
        const int64_t st = start > t ? t : (start < 0 ? 0 : start); // malformed cu_seqlens stay in bounds
        float acc[V];
#pragma unroll
        for (int i = 0; i < V; ++i)
            acc[i] = 0.f;
#pragma unroll
        for (int tap = 0; tap < 4; ++tap) {
            const int64_t src = t - 3 + tap;
            VecT x;
            if (src >= st)
                x = VecIO<VecT, T>::load(io.qkv + src * C + cc); // rows[] would need a dynamic index here
            else if (io.init_conv != nullptr)
                x = VecIO<VecT, T>::load(io.init_conv + ((int64_t)n * 3 + (3 + (src - st))) * C + cc);
            else
                x = VecIO<VecT, T>::zero();
#pragma unroll
            for (int i = 0; i < V; ++i)
                acc[i] = fmaf(w[i][tap], x.get(i), acc[i]);
        }
        emit(t, acc);
    }
}

// conv_emit with the rows loaded from global memory first, so that all their
// loads overlap.
template <typename T, int D, bool V_ONLY = false, typename VecT = Vec16<T>>
__device__ __forceinline__ void conv_thread(const ConvIO<T> &io, int cc, bool active, int64_t t0,
                                            int64_t tend, int n) {
    const int C = (2 * io.Hk + io.Hv) * D;
    VecT rows[kConvTokens + 3];
#pragma unroll
    for (int k = 0; k < kConvTokens + 3; ++k) {
        const int64_t src = t0 - 3 + k;
        rows[k] = (src >= 0 && src < io.N) ? VecIO<VecT, T>::load(io.qkv + src * C + cc)
                                          : VecIO<VecT, T>::zero();
    }
    conv_emit<T, D, V_ONLY, VecT>(io, cc, active, t0, tend, n, rows);
}

} // namespace gdn
