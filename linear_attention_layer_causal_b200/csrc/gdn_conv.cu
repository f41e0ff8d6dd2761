// gdn_conv.cu -- prefill front end: depthwise causal conv (kernel 4) + SiLU over
// the q|k|v channels, L2 normalisation of q and k per q/k head, and the final
// conv window of every sequence.
//
// The conv, its kernel size and the SiLU follow the Gated DeltaNet row of the
// component table on "Qwen3.8-2.4T-A95B vs Inkling" (and linear_conv_kernel_dim
// in the raw config fields of "Qwen3.8 2.4T A95B"); the q/k normalisation is
// the L2 norm the layer applies before its recurrence.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

constexpr int kConvThreads = 256;
constexpr int kConvTokens = 8; // tokens per thread

// One thread: 16 bytes of channels (V = 8 bf16 or 4 float) for kConvTokens
// consecutive packed tokens.  The lanes covering one head are consecutive and
// the head width d / V divides 32, so the L2 reduction is a shuffle within an
// aligned lane group.
template <typename T, int D>
__global__ void __launch_bounds__(kConvThreads)
conv_prep_kernel(const T *__restrict__ qkv, const int32_t *__restrict__ cu, int batch,
                 int64_t N, const T *__restrict__ init_conv, const float *__restrict__ conv_w,
                 int Hk, int Hv, float l2_eps, float q_scale, float *__restrict__ qk_out,
                 float *__restrict__ v_out, unsigned int *__restrict__ err, bool round_v) {
    constexpr int V = Vec16<T>::N;
    constexpr int LANES = D / V; // lanes per head
    static_assert(LANES >= 1 && LANES <= 32 && (32 % LANES) == 0, "head must tile a warp");
    const int C = (2 * Hk + Hv) * D;
    if (err != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
        err[0] = 0u; // status word of this call; later kernels only set bits
        err[1] = 0u; // where the first timed-out wait gave up
    }
    const int c0 = (blockIdx.y * kConvThreads + threadIdx.x) * V;
    const bool active = c0 < C;
    const int cc = active ? c0 : 0; // inactive lanes still join the shuffles
    const int region = cc < Hk * D ? 0 : (cc < 2 * Hk * D ? 1 : 2); // q, k, v
    float w[V][4];
#pragma unroll
    for (int i = 0; i < V; ++i) {
        float4 wv = __ldg(reinterpret_cast<const float4 *>(conv_w) + (cc + i));
        w[i][0] = wv.x; w[i][1] = wv.y; w[i][2] = wv.z; w[i][3] = wv.w;
    }
    const int64_t t0 = (int64_t)blockIdx.x * kConvTokens;
    // all source rows of the block's tokens first (rows t0 - 3 .. t0 + 7; rows
    // outside [0, N) read as zero and feed no output), so that their loads overlap
    Vec16<T> rows[kConvTokens + 3];
#pragma unroll
    for (int k = 0; k < kConvTokens + 3; ++k) {
        const int64_t src = t0 - 3 + k;
        rows[k] = (src >= 0 && src < N) ? ld16_nc(qkv + src * C + cc) : zero16<T>();
    }
    int n = seq_of_token(cu, batch, t0 < N ? t0 : N - 1);
    int64_t start = __ldg(cu + n), next = __ldg(cu + n + 1);
    const int64_t tend = t0 + kConvTokens < N ? t0 + kConvTokens : N;
    // q and k leave L2-normalised (the warp reduces only if some lane holds q
    // or k), v as is; all in float32 so that no rounding is added before the
    // recurrence, except that v, when only the tensor-core path reads it, is
    // rounded to its tf32 operand here
    const bool norm_warp = __any_sync(0xffffffffu, region < 2);
    auto emit = [&](int64_t t, float (&acc)[V]) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            acc[i] = siluf_(acc[i]);
            ss = fmaf(acc[i], acc[i], ss);
        }
        if (norm_warp)
            ss = group_sum<LANES>(ss);
        if (!active)
            return;
        const float f = region == 2 ? 1.0f : rsqrtf(ss + l2_eps) * (region == 0 ? q_scale : 1.0f);
        if (region == 2 && round_v) {
#pragma unroll
            for (int i = 0; i < V; ++i) {
                uint32_t r;
                asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(acc[i]));
                acc[i] = __uint_as_float(r);
            }
        }
        float *dst = region < 2 ? qk_out + t * (2 * Hk * D) + cc
                                : v_out + t * ((int64_t)Hv * D) + (cc - 2 * Hk * D);
#pragma unroll
        for (int i = 0; i < V; i += 4)
            *reinterpret_cast<float4 *>(dst + i) =
                make_float4(acc[i] * f, acc[i + 1] * f, acc[i + 2] * f, acc[i + 3] * f);
    };
    if (start <= t0 - 3 && next >= tend) {
        // one sequence covers every tap of every token of the block (the usual case)
#pragma unroll
        for (int tt = 0; tt < kConvTokens; ++tt) {
            if (t0 + tt >= N)
                break; // uniform over the block
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
        if (t >= N)
            break; // uniform over the block
        while (t >= next && n + 1 < batch) { // t starts a new sequence (after any empty ones)
            ++n;
            start = next;
            next = __ldg(cu + n + 1);
        }
        const int64_t st = start > t ? t : (start < 0 ? 0 : start); // malformed cu_seqlens stay in bounds
        float acc[V];
#pragma unroll
        for (int i = 0; i < V; ++i)
            acc[i] = 0.f;
#pragma unroll
        for (int tap = 0; tap < 4; ++tap) {
            const int64_t src = t - 3 + tap;
            Vec16<T> x;
            if (src >= st)
                x = ld16_nc(qkv + src * C + cc); // rows[] would need a dynamic index here
            else if (init_conv != nullptr)
                x = ld16_nc(init_conv + ((int64_t)n * 3 + (3 + (src - st))) * C + cc);
            else
                x = zero16<T>();
#pragma unroll
            for (int i = 0; i < V; ++i)
                acc[i] = fmaf(w[i][tap], x.get(i), acc[i]);
        }
        emit(t, acc);
    }
}

// final_conv[n] = the last 3 pre-conv rows of [init_conv[n]; sequence n].
// Each thread reads all three source rows of its channels before writing, so
// final_conv may alias init_conv.
template <typename T>
__global__ void final_conv_kernel(const T *__restrict__ qkv, const int32_t *__restrict__ cu,
                                  int batch, int64_t N, const T *init_conv, T *final_conv, int C) {
    constexpr int V = Vec16<T>::N;
    const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * V;
    const int n = blockIdx.y;
    if (c0 >= C || n >= batch)
        return;
    int64_t start, end;
    seq_bounds(cu, n, N, start, end);
    Vec16<T> r[3];
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const int64_t src = end - 3 + i;
        if (src >= start)
            r[i] = ld16_nc(qkv + src * C + c0);
        else if (init_conv != nullptr)
            r[i] = ld16(init_conv + ((int64_t)n * 3 + (3 + (src - start))) * C + c0);
        else
            r[i] = zero16<T>();
    }
#pragma unroll
    for (int i = 0; i < 3; ++i)
        st16(final_conv + ((int64_t)n * 3 + i) * C + c0, r[i]);
}

template <typename T, int D>
cudaError_t launch_conv_prep_t(const PrefillArgs &p, cudaStream_t s) {
    constexpr int V = Vec16<T>::N;
    const int C = (2 * p.Hk + p.Hv) * D;
    dim3 grid((unsigned)((p.N + kConvTokens - 1) / kConvTokens),
              (C / V + kConvThreads - 1) / kConvThreads);
    conv_prep_kernel<T, D><<<grid, kConvThreads, 0, s>>>(
        (const T *)p.qkv, p.cu, p.batch, p.N, (const T *)p.init_conv, p.conv_w, p.Hk, p.Hv,
        p.l2_eps, p.q_scale, (float *)p.ws_qk, (float *)p.ws_v, p.ws_err, p.chunked);
    return cudaGetLastError();
}

template <typename T> cudaError_t launch_final_conv_t(const PrefillArgs &p, cudaStream_t s) {
    constexpr int V = Vec16<T>::N;
    const int C = (2 * p.Hk + p.Hv) * p.D;
    dim3 grid((C / V + 255) / 256, p.batch);
    final_conv_kernel<T><<<grid, 256, 0, s>>>((const T *)p.qkv, p.cu, p.batch, p.N,
                                              (const T *)p.init_conv, (T *)p.final_conv, C);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_conv_prep(const PrefillArgs &p, cudaStream_t s) {
    if (p.N == 0)
        return cudaSuccess;
    if (p.bf16)
        return p.D == 128 ? launch_conv_prep_t<__nv_bfloat16, 128>(p, s)
                          : launch_conv_prep_t<__nv_bfloat16, 32>(p, s);
    return p.D == 128 ? launch_conv_prep_t<float, 128>(p, s) : launch_conv_prep_t<float, 32>(p, s);
}

cudaError_t launch_final_conv(const PrefillArgs &p, cudaStream_t s) {
    if (p.final_conv == nullptr || p.batch == 0)
        return cudaSuccess;
    return p.bf16 ? launch_final_conv_t<__nv_bfloat16>(p, s) : launch_final_conv_t<float>(p, s);
}

} // namespace gdn
