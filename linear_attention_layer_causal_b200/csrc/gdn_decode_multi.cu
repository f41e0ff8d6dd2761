// gdn_decode_multi.cu -- several new tokens per sequence against resident FP32
// states: plain multi-token decode, and the verify / commit pair that
// speculative decoding with multi-token-prediction drafts needs ("Qwen3.8 2.4T
// A95B", key facts: one extra multi-token-prediction layer used to accelerate
// decoding; raw config field mtp_num_hidden_layers = 1).
//
// The update of one state row (one value channel v of one value head) over
// tokens t = 0 .. k-1 needs only that row and the tokens' q, k, v[v], gates:
//     p = s . k_t,  r = s . q_t,  u = beta_t (v_t - alpha_t p),
//     s <- alpha_t s + u k_t,      o_t[v] = alpha_t r + u (k_t . q_t),
// the gated delta rule S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) +
// beta_t v_t k_t^T, o_t = S_t q_t of the Gated DeltaNet row ("Qwen3.8-2.4T-A95B
// vs Inkling", component table) written per row.  So every row is read from
// HBM once, carried through all k tokens in registers, and written once (or
// not at all): k tokens cost one pass over the state instead of k.
//
// One CTA per (sequence, q/k head group), as in the one-token decode: it
// convolves the group's q, k and v channels for the k tokens from the conv
// cache (kernel-4 causal conv + SiLU), normalises q and k per token, forms
// the gates, streams the G states of the group, and finishes with the gated
// RMSNorm of every (token, value head) (output-gate row of the same table).
// Modes:
//   kMulti  -- all k tokens are taken: state and conv cache advance by k, y out;
//   kVerify -- y for the k tokens, state and conv cache untouched (read only);
//   kCommit -- state and conv cache advance by accepted[n] (0..k) tokens, no y.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

constexpr int kMtThreads = 256; // two CTAs per SM: one streams the state while the other convolves
constexpr int kMtWarps = kMtThreads / 32;
constexpr int kRowUnroll = 2; // rows in flight per lane group

template <typename T, int D, int MODE>
__global__ void __launch_bounds__(kMtThreads)
decode_multi_kernel(DecodeArgs p) {
    constexpr int V = Vec16<T>::N;  // channels per 16-byte vector
    constexpr int LR = D / 16;      // lanes per state row (16 floats each)
    constexpr int RPW = 32 / LR;    // rows per warp per step
    const int K = p.k;
    const int G = p.G;
    const int j = blockIdx.x; // q/k head
    const int n = blockIdx.y; // sequence
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // tokens taken into the state and conv cache
    int m = K;
    if (MODE == kDecodeVerify)
        m = 0;
    else if (MODE == kDecodeCommit) {
        m = __ldg(p.accepted + n);
        m = m < 0 ? 0 : (m > K ? K : m);
        if (m == 0)
            return; // nothing to take: state and cache stay as they are
    }
    const int Kc = MODE == kDecodeCommit ? m : K; // tokens this CTA computes

    // shared memory, sized for K tokens (decode_multi_smem_bytes)
    extern __shared__ __align__(16) float msm[];
    float *qs = msm;                    // [K][D] normalised q
    float *ks = qs + K * D;             // [K][D] normalised k
    float *vs = ks + K * D;             // [K][G*D]
    float *os = vs + (size_t)K * G * D; // [K][G*D] (not in commit mode)
    float *gal = os + (MODE == kDecodeCommit ? 0 : (size_t)K * G * D); // [K][G] alpha
    float *gbe = gal + K * G;           // [K][G] beta
    float *nrm = gbe + K * G;           // [K][3]: |q|^2, |k|^2, k.q (then k.q normalised)

    const int C = (2 * p.Hk + p.Hv) * D;
    const T *x = (const T *)p.qkv + (size_t)n * K * C;
    T *cache = (T *)p.conv_cache + (size_t)n * 3 * C;

    // ---- phase 1: conv + SiLU of this group's channels for the Kc tokens; the
    //      conv cache becomes the last 3 rows of [cache; first m new rows]
    const int groups = (2 + G) * (D / V);
    for (int gi = tid; gi < groups; gi += kMtThreads) {
        int c;
        float *dst;
        int stride;
        if (gi < D / V) {
            const int off = gi * V;
            c = j * D + off; dst = qs + off; stride = D;
        } else if (gi < 2 * (D / V)) {
            const int off = (gi - D / V) * V;
            c = p.Hk * D + j * D + off; dst = ks + off; stride = D;
        } else {
            const int off = (gi - 2 * (D / V)) * V;
            c = 2 * p.Hk * D + j * G * D + off; dst = vs + off; stride = G * D;
        }
        float w[V][4];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const float4 wv = __ldg(reinterpret_cast<const float4 *>(p.conv_w) + (c + i));
            w[i][0] = wv.x; w[i][1] = wv.y; w[i][2] = wv.z; w[i][3] = wv.w;
        }
        // rows of [cache; new rows]: index < 3 is a cache row, else new row index - 3
        auto row = [&](int idx) {
            return idx < 3 ? ld16(cache + (size_t)idx * C + c) : ld16_nc(x + (size_t)(idx - 3) * C + c);
        };
        // the new cache rows m, m + 1, m + 2, read before anything is written
        Vec16<T> nv[3];
        if (MODE != kDecodeVerify) {
#pragma unroll
            for (int i = 0; i < 3; ++i)
                nv[i] = row(m + i);
        }
        // sliding window of four rows over the tokens
        Vec16<T> r0 = row(0), r1 = row(1), r2 = row(2);
#pragma unroll 1
        for (int t = 0; t < Kc; ++t) {
            const Vec16<T> r3 = row(3 + t);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                float acc = w[i][0] * r0.get(i);
                acc = fmaf(w[i][1], r1.get(i), acc);
                acc = fmaf(w[i][2], r2.get(i), acc);
                acc = fmaf(w[i][3], r3.get(i), acc);
                dst[t * stride + i] = siluf_(acc);
            }
            r0 = r1; r1 = r2; r2 = r3;
        }
        if (MODE != kDecodeVerify) {
            // only this thread reads or writes these cache channels
#pragma unroll
            for (int i = 0; i < 3; ++i)
                st16(cache + (size_t)i * C + c, nv[i]);
        }
    }
    for (int e = tid; e < Kc * G; e += kMtThreads) {
        const int t = e / G, hh = e % G, h = j * G + hh;
        const size_t ab = ((size_t)n * K + t) * p.Hv + h;
        const float g = -expf(__ldg(p.A_log + h)) *
                        softplusf_(to_f(((const T *)p.a)[ab]) + __ldg(p.dt_bias + h));
        gal[t * G + hh] = expf(g);
        gbe[t * G + hh] = sigmoidf_(to_f(((const T *)p.b)[ab]));
    }
    __syncthreads();
    // |q_t|^2, |k_t|^2, k_t . q_t: one warp per (token, product)
    for (int e = warp; e < 3 * Kc; e += kMtWarps) {
        const int t = e / 3, which = e % 3;
        const float *a0 = which == 1 ? ks + t * D : qs + t * D;
        const float *a1 = which == 0 ? qs + t * D : ks + t * D;
        float acc = 0.f;
        for (int c = lane; c < D; c += 32)
            acc = fmaf(a0[c], a1[c], acc);
        acc = group_sum<32>(acc);
        if (lane == 0)
            nrm[3 * t + which] = acc;
    }
    __syncthreads();
    // normalise q and k in place; kq becomes k_t . q_t of the normalised vectors
    for (int e = tid; e < Kc * D; e += kMtThreads) {
        const int t = e / D;
        const float sq = rsqrtf(nrm[3 * t] + p.l2_eps) * p.q_scale;
        const float sk = rsqrtf(nrm[3 * t + 1] + p.l2_eps);
        qs[e] *= sq;
        ks[e] *= sk;
    }
    __syncthreads();
    if (tid < Kc)
        nrm[3 * tid + 2] *= rsqrtf(nrm[3 * tid] + p.l2_eps) * p.q_scale *
                            rsqrtf(nrm[3 * tid + 1] + p.l2_eps);
    __syncthreads();

    // ---- phase 2: every row of the group's G states through the Kc tokens
    // a row's LR lanes interleave its float4s: lane l8 holds float4s l8, l8 + LR,
    // l8 + 2 LR, l8 + 3 LR, so that the lanes read k and q from shared memory
    // without bank conflicts and each load of the state is contiguous
    const int lr = lane / LR;  // row within the warp step
    const int l8 = lane % LR;  // lane within the row
    const int R = G * D;
    float *Sg = p.state + ((size_t)n * p.Hv + (size_t)j * G) * D * D;
    for (int base = warp * RPW; base < R; base += kMtWarps * RPW * kRowUnroll) {
        float s[kRowUnroll][16];
#pragma unroll
        for (int uu = 0; uu < kRowUnroll; ++uu) {
            const int r = base + uu * kMtWarps * RPW + lr;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float4 x4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (r < R) {
                    const float4 *src = reinterpret_cast<const float4 *>(Sg + (size_t)r * D) + l8 + LR * i;
                    x4 = MODE == kDecodeVerify ? __ldg(src) : __ldcs(src);
                }
                s[uu][4 * i] = x4.x; s[uu][4 * i + 1] = x4.y;
                s[uu][4 * i + 2] = x4.z; s[uu][4 * i + 3] = x4.w;
            }
        }
#pragma unroll 1
        for (int t = 0; t < Kc; ++t) {
            const float4 *k4 = reinterpret_cast<const float4 *>(ks + t * D) + l8;
            const float4 *q4 = reinterpret_cast<const float4 *>(qs + t * D) + l8;
            const float kq = nrm[3 * t + 2];
#pragma unroll
            for (int uu = 0; uu < kRowUnroll; ++uu) {
                const int r = base + uu * kMtWarps * RPW + lr;
                float pk = 0.f, pq = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 kv = k4[LR * i];
                    pk = fmaf(s[uu][4 * i], kv.x, pk);
                    pk = fmaf(s[uu][4 * i + 1], kv.y, pk);
                    pk = fmaf(s[uu][4 * i + 2], kv.z, pk);
                    pk = fmaf(s[uu][4 * i + 3], kv.w, pk);
                    if (MODE != kDecodeCommit) {
                        const float4 qv = q4[LR * i];
                        pq = fmaf(s[uu][4 * i], qv.x, pq);
                        pq = fmaf(s[uu][4 * i + 1], qv.y, pq);
                        pq = fmaf(s[uu][4 * i + 2], qv.z, pq);
                        pq = fmaf(s[uu][4 * i + 3], qv.w, pq);
                    }
                }
#pragma unroll
                for (int o = LR / 2; o > 0; o >>= 1) {
                    pk += __shfl_xor_sync(0xffffffffu, pk, o);
                    if (MODE != kDecodeCommit)
                        pq += __shfl_xor_sync(0xffffffffu, pq, o);
                }
                const int hh = (r < R ? r : 0) / D;
                const float al = gal[t * G + hh], be = gbe[t * G + hh];
                const float u = be * ((r < R ? vs[t * R + r] : 0.f) - al * pk);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 kv = k4[LR * i];
                    s[uu][4 * i] = fmaf(u, kv.x, al * s[uu][4 * i]);
                    s[uu][4 * i + 1] = fmaf(u, kv.y, al * s[uu][4 * i + 1]);
                    s[uu][4 * i + 2] = fmaf(u, kv.z, al * s[uu][4 * i + 2]);
                    s[uu][4 * i + 3] = fmaf(u, kv.w, al * s[uu][4 * i + 3]);
                }
                if (MODE != kDecodeCommit && r < R && (lane % LR) == 0)
                    os[t * R + r] = fmaf(al, pq, u * kq);
            }
        }
        if (MODE != kDecodeVerify) {
#pragma unroll
            for (int uu = 0; uu < kRowUnroll; ++uu) {
                const int r = base + uu * kMtWarps * RPW + lr;
                if (r < R) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        __stcs(reinterpret_cast<float4 *>(Sg + (size_t)r * D) + l8 + LR * i,
                               make_float4(s[uu][4 * i], s[uu][4 * i + 1], s[uu][4 * i + 2],
                                           s[uu][4 * i + 3]));
                }
            }
        }
    }
    if (MODE == kDecodeCommit)
        return;
    __syncthreads();

    // ---- phase 3: gated RMSNorm, one warp per (token, value head)
    constexpr int PER = D / 32;
    for (int e = warp; e < Kc * G; e += kMtWarps) {
        const int t = e / G, hh = e % G, h = j * G + hh;
        float ov[PER];
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            ov[i] = os[t * R + hh * D + lane * PER + i];
            ss = fmaf(ov[i], ov[i], ss);
        }
        ss = group_sum<32>(ss);
        const float rr = rsqrtf(ss / (float)D + p.rms_eps);
        const size_t yb = (((size_t)n * K + t) * p.Hv + h) * D + lane * PER;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const float zz = to_f(((const T *)p.z)[yb + i]);
            ((T *)p.y)[yb + i] = from_f<T>(ov[i] * rr * __ldg(p.norm_w + lane * PER + i) * siluf_(zz));
        }
    }
}

template <typename T, int D, int MODE> cudaError_t launch_t(const DecodeArgs &p, cudaStream_t s) {
    const size_t smem = decode_multi_smem_bytes(p.G, D, p.k, MODE);
    cudaError_t e = cudaFuncSetAttribute(decode_multi_kernel<T, D, MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    dim3 grid(p.Hk, p.batch);
    decode_multi_kernel<T, D, MODE><<<grid, kMtThreads, smem, s>>>(p);
    return cudaGetLastError();
}

template <int MODE> cudaError_t launch_mode(const DecodeArgs &p, cudaStream_t s) {
    if (p.bf16)
        return p.D == 128 ? launch_t<__nv_bfloat16, 128, MODE>(p, s)
                          : launch_t<__nv_bfloat16, 32, MODE>(p, s);
    return p.D == 128 ? launch_t<float, 128, MODE>(p, s) : launch_t<float, 32, MODE>(p, s);
}

} // namespace

size_t decode_multi_smem_bytes(int G, int D, int k, int mode) {
    const size_t K = (size_t)k;
    size_t f = 2 * K * D + K * (size_t)G * D + 2 * K * G + 3 * K;
    if (mode != kDecodeCommit)
        f += K * (size_t)G * D;
    return f * sizeof(float);
}

cudaError_t launch_decode_multi(const DecodeArgs &p, int mode, cudaStream_t s) {
    if (p.batch == 0)
        return cudaSuccess;
    switch (mode) {
    case kDecodeMulti: return launch_mode<kDecodeMulti>(p, s);
    case kDecodeVerify: return launch_mode<kDecodeVerify>(p, s);
    default: return launch_mode<kDecodeCommit>(p, s);
    }
}

} // namespace gdn
