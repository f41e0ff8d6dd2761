// gdn_kda.cu -- Kimi Delta Attention (KDA): the delta rule with a decay per key
// channel ("Inkling vs Kimi K3", component table, linear-attention row: 96
// heads of dimension 128, short conv (kernel 4) + SiLU on q, k and v,
// L2-normalised q and k, per-channel log-decay g = -5 sigmoid(exp(A) z)), and
// its output gate (output-gate row: the head-wise RMSNorm of the recurrent
// output times a full-rank channel-wise sigmoid gate).
//
// Per head and token, with alpha = exp(g) in R^{d_k} and D = Diag(alpha):
//     S_t = S_{t-1} D (I - beta k k^T) + beta v k^T,   o_t = S_t q_t,
//     y_t = o_t / rms(o_t) * w * sigmoid(gate_t),
// which, one state row s (value channel) at a time, is
//     s <- s * alpha;  u = beta (v - s . k);  s <- s + u k;  o = s . q.
// Each head has its own q and k (no sharing).  Both kernels run the update on
// CUDA cores in FP32: the token-serial prefill (one CTA per (head, sequence);
// the conv, SiLU and L2 norm come from the shared front kernel) and the
// one-token decode (one CTA per (sequence, head), conv from the cache).
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

constexpr int kTB = 32; // tokens staged per batch

template <int D> struct KdaSmem {
    float k[kTB][D];
    float q[kTB][D];
    float v[kTB][D];
    float al[kTB][D]; // per-channel decay factors
    float o[kTB][D];
    float beta[kTB];
};

// -5 sigmoid(e^A z): the bounded per-channel log-decay
__device__ __forceinline__ float kda_log_decay(float eA, float z) { return -5.0f * sigmoidf_(eA * z); }

// Thread (row v, part p) keeps D/4 entries of row v of the FP32 state (columns
// 16 i + 4 p + e).
template <typename T, int D>
__global__ void __launch_bounds__(4 * D)
kda_prefill_kernel(PrefillArgs p) {
    constexpr int NT = 4 * D;
    constexpr int NI = D / 16;
    extern __shared__ __align__(16) unsigned char kda_smem_raw[];
    KdaSmem<D> &sm = *reinterpret_cast<KdaSmem<D> *>(kda_smem_raw);
    const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x;
    const int row = tid >> 2, part = tid & 3;
    int64_t start, end;
    seq_bounds(p.cu, n, p.N, start, end);
    const int64_t len = end - start;
    const float *qk = (const float *)p.ws_qk;
    const float *vv = (const float *)p.ws_v;
    const int QK = 2 * p.Hk * D;
    const int64_t HD = (int64_t)p.Hv * D;
    float s[NI][4];
    const size_t sbase = (((size_t)n * p.Hv + h) * D + row) * D;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p.init_state != nullptr)
            x = *reinterpret_cast<const float4 *>(p.init_state + sbase + 16 * i + 4 * part);
        s[i][0] = x.x; s[i][1] = x.y; s[i][2] = x.z; s[i][3] = x.w;
    }
    const float eA = expf(__ldg(p.A_log + h));
    for (int64_t b0 = 0; b0 < len; b0 += kTB) {
        const int nb = (len - b0) < kTB ? (int)(len - b0) : kTB;
        for (int e = tid; e < kTB * (D / 4); e += NT) {
            const int tk = e / (D / 4), c = (e % (D / 4)) * 4;
            if (tk < nb) {
                const int64_t t = start + b0 + tk;
                *reinterpret_cast<float4 *>(&sm.q[tk][c]) =
                    __ldg(reinterpret_cast<const float4 *>(qk + t * QK + h * D + c));
                *reinterpret_cast<float4 *>(&sm.k[tk][c]) =
                    __ldg(reinterpret_cast<const float4 *>(qk + t * QK + p.Hk * D + h * D + c));
                *reinterpret_cast<float4 *>(&sm.v[tk][c]) =
                    __ldg(reinterpret_cast<const float4 *>(vv + t * HD + (int64_t)h * D + c));
                const T *zp = (const T *)p.kda_zdec + t * HD + (int64_t)h * D + c;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    sm.al[tk][c + i] = expf(kda_log_decay(eA, to_f(zp[i])));
            }
        }
        if (tid < nb)
            sm.beta[tid] = sigmoidf_(to_f(((const T *)p.b)[(start + b0 + tid) * p.Hv + h]));
        __syncthreads();
        for (int tk = 0; tk < nb; ++tk) {
            const float beta = sm.beta[tk];
            const float4 *k4 = reinterpret_cast<const float4 *>(sm.k[tk]);
            const float4 *q4 = reinterpret_cast<const float4 *>(sm.q[tk]);
            const float4 *a4 = reinterpret_cast<const float4 *>(sm.al[tk]);
            float kr[NI][4];
            float pk0 = 0.f, pk1 = 0.f;
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                const float4 kk = k4[4 * i + part], aa = a4[4 * i + part];
                kr[i][0] = kk.x; kr[i][1] = kk.y; kr[i][2] = kk.z; kr[i][3] = kk.w;
                s[i][0] *= aa.x; s[i][1] *= aa.y; s[i][2] *= aa.z; s[i][3] *= aa.w;
                pk0 = fmaf(s[i][0], kk.x, pk0);
                pk1 = fmaf(s[i][1], kk.y, pk1);
                pk0 = fmaf(s[i][2], kk.z, pk0);
                pk1 = fmaf(s[i][3], kk.w, pk1);
            }
            float pk = pk0 + pk1;
            pk += __shfl_xor_sync(0xffffffffu, pk, 1);
            pk += __shfl_xor_sync(0xffffffffu, pk, 2);
            const float u = beta * (sm.v[tk][row] - pk);
            float po0 = 0.f, po1 = 0.f;
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                const float4 qq = q4[4 * i + part];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    s[i][e] = fmaf(u, kr[i][e], s[i][e]);
                po0 = fmaf(s[i][0], qq.x, po0);
                po1 = fmaf(s[i][1], qq.y, po1);
                po0 = fmaf(s[i][2], qq.z, po0);
                po1 = fmaf(s[i][3], qq.w, po1);
            }
            float po = po0 + po1;
            po += __shfl_xor_sync(0xffffffffu, po, 1);
            po += __shfl_xor_sync(0xffffffffu, po, 2);
            if (part == 0)
                sm.o[tk][row] = po;
        }
        __syncthreads();
        // RMSNorm of each token's output times w sigmoid(gate), one warp per token
        const int warp = tid >> 5, lane = tid & 31;
        constexpr int PER = D / 32;
        for (int tk = warp; tk < nb; tk += NT / 32) {
            const int64_t t = start + b0 + tk;
            float ov[PER];
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < PER; ++e) {
                ov[e] = sm.o[tk][lane * PER + e];
                ss = fmaf(ov[e], ov[e], ss);
            }
            ss = group_sum<32>(ss);
            const float r = rsqrtf(ss / (float)D + p.rms_eps);
            const int64_t base = t * HD + (int64_t)h * D + lane * PER;
#pragma unroll
            for (int e = 0; e < PER; ++e) {
                const float gt = to_f(((const T *)p.z)[base + e]);
                ((T *)p.y)[base + e] = from_f<T>(ov[e] * r * __ldg(p.norm_w + lane * PER + e) * sigmoidf_(gt));
                if (p.o_raw != nullptr)
                    p.o_raw[base + e] = ov[e];
            }
        }
        __syncthreads();
    }
    if (p.final_state != nullptr) {
#pragma unroll
        for (int i = 0; i < NI; ++i)
            *reinterpret_cast<float4 *>(p.final_state + sbase + 16 * i + 4 * part) =
                make_float4(s[i][0], s[i][1], s[i][2], s[i][3]);
    }
}

// One token per sequence: CTA (head j, sequence n) convolves its q, k, v channels
// from the conv cache (shifted in place), normalises q and k, forms the
// per-channel decay, streams the head's state once (a lane holds 4 columns of
// a row; the state is read and written once), then the gated RMSNorm.
template <typename T, int D>
__global__ void __launch_bounds__(256)
kda_decode_kernel(DecodeArgs p) {
    constexpr int V = Vec16<T>::N;
    constexpr int L = D / 4, RPI = 32 / L, NW = 8;
    __shared__ __align__(16) float qs[D], ks[D], vs[D], as[D], os[D];
    __shared__ float red[4];
    const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.Hv;
    const int C = 3 * H * D;
    const T *x = (const T *)p.qkv + (size_t)n * C;
    T *cache = (T *)p.conv_cache + (size_t)n * 3 * C;
    const float eA = expf(__ldg(p.A_log + h));
    for (int gi = tid; gi < 3 * (D / V); gi += 256) {
        const int part = gi / (D / V), off = (gi % (D / V)) * V;
        const int c = part * H * D + h * D + off;
        float *dst = (part == 0 ? qs : (part == 1 ? ks : vs)) + off;
        Vec16<T> r0 = ld16(cache + c), r1 = ld16(cache + C + c), r2 = ld16(cache + 2 * C + c);
        Vec16<T> r3 = ld16_nc(x + c);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const float4 w = __ldg(reinterpret_cast<const float4 *>(p.conv_w) + (c + i));
            float acc = w.x * r0.get(i);
            acc = fmaf(w.y, r1.get(i), acc);
            acc = fmaf(w.z, r2.get(i), acc);
            acc = fmaf(w.w, r3.get(i), acc);
            dst[i] = siluf_(acc);
        }
        st16(cache + c, r1);
        st16(cache + C + c, r2);
        st16(cache + 2 * C + c, r3);
    }
    for (int c = tid; c < D; c += 256)
        as[c] = expf(kda_log_decay(eA, to_f(((const T *)p.kda_zdec)[((size_t)n * H + h) * D + c])));
    __syncthreads();
    if (warp < 3) { // |q|^2, |k|^2, k.q before normalisation
        float acc = 0.f;
        for (int c = lane; c < D; c += 32) {
            const float a0 = warp == 1 ? ks[c] : qs[c];
            const float a1 = warp == 0 ? qs[c] : ks[c];
            acc = fmaf(a0, a1, acc);
        }
        acc = group_sum<32>(acc);
        if (lane == 0)
            red[warp] = acc;
    }
    __syncthreads();
    const float sq = rsqrtf(red[0] + p.l2_eps) * p.q_scale, sk = rsqrtf(red[1] + p.l2_eps);
    const float kq = red[2] * sq * sk;
    const float beta = sigmoidf_(to_f(((const T *)p.b)[(size_t)n * H + h]));
    const int lr = lane / L, c4 = (lane % L) * 4;
    float ka[4], qa[4], kr[4], al[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        al[e] = as[c4 + e];
        kr[e] = ks[c4 + e] * sk;
        ka[e] = kr[e] * al[e];          // (S D) k = S (D k)
        qa[e] = qs[c4 + e] * sq * al[e]; // (S D) q
    }
    float *Sg = p.state + ((size_t)n * H + h) * D * D;
    for (int r = warp * RPI + lr; r < D; r += NW * RPI) {
        const float4 sv = __ldcs(reinterpret_cast<const float4 *>(Sg + (size_t)r * D + c4));
        float pk = sv.x * ka[0] + sv.y * ka[1] + sv.z * ka[2] + sv.w * ka[3];
        float pq = sv.x * qa[0] + sv.y * qa[1] + sv.z * qa[2] + sv.w * qa[3];
#pragma unroll
        for (int o = L / 2; o > 0; o >>= 1) {
            pk += __shfl_xor_sync(0xffffffffu, pk, o);
            pq += __shfl_xor_sync(0xffffffffu, pq, o);
        }
        const float u = beta * (vs[r] - pk);
        float4 nv;
        nv.x = fmaf(u, kr[0], al[0] * sv.x);
        nv.y = fmaf(u, kr[1], al[1] * sv.y);
        nv.z = fmaf(u, kr[2], al[2] * sv.z);
        nv.w = fmaf(u, kr[3], al[3] * sv.w);
        __stcs(reinterpret_cast<float4 *>(Sg + (size_t)r * D + c4), nv);
        if ((lane % L) == 0)
            os[r] = pq + u * kq; // o = (S D) q + u (k . q)
    }
    __syncthreads();
    if (warp == 0) {
        constexpr int PER = D / 32;
        float ov[PER], ss = 0.f;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            ov[e] = os[lane * PER + e];
            ss = fmaf(ov[e], ov[e], ss);
        }
        ss = group_sum<32>(ss);
        const float rr = rsqrtf(ss / (float)D + p.rms_eps);
        const size_t yb = ((size_t)n * H + h) * D + lane * PER;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const float gt = to_f(((const T *)p.z)[yb + e]);
            ((T *)p.y)[yb + e] = from_f<T>(ov[e] * rr * __ldg(p.norm_w + lane * PER + e) * sigmoidf_(gt));
        }
    }
}

template <typename T, int D> cudaError_t launch_prefill_t(const PrefillArgs &p, cudaStream_t s) {
    const size_t smem = sizeof(KdaSmem<D>);
    cudaError_t e = cudaFuncSetAttribute(kda_prefill_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    dim3 grid(p.Hv, p.batch);
    kda_prefill_kernel<T, D><<<grid, 4 * D, smem, s>>>(p);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_kda_prefill(const PrefillArgs &p, cudaStream_t s) {
    if (p.batch == 0)
        return cudaSuccess;
    if (p.bf16)
        return p.D == 128 ? launch_prefill_t<__nv_bfloat16, 128>(p, s) : launch_prefill_t<__nv_bfloat16, 32>(p, s);
    return p.D == 128 ? launch_prefill_t<float, 128>(p, s) : launch_prefill_t<float, 32>(p, s);
}

cudaError_t launch_kda_decode(const DecodeArgs &p, cudaStream_t s) {
    if (p.batch == 0)
        return cudaSuccess;
    dim3 grid(p.Hv, p.batch);
    if (p.bf16) {
        if (p.D == 128)
            kda_decode_kernel<__nv_bfloat16, 128><<<grid, 256, 0, s>>>(p);
        else
            kda_decode_kernel<__nv_bfloat16, 32><<<grid, 256, 0, s>>>(p);
    } else {
        if (p.D == 128)
            kda_decode_kernel<float, 128><<<grid, 256, 0, s>>>(p);
        else
            kda_decode_kernel<float, 32><<<grid, 256, 0, s>>>(p);
    }
    return cudaGetLastError();
}

} // namespace gdn
