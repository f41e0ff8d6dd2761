// gdn_decode.cu -- one new token per sequence against resident FP32 states.
//
// One CTA per (sequence, q/k head group): it convolves the group's q, k and
// the G value heads' v channels from the conv cache plus the new row (kernel-4
// causal conv + SiLU), shifts that part of the conv cache in place,
// L2-normalises q and k, forms the gates, then streams the G states of the
// group (G x 64 KiB at d = 128) once through registers:
//     p = S k, r = S q (one read),  u = beta (v - alpha p),
//     S <- alpha S + u k^T (one write),  o = alpha r + u (k . q),
// which is the gated delta rule S_t = alpha S_{t-1}(I - beta k k^T) + beta v k^T,
// o_t = S_t q_t for a single token (Gated DeltaNet row of the component table
// on "Qwen3.8-2.4T-A95B vs Inkling"), followed by the per-head RMSNorm gated
// by SiLU(z) (output-gate row of the same table).  The state traffic is the
// whole cost: the kernel is HBM-bound by design.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kUnroll = 4; // rows in flight per lane group

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads)
decode_kernel(DecodeArgs p) {
    constexpr int V = Vec16<T>::N;
    constexpr int L = D / 4;      // lanes per state row (float4 each)
    constexpr int RPI = 32 / L;   // rows per warp per step
    extern __shared__ __align__(16) float dsm[];
    const int G = p.G;
    float *qs = dsm;              // [D]
    float *ks = qs + D;           // [D]
    float *vs = ks + D;           // [G*D]
    float *os = vs + G * D;       // [G*D]
    float *gal = os + G * D;      // [G] alpha
    float *gbe = gal + G;         // [G] beta
    float *red = gbe + G;         // [4]

    const int j = blockIdx.x;     // q/k head
    const int n = blockIdx.y;     // sequence
    const int tid = threadIdx.x;
    const int C = (2 * p.Hk + p.Hv) * D;
    const T *x = (const T *)p.qkv + (size_t)n * C;
    T *cache = (T *)p.conv_cache + (size_t)n * 3 * C;

    // ---- phase 1: conv + SiLU of this group's channels, cache shift, gates
    const int groups = (2 + G) * (D / V);
    for (int gi = tid; gi < groups; gi += kDecThreads) {
        int c, off;
        float *dst;
        if (gi < D / V) {
            off = gi * V; c = j * D + off; dst = qs + off;
        } else if (gi < 2 * (D / V)) {
            off = (gi - D / V) * V; c = p.Hk * D + j * D + off; dst = ks + off;
        } else {
            off = (gi - 2 * (D / V)) * V; c = 2 * p.Hk * D + j * G * D + off; dst = vs + off;
        }
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
        // only this thread reads or writes these cache channels
        st16(cache + c, r1);
        st16(cache + C + c, r2);
        st16(cache + 2 * C + c, r3);
    }
    if (tid < G) {
        const int h = j * G + tid;
        const float g = -expf(__ldg(p.A_log + h)) *
                        softplusf_(to_f(((const T *)p.a)[(size_t)n * p.Hv + h]) + __ldg(p.dt_bias + h));
        gal[tid] = expf(g);
        gbe[tid] = sigmoidf_(to_f(((const T *)p.b)[(size_t)n * p.Hv + h]));
    }
    __syncthreads();
    {
        const int warp = tid >> 5, lane = tid & 31;
        if (warp < 3) {
            float acc = 0.f;
            for (int c = lane; c < D; c += 32) {
                const float a0 = warp == 1 ? ks[c] : qs[c];
                const float a1 = warp == 0 ? qs[c] : ks[c];
                acc = fmaf(a0, a1, acc);
            }
            acc = group_sum<32>(acc);
            if (lane == 0)
                red[warp] = acc; // |q|^2, |k|^2, k.q (before normalisation)
        }
    }
    __syncthreads();
    const float sq = rsqrtf(red[0] + p.l2_eps) * p.q_scale;
    const float sk = rsqrtf(red[1] + p.l2_eps);
    const float kq = red[2] * sq * sk;

    // ---- phase 2: stream the G states of the group
    const int warp = tid >> 5, lane = tid & 31;
    const int lr = lane / L;          // row within the warp step
    const int c4 = (lane % L) * 4;    // first column of this lane
    float kr[4], qr[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        kr[e] = ks[c4 + e] * sk;
        qr[e] = qs[c4 + e] * sq;
    }
    const int R = G * D; // rows of the group
    float *Sg = p.state + ((size_t)n * p.Hv + (size_t)j * G) * D * D;
    for (int base = warp * RPI; base < R; base += kDecWarps * RPI * kUnroll) {
        float4 sv[kUnroll];
#pragma unroll
        for (int uu = 0; uu < kUnroll; ++uu) {
            const int r = base + uu * kDecWarps * RPI + lr;
            sv[uu] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < R)
                sv[uu] = __ldcs(reinterpret_cast<const float4 *>(Sg + (size_t)r * D + c4));
        }
#pragma unroll
        for (int uu = 0; uu < kUnroll; ++uu) {
            const int r = base + uu * kDecWarps * RPI + lr;
            float pk = sv[uu].x * kr[0] + sv[uu].y * kr[1] + sv[uu].z * kr[2] + sv[uu].w * kr[3];
            float pq = sv[uu].x * qr[0] + sv[uu].y * qr[1] + sv[uu].z * qr[2] + sv[uu].w * qr[3];
#pragma unroll
            for (int o = L / 2; o > 0; o >>= 1) {
                pk += __shfl_xor_sync(0xffffffffu, pk, o);
                pq += __shfl_xor_sync(0xffffffffu, pq, o);
            }
            if (r < R) {
                const int hh = r / D;
                const float al = gal[hh], be = gbe[hh];
                const float u = be * (vs[r] - al * pk);
                float4 nv;
                nv.x = fmaf(u, kr[0], al * sv[uu].x);
                nv.y = fmaf(u, kr[1], al * sv[uu].y);
                nv.z = fmaf(u, kr[2], al * sv[uu].z);
                nv.w = fmaf(u, kr[3], al * sv[uu].w);
                __stcs(reinterpret_cast<float4 *>(Sg + (size_t)r * D + c4), nv);
                if ((lane % L) == 0)
                    os[r] = fmaf(al, pq, u * kq);
            }
        }
    }
    __syncthreads();

    // ---- phase 3: gated RMSNorm, one warp per value head
    constexpr int PER = D / 32;
    for (int hh = warp; hh < G; hh += kDecWarps) {
        const int h = j * G + hh;
        float ov[PER];
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            ov[e] = os[hh * D + lane * PER + e];
            ss = fmaf(ov[e], ov[e], ss);
        }
        ss = group_sum<32>(ss);
        const float rr = rsqrtf(ss / (float)D + p.rms_eps);
        const size_t yb = ((size_t)n * p.Hv + h) * D + lane * PER;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const float zz = to_f(((const T *)p.z)[yb + e]);
            ((T *)p.y)[yb + e] =
                from_f<T>(ov[e] * rr * __ldg(p.norm_w + lane * PER + e) * siluf_(zz));
        }
    }
}

template <typename T, int D> cudaError_t launch_t(const DecodeArgs &p, cudaStream_t s) {
    const size_t smem = sizeof(float) * (2 * D + 2 * (size_t)p.G * D + 2 * p.G + 4);
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    dim3 grid(p.Hk, p.batch);
    decode_kernel<T, D><<<grid, kDecThreads, smem, s>>>(p);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_decode(const DecodeArgs &p, cudaStream_t s) {
    if (p.batch == 0)
        return cudaSuccess;
    if (p.bf16)
        return p.D == 128 ? launch_t<__nv_bfloat16, 128>(p, s) : launch_t<__nv_bfloat16, 32>(p, s);
    return p.D == 128 ? launch_t<float, 128>(p, s) : launch_t<float, 32>(p, s);
}

} // namespace gdn
