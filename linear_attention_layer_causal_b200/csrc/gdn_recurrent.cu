// gdn_recurrent.cu -- token-serial gated delta rule on CUDA cores, with the
// gates computed on the fly and the gated RMSNorm fused into the output store.
//
// One CTA per (sequence, value head).  Thread (row v, part p) keeps D/4
// entries of row v of the FP32 state in registers; per token it performs
//     S <- alpha S;  p = S k;  u = beta (v - p);  S <- S + u k^T;  o = S q,
// the gated delta rule S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
// o_t = S_t q_t on a d_v x d_k FP32 state (Gated DeltaNet row of the component
// table on "Qwen3.8-2.4T-A95B vs Inkling"; mamba_ssm_dtype float32 in the raw
// config fields of "Qwen3.8 2.4T A95B").  The gates are
// alpha = exp(-exp(A_log) softplus(a + dt_bias)) and beta = sigmoid(b) (same
// row), and y = RMSNorm(o) * w * SiLU(z) (output-gate row of the same table).
//
// This kernel serves every head size (it is the path for head_dim 32) and is
// the plain reference point for the tensor-core chunked kernel.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

constexpr int kTB = 32; // tokens staged per batch

template <int D> struct RecSmem {
    float k[kTB][D];
    float q[kTB][D];
    float v[kTB][D];
    float o[kTB][D];
    float alpha[kTB];
    float beta[kTB];
};

template <typename T, int D>
__global__ void __launch_bounds__(4 * D)
recurrent_prefill_kernel(PrefillArgs p) {
    constexpr int NT = 4 * D;
    constexpr int NI = D / 16; // float4 groups per thread
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RecSmem<D> &sm = *reinterpret_cast<RecSmem<D> *>(smem_raw);

    const int h = blockIdx.x;
    const int n = blockIdx.y;
    const int j = h / p.G;
    const int tid = threadIdx.x;
    const int row = tid >> 2;
    const int part = tid & 3;
    int64_t start, end;
    seq_bounds(p.cu, n, p.N, start, end);
    const int64_t len = end - start;

    const float *qk = (const float *)p.ws_qk;
    const float *vv = (const float *)p.ws_v;
    const T *za = (const T *)p.z;
    const T *ga = (const T *)p.a;
    const T *gb = (const T *)p.b;
    T *yo = (T *)p.y;
    const int QK = 2 * p.Hk * D;
    const int64_t HD = (int64_t)p.Hv * D;

    // state row `row`, columns 16 i + 4 part + (0..3)
    float s[NI][4];
    const size_t sbase = (((size_t)n * p.Hv + h) * D + row) * D;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p.init_state != nullptr)
            x = *reinterpret_cast<const float4 *>(p.init_state + sbase + 16 * i + 4 * part);
        s[i][0] = x.x; s[i][1] = x.y; s[i][2] = x.z; s[i][3] = x.w;
    }
    const float negA = -expf(__ldg(p.A_log + h));
    const float dtb = __ldg(p.dt_bias + h);

    for (int64_t b0 = 0; b0 < len; b0 += kTB) {
        const int nb = (len - b0) < kTB ? (int)(len - b0) : kTB;
        // ---- stage k, q, v of this batch as float, and the gates
        for (int e = tid; e < kTB * (D / 4); e += NT) {
            const int tk = e / (D / 4);
            const int c = (e % (D / 4)) * 4;
            if (tk < nb) {
                const int64_t t = start + b0 + tk;
                *reinterpret_cast<float4 *>(&sm.q[tk][c]) =
                    __ldg(reinterpret_cast<const float4 *>(qk + t * QK + j * D + c));
                *reinterpret_cast<float4 *>(&sm.k[tk][c]) =
                    __ldg(reinterpret_cast<const float4 *>(qk + t * QK + p.Hk * D + j * D + c));
                *reinterpret_cast<float4 *>(&sm.v[tk][c]) =
                    __ldg(reinterpret_cast<const float4 *>(vv + t * HD + (int64_t)h * D + c));
            }
        }
        if (tid < nb) {
            const int64_t t = start + b0 + tid;
            const float g = negA * softplusf_(to_f(ga[t * p.Hv + h]) + dtb);
            sm.alpha[tid] = expf(g);
            sm.beta[tid] = sigmoidf_(to_f(gb[t * p.Hv + h]));
        }
        __syncthreads();

        // ---- the serial recurrence over the batch
        for (int tk = 0; tk < nb; ++tk) {
            const float alpha = sm.alpha[tk];
            const float beta = sm.beta[tk];
            const float4 *k4 = reinterpret_cast<const float4 *>(sm.k[tk]);
            const float4 *q4 = reinterpret_cast<const float4 *>(sm.q[tk]);
            float kr[NI][4];
            float pk0 = 0.f, pk1 = 0.f;
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                float4 kk = k4[4 * i + part];
                kr[i][0] = kk.x; kr[i][1] = kk.y; kr[i][2] = kk.z; kr[i][3] = kk.w;
                pk0 = fmaf(s[i][0], kk.x, pk0);
                pk1 = fmaf(s[i][1], kk.y, pk1);
                pk0 = fmaf(s[i][2], kk.z, pk0);
                pk1 = fmaf(s[i][3], kk.w, pk1);
            }
            float pk = pk0 + pk1;
            pk += __shfl_xor_sync(0xffffffffu, pk, 1);
            pk += __shfl_xor_sync(0xffffffffu, pk, 2);
            const float u = beta * (sm.v[tk][row] - alpha * pk);
            float po0 = 0.f, po1 = 0.f;
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                float4 qq = q4[4 * i + part];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    s[i][e] = fmaf(u, kr[i][e], alpha * s[i][e]);
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

        // ---- gated RMSNorm of the batch's outputs, one warp per token
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
                const float zz = to_f(za[base + e]);
                yo[base + e] = from_f<T>(ov[e] * r * __ldg(p.norm_w + lane * PER + e) * siluf_(zz));
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

template <typename T, int D> cudaError_t launch_t(const PrefillArgs &p, cudaStream_t s) {
    const size_t smem = sizeof(RecSmem<D>);
    cudaError_t e = cudaFuncSetAttribute(recurrent_prefill_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    dim3 grid(p.Hv, p.batch);
    recurrent_prefill_kernel<T, D><<<grid, 4 * D, smem, s>>>(p);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_recurrent_prefill(const PrefillArgs &p, cudaStream_t s) {
    if (p.batch == 0)
        return cudaSuccess;
    if (p.bf16)
        return p.D == 128 ? launch_t<__nv_bfloat16, 128>(p, s) : launch_t<__nv_bfloat16, 32>(p, s);
    return p.D == 128 ? launch_t<float, 128>(p, s) : launch_t<float, 32>(p, s);
}

} // namespace gdn
