// gdn_front.cu -- the q/k front end of the tensor-core chunked prefill: the
// depthwise causal conv (kernel 4) + SiLU and the L2 normalisation of the q and
// k channels (Gated DeltaNet row of the component table on "Qwen3.8-2.4T-A95B
// vs Inkling"; linear_conv_kernel_dim in the raw config fields of "Qwen3.8
// 2.4T A95B"), fused with the intra-chunk Gram rows K K^T and Q K^T that the
// chunked form of the recurrence needs.
//
// One CTA per (64-token chunk, q/k head j) reads the chunk's pre-conv q and k
// rows of head j (bf16 or fp32) plus the three rows before the chunk (the
// previous chunk's tail, or the caller's initial conv window / zeros at the
// start of a sequence), and
//   1. convolves, applies SiLU and L2-normalises q and k per token in FP32 and
//      writes them to the workspace ([N, 2 H_k d]: q heads, then k heads), for
//      the chunk kernel's TMA loads;
//   2. forms, with the chunk's rows t = t0 + r (r < nr),
//        kq[t][j][0][s] = k_t . k_{t0+s} for s < r, else 0
//        kq[t][j][1][s] = q_t . k_{t0+s} for s <= r, else 0
//      on the tensor core as D = [K; Q] K^T (M = 128: the 64 k rows then the
//      64 q rows; N = 64), each operand split into tf32 hi + lo parts and
//      D = hi hi^T + hi lo^T + lo hi^T (the lo lo^T term is below 2^-21
//      relative): FP32-accurate products, which the near-cancelling outputs
//      of the layer need.  The 128 columns go in two halves of 64 through one
//      64 KiB shared-memory stage.
#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_sm100.cuh"

namespace gdn {

namespace {

constexpr int kC = 64;  // chunk length
constexpr int kD = 128; // head dim (d_k = d_v)
constexpr int kFrontThreads = 512;
constexpr int kTokPerThread = 8; // tokens per thread: warp w takes tokens 8 (w / 2) .. + 7

struct __align__(1024) FrontSmem {
    float hi[128 * 64]; // [K; Q] hi parts of a 64-column half (two 32-column blocks)
    float lo[128 * 64];
    unsigned long long bar; // the MMAs of the staged half are done
    uint32_t tmem;
};

// 4 activation channels of one row: 8 bytes of bf16 or 16 of fp32, kept raw
// (registers are the kernel's limit) and widened to float4 where used.
template <typename T> struct Quad;
template <> struct Quad<__nv_bfloat16> {
    using raw = uint2;
    static __device__ __forceinline__ raw load(const __nv_bfloat16 *p) {
        return __ldg(reinterpret_cast<const uint2 *>(p));
    }
    static __device__ __forceinline__ raw zero() { return make_uint2(0u, 0u); }
    // a bf16 is the top half of the float with the same value
    static __device__ __forceinline__ float4 f4(raw r) {
        return make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xffff0000u),
                           __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xffff0000u));
    }
};
template <> struct Quad<float> {
    using raw = float4;
    static __device__ __forceinline__ raw load(const float *p) {
        return __ldg(reinterpret_cast<const float4 *>(p));
    }
    static __device__ __forceinline__ raw zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
    static __device__ __forceinline__ float4 f4(raw r) { return r; }
};

template <typename T>
__global__ void __launch_bounds__(kFrontThreads, 1)
qk_front_kernel(PrefillArgs p) {
    using namespace sm100;
    extern __shared__ __align__(1024) unsigned char front_smem_raw[];
    const int ci = blockIdx.x, j = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (ci >= __ldg(p.ws_offs + p.batch))
        return;
    if ((smem_u32(front_smem_raw) & 1023u) != 0) { // swizzled tiles need 1024-byte alignment
        if (tid == 0)
            atomicOr(p.ws_err, 2u);
        return;
    }
    FrontSmem &sm = *reinterpret_cast<FrontSmem *>(front_smem_raw);
    int lo = 0, hi = p.batch - 1; // the sequence n with offs[n] <= ci < offs[n+1]
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(p.ws_offs + mid) <= ci)
            lo = mid;
        else
            hi = mid - 1;
    }
    const int n = lo;
    int64_t s0, e0;
    seq_bounds(p.cu, n, p.N, s0, e0);
    const int cl = ci - __ldg(p.ws_offs + n); // chunk index within the sequence
    const int64_t t0 = s0 + (int64_t)cl * kC;
    const int nr = (int)((e0 - t0) < kC ? (e0 - t0) : kC);
    const int C = (2 * p.Hk + p.Hv) * kD;
    const uint32_t bar = smem_u32(&sm.bar);
    if (tid == 0) {
        mbar_init(bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&sm.tmem), 64);
        tmem_relinquish();
    }

    // ---- conv + SiLU + L2 of 4 channels x 8 tokens per thread.  Warp w: tokens
    //      8 (w / 2) .. + 7, q (w even) or k (w odd); lane: channels 4 lane .. + 3
    //      of head j, so a token's L2 norm is one warp reduction.
    const bool isq = (warp & 1) == 0;
    const int tk0 = kTokPerThread * (warp >> 1);
    const int cc = (isq ? 0 : p.Hk * kD) + j * kD + 4 * lane; // pre-conv channel
    const T *xq = (const T *)p.qkv;
    // taps of the four channels, re-read from L1 at each use (registers are short)
    const float4 *w4 = reinterpret_cast<const float4 *>(p.conv_w) + cc;
    // rows t0 + tk0 - 3 .. t0 + tk0 + 7: inside the sequence from qkv, before it
    // from the initial conv window (or zeros), past its end zeros
    typename Quad<T>::raw rows[kTokPerThread + 3];
#pragma unroll
    for (int k = 0; k < kTokPerThread + 3; ++k) {
        const int64_t t = t0 + tk0 - 3 + k;
        typename Quad<T>::raw x = Quad<T>::zero();
        if (t >= s0 && t < e0)
            x = Quad<T>::load(xq + t * C + cc);
        else if (t < s0 && t >= s0 - 3 && p.init_conv != nullptr)
            x = Quad<T>::load((const T *)p.init_conv + ((int64_t)n * 3 + (3 + (t - s0))) * C + cc);
        rows[k] = x;
    }
    // conv + SiLU of token tt of this thread's four channels
    auto conv = [&](int tt, float (&a)[4]) {
        const float4 r0 = Quad<T>::f4(rows[tt]), r1 = Quad<T>::f4(rows[tt + 1]);
        const float4 r2 = Quad<T>::f4(rows[tt + 2]), r3 = Quad<T>::f4(rows[tt + 3]);
        const float x0[4] = {r0.x, r0.y, r0.z, r0.w}, x1[4] = {r1.x, r1.y, r1.z, r1.w};
        const float x2[4] = {r2.x, r2.y, r2.z, r2.w}, x3[4] = {r3.x, r3.y, r3.z, r3.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 w = __ldg(w4 + i);
            float acc = w.x * x0[i];
            acc = fmaf(w.y, x1[i], acc);
            acc = fmaf(w.z, x2[i], acc);
            acc = fmaf(w.w, x3[i], acc);
            a[i] = siluf_(acc);
        }
    };
    // normalised q | k rows, rounded to nearest tf32 (the operands the chunk
    // kernel's tensor-core products read), go to the workspace; rows past the
    // sequence's end (a partial last chunk) are not written.  The factors stay
    // for the Gram below, which needs the unrounded values.
    float fac[kTokPerThread];
    float *dst = (float *)p.ws_qk + (isq ? 0 : p.Hk * kD) + j * kD + 4 * lane;
    const int64_t QKW = 2 * (int64_t)p.Hk * kD;
#pragma unroll
    for (int tt = 0; tt < kTokPerThread; ++tt) {
        float a[4];
        conv(tt, a);
        float ss = a[0] * a[0];
        ss = fmaf(a[1], a[1], ss);
        ss = fmaf(a[2], a[2], ss);
        ss = fmaf(a[3], a[3], ss);
        ss = group_sum<32>(ss);
        // rows past the sequence's end enter the Gram as zeros
        fac[tt] = tk0 + tt < nr ? rsqrtf(ss + p.l2_eps) * (isq ? p.q_scale : 1.0f) : 0.f;
        if (tk0 + tt < nr)
            *reinterpret_cast<float4 *>(dst + (t0 + tk0 + tt) * QKW) =
                tf32_rna(make_float4(a[0] * fac[tt], a[1] * fac[tt], a[2] * fac[tt], a[3] * fac[tt]));
    }

    // ---- Gram rows on the tensor core, in two 64-column halves through one
    //      stage: stage rows 0..63 are the chunk's k rows, 64..127 its q rows.
    //      Lanes 0..15 of a warp hold columns 0..63 of their head, lanes 16..31
    //      columns 64..127; each lane recomputes its exact normalised values for
    //      its half (cheaper than holding them through the first half's MMAs).
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    bool ok = true;
    constexpr uint32_t id = idesc_tf32(128, 64, false, false);
    const int half_of_lane = lane >> 4;
#pragma unroll 1
    for (int hf = 0; hf < 2; ++hf) {
        if (hf == 1) // the MMAs of half 0 read the stage
            ok = mbar_wait_bounded(bar, 0u, kDefaultWaitLimit) && ok;
        if (half_of_lane == hf) {
            // element (r, c) of the stage (K-major, 128-byte swizzle, 32-column
            // blocks of 128 rows): (c / 32) 4096 + 32 r + 4 ((c % 32) / 4 xor r % 8) + c % 4
            const int c = 4 * (lane & 15);
#pragma unroll
            for (int tt = 0; tt < kTokPerThread; ++tt) {
                float a[4];
                conv(tt, a);
                const float4 x = make_float4(a[0] * fac[tt], a[1] * fac[tt], a[2] * fac[tt], a[3] * fac[tt]);
                const int r = (isq ? kC : 0) + tk0 + tt;
                const int o = (c >> 5) * 4096 + 32 * r + ((((c & 31) >> 2) ^ (r & 7)) << 2);
                const float4 h4 = tf32_rna(x);
                const float4 l4 = tf32_rna(make_float4(x.x - h4.x, x.y - h4.y, x.z - h4.z, x.w - h4.w));
                *reinterpret_cast<float4 *>(sm.hi + o) = h4;
                *reinterpret_cast<float4 *>(sm.lo + o) = l4;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 0) {
            // A = [K; Q] (128 rows), B = its first 64 rows (K); 8 columns a step.
            // The whole warp runs the loop (uniform descriptors), one lane issues.
            const uint32_t is = elect_one() && ok;
            const uint64_t aH = sdesc_sw128(smem_u32(sm.hi), 16, 1024);
            const uint64_t aL = sdesc_sw128(smem_u32(sm.lo), 16, 1024);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint64_t ks = (uint64_t)((((s >> 2) * 4096 + (s & 3) * 8) * 4) >> 4);
                mma_tf32_ss_if(tmem, aH + ks, aH + ks, id, (hf > 0 || s > 0) ? 1u : 0u, is);
                mma_tf32_ss_if(tmem, aH + ks, aL + ks, id, 1, is);
                mma_tf32_ss_if(tmem, aL + ks, aH + ks, id, 1, is);
            }
            mma_commit_if(bar, is);
        }
    }
    ok = mbar_wait_bounded(bar, 1u, kDefaultWaitLimit) && ok; // half 1, and with it every MMA
    tc_fence_after();
    // ---- TMEM lane r = row r of D, columns s.  Warp w reads lanes 32 (w % 4) ..
    //      + 31, columns 16 (w / 4) .. + 15.
    {
        const int r = 32 * (warp & 3) + lane, rr = r & 63, c0 = 16 * (warp >> 2);
        const bool qrow = r >= 64;
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + c0, v);
        tmem_wait_ld();
        if (ok && rr < nr) {
            float *o = (float *)p.ws_kq + ((t0 + rr) * p.Hk + j) * (2 * kC) + (qrow ? kC : 0) + c0;
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
                const int s = c0 + i;
                float4 w;
                w.x = (qrow ? s <= rr : s < rr) ? v[i] : 0.f;
                w.y = (qrow ? s + 1 <= rr : s + 1 < rr) ? v[i + 1] : 0.f;
                w.z = (qrow ? s + 2 <= rr : s + 2 < rr) ? v[i + 2] : 0.f;
                w.w = (qrow ? s + 3 <= rr : s + 3 < rr) ? v[i + 3] : 0.f;
                *reinterpret_cast<float4 *>(o + i) = w;
            }
        }
    }
    if (__syncthreads_or(!ok) && tid == 0)
        atomicOr(p.ws_err, 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        tmem_dealloc(tmem, 64);
}

} // namespace

cudaError_t launch_qk_front(const PrefillArgs &p, cudaStream_t s) {
    if (p.N == 0 || p.batch == 0)
        return cudaSuccess;
    const size_t smem = sizeof(FrontSmem);
    auto kern = p.bf16 ? qk_front_kernel<__nv_bfloat16> : qk_front_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    // upper bound on the chunk count: every sequence adds at most one partial chunk
    dim3 grid((unsigned)((p.N + kC - 1) / kC + p.batch), p.Hk);
    kern<<<grid, kFrontThreads, smem, s>>>(p);
    return cudaGetLastError();
}

} // namespace gdn
