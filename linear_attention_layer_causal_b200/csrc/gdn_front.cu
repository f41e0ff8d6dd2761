// gdn_front.cu -- the intra-chunk Gram rows K K^T and Q K^T of the
// tensor-core chunked prefill (the K K^T and Q K^T factors of the chunked form
// of the Gated DeltaNet recurrence, "Qwen3.8-2.4T-A95B vs Inkling", component
// table, Gated DeltaNet row).
#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_sm100.cuh"

namespace gdn {

namespace {

constexpr int kC = 64;  // chunk length
constexpr int kD = 128; // head dim (d_k = d_v)
constexpr long long kWaitLimit = 2000000000LL; // bounded waits: ~1 s of SM cycles

// One CTA per (chunk, q/k head j): with the chunk's rows t = t0 + r, r < nr,
//   kq[t][j][0][s] = k_t . k_{t0+s} for s < r, else 0
//   kq[t][j][1][s] = q_t . k_{t0+s} for s <= r, else 0
// from the normalised float32 q|k rows of the workspace, on the tensor core:
// D = [K; Q] K^T (M = 128: the chunk's 64 k rows then its 64 q rows, N = 64).
// Every operand is split into tf32 hi + lo parts and D = hi hi^T + hi lo^T +
// lo hi^T (the lo lo^T term is below 2^-21 relative), which is FP32-accurate:
// the near-cancelling outputs of the layer are sensitive to these products,
// and one tf32 pass is not enough.  The 128 columns (d) go in four blocks of
// 32, staged as hi and lo tiles (K-major, 128-byte swizzle) in 32 KB of shared
// memory: each thread loads the next block into registers while the MMAs of
// the current one run, and the small stage lets four CTAs share an SM.
constexpr int kKqThreads = 128;

struct __align__(1024) KqSmem {
    float hi[1][128 * 32]; // [K; Q] hi parts of a 32-column block
    float lo[1][128 * 32];
    unsigned long long bar[1]; // the MMAs of the staged block are done
    uint32_t tmem;
};

__global__ void __launch_bounds__(kKqThreads)
kq_prep_kernel(const float *__restrict__ qk, const int32_t *__restrict__ cu, int batch, int64_t N,
               int Hk, const int32_t *__restrict__ offs, float *__restrict__ kq,
               unsigned int *__restrict__ err) {
    using namespace sm100;
    extern __shared__ __align__(1024) unsigned char kq_smem_raw[];
    const int ci = blockIdx.x, j = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (ci >= __ldg(offs + batch))
        return;
    if ((smem_u32(kq_smem_raw) & 1023u) != 0) { // swizzled tiles need 1024-byte alignment
        if (tid == 0 && err != nullptr)
            atomicOr(err, 2u);
        return;
    }
    KqSmem &sm = *reinterpret_cast<KqSmem *>(kq_smem_raw);
    int lo = 0, hi = batch - 1; // the sequence n with offs[n] <= ci < offs[n+1]
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(offs + mid) <= ci)
            lo = mid;
        else
            hi = mid - 1;
    }
    int64_t s0, e0;
    seq_bounds(cu, lo, N, s0, e0);
    const int64_t t0 = s0 + (int64_t)(ci - __ldg(offs + lo)) * kC;
    const int nr = (int)((e0 - t0) < kC ? (e0 - t0) : kC);
    const int64_t QKW = 2 * (int64_t)Hk * kD;
    const uint32_t bar0 = smem_u32(&sm.bar[0]);
    if (tid == 0) {
        mbar_init(bar0, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&sm.tmem), 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    bool ok = true;
    constexpr uint32_t id = idesc_tf32(128, 64, false, false);
    // row r < 64: k of token t0 + r; r >= 64: q of token t0 + r - 64 (zeros past
    // nr); columns 32 q .. + 31 of the head; thread tid takes the float4 f =
    // tid + 128 i (row f / 8, column 4 (f % 8))
    auto load_block = [&](int q, float4 (&x)[8]) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int f = tid + kKqThreads * i, r = f >> 3, c = 4 * (f & 7), rr = r & 63;
            x[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (rr < nr)
                x[i] = __ldg(reinterpret_cast<const float4 *>(
                    qk + (t0 + rr) * QKW + (r < 64 ? Hk * kD : 0) + j * kD + 32 * q + c));
        }
    };
    float4 xn[8];
    load_block(0, xn);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float4 x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            x[i] = xn[i];
        if (q < 3)
            load_block(q + 1, xn);
        const int st = 0;
        if (q >= 1) // the MMAs of block q - 1 read the stage
            ok = mbar_wait_bounded(bar0, (uint32_t)((q - 1) & 1), kWaitLimit) && ok;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int f = tid + kKqThreads * i, r = f >> 3, c = 4 * (f & 7);
            const float4 h4 = tf32_rna(x[i]);
            const float4 l4 = tf32_rna(make_float4(x[i].x - h4.x, x[i].y - h4.y, x[i].z - h4.z, x[i].w - h4.w));
            const int o = r * 32 + (((c >> 2) ^ (r & 7)) << 2);
            *reinterpret_cast<float4 *>(sm.hi[st] + o) = h4;
            *reinterpret_cast<float4 *>(sm.lo[st] + o) = l4;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0 && ok) {
            // A = [K; Q] (128 rows), B = its first 64 rows (K), K-major, 8 columns a step
            const uint64_t aH = sdesc_sw128(smem_u32(sm.hi[st]), 16, 1024);
            const uint64_t aL = sdesc_sw128(smem_u32(sm.lo[st]), 16, 1024);
#pragma unroll 1
            for (int s = 0; s < 4; ++s) {
                const uint64_t ks = (uint64_t)(s * 32 >> 4);
                mma_tf32_ss(tmem, aH + ks, aH + ks, id, (q > 0 || s > 0) ? 1u : 0u);
                mma_tf32_ss(tmem, aH + ks, aL + ks, id, 1);
                mma_tf32_ss(tmem, aL + ks, aH + ks, id, 1);
            }
            mma_commit(bar0);
        }
    }
    ok = mbar_wait_bounded(bar0, 1u, kWaitLimit) && ok; // block 3, and with it every MMA
    tc_fence_after();
    // TMEM lane r = row r of D; columns s.  Warp w reads lanes 32 w .. + 31.
    {
        const int r = 32 * warp + lane, rr = r & 63;
        const bool isq = r >= 64;
        const uint32_t tl = tmem + ((uint32_t)(32 * warp) << 16);
        float v[2][32];
        tmem_ld32(tl, v[0]);
        tmem_ld32(tl + 32, v[1]);
        tmem_wait_ld();
        if (ok && rr < nr) {
            float *o = kq + ((t0 + rr) * Hk + j) * (2 * kC) + (isq ? kC : 0);
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const int s = 32 * b + i;
                    float4 w4;
                    w4.x = (isq ? s <= rr : s < rr) ? v[b][i] : 0.f;
                    w4.y = (isq ? s + 1 <= rr : s + 1 < rr) ? v[b][i + 1] : 0.f;
                    w4.z = (isq ? s + 2 <= rr : s + 2 < rr) ? v[b][i + 2] : 0.f;
                    w4.w = (isq ? s + 3 <= rr : s + 3 < rr) ? v[b][i + 3] : 0.f;
                    *reinterpret_cast<float4 *>(o + s) = w4;
                }
        }
    }
    if (__syncthreads_or(!ok) && tid == 0 && err != nullptr)
        atomicOr(err, 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        tmem_dealloc(tmem, 64);
}


} // namespace

cudaError_t launch_kq_prep(const PrefillArgs &p, cudaStream_t s) {
    if (p.N == 0 || p.batch == 0)
        return cudaSuccess;
    const size_t smem = sizeof(KqSmem);
    cudaError_t e = cudaFuncSetAttribute(kq_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    // upper bound on the chunk count: every sequence adds at most one partial chunk
    dim3 grid((unsigned)((p.N + kC - 1) / kC + p.batch), p.Hk);
    kq_prep_kernel<<<grid, kKqThreads, smem, s>>>((const float *)p.ws_qk, p.cu, p.batch, p.N, p.Hk,
                                                  p.ws_offs, (float *)p.ws_kq, p.ws_err);
    return cudaGetLastError();
}

} // namespace gdn
