// gdn_front.cu -- the front of the tensor-core chunked prefill, after the
// conv (gdn_conv.cu): the intra-chunk Gram rows and the triangular inverses of
// the chunked form of the Gated DeltaNet recurrence ("Qwen3.8-2.4T-A95B vs
// Inkling", component table, Gated DeltaNet row).
//
// gram_kernel, one CTA per (64-token chunk, q/k head j), with the chunk's
// rows t = t0 + r (r < nr):
//   kq[t][j][s] = q_t . k_{t0+s} for s <= r, else 0           (for P)
//   kk[chunk][j] = k_r . k_s for s < r, a triangular tile    (for A)
// from the normalised float32 q|k rows of the workspace, on the tensor core:
// D = [K; Q] K^T (M = 128: the chunk's 64 k rows then its 64 q rows, N = 64).
// Every operand is split into tf32 hi + lo parts and D = hi hi^T + hi lo^T +
// lo hi^T (the lo lo^T term is below 2^-21 relative), which is FP32-accurate:
// the near-cancelling outputs of the layer are sensitive to these products,
// and one tf32 pass is not enough.  The 128 columns (d) go in four blocks of
// 32, staged as hi and lo tiles (K-major, 128-byte swizzle) in 32 KB of shared
// memory: each thread loads the next block into registers while the MMAs of
// the current one run, and the small stage lets four CTAs share an SM.  The
// q and k rows it has read go back rounded to nearest tf32: the chunk kernel's
// tensor-core products read them there.
//
// tri_kernel, 64 threads per (chunk, value head h), two value heads a CTA:
// the gates of the chunk's tokens (g = -exp(A_log) softplus(a + dt_bias),
// beta = sigmoid(b), G = prefix sums of g; Gated DeltaNet row),
// A[r][s] = beta_r exp(G_r - G_s) kk[r][s], T = (I + A)^-1 as 2 x 2 blocks of
// 32 (each warp solves a diagonal block by forward substitution, one column a
// lane; T21 = -T22 A21 T11 on the tensor core with three tf32 products a tile,
// about FP32 accuracy), and T diag(beta) and -T diag(beta gamma) rounded to
// nearest tf32 into the workspace as 96 rows of 32 floats: the B operands of
// the chunk kernel's MMA 1 and MMA 2b, ready for a TMA load with 128-byte
// swizzle.
#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_sm100.cuh"
#include "gdn_tri.cuh"

namespace gdn {

namespace {

constexpr int kC = 64;  // chunk length
constexpr int kD = 128; // head dim (d_k = d_v)
constexpr long long kWaitLimit = kDefaultWaitLimit; // waits for this CTA's own MMAs

constexpr int kKqThreads = 128;

struct __align__(1024) KqSmem {
    float hi[1][128 * 32]; // [K; Q] hi parts of a 32-column block
    float lo[1][128 * 32];
    unsigned long long bar[1]; // the MMAs of the staged block are done
    uint32_t tmem;
};

__global__ void __launch_bounds__(kKqThreads)
gram_kernel(float *__restrict__ qk, const int32_t *__restrict__ cu, int batch, int64_t N,
               int Hk, const int32_t *__restrict__ offs, float *__restrict__ kq,
            float *__restrict__ kk, unsigned int *__restrict__ err) {
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
                x[i] = __ldcg(reinterpret_cast<const float4 *>(
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
        // the chunk kernel's tensor-core products read q and k: the workspace keeps
        // them rounded to nearest tf32 (only this CTA reads or writes these rows)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int f = tid + kKqThreads * i, r = f >> 3, c = 4 * (f & 7), rr = r & 63;
            if (rr < nr)
                *reinterpret_cast<float4 *>(qk + (t0 + rr) * QKW + (r < 64 ? Hk * kD : 0) + j * kD + 32 * q + c) =
                    tf32_rna(x[i]);
        }
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
        if (warp == 0) {
            // A = [K; Q] (128 rows), B = its first 64 rows (K), K-major, 8 columns a
            // step; the warp runs the loop, one elected lane issues
            const uint32_t is = elect_one() && ok;
            const uint64_t aH = sdesc_sw128(smem_u32(sm.hi[st]), 16, 1024);
            const uint64_t aL = sdesc_sw128(smem_u32(sm.lo[st]), 16, 1024);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint64_t ks = (uint64_t)(s * 32 >> 4);
                mma_tf32_ss_if(tmem, aH + ks, aH + ks, id, (q > 0 || s > 0) ? 1u : 0u, is);
                mma_tf32_ss_if(tmem, aH + ks, aL + ks, id, 1, is);
                mma_tf32_ss_if(tmem, aL + ks, aH + ks, id, 1, is);
            }
            mma_commit_if(bar0, is);
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
        if (ok && isq && rr < nr) { // Q K^T row rr, s <= rr
            float *o = kq + ((t0 + rr) * Hk + j) * kC;
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const int s = 32 * b + i;
                    *reinterpret_cast<float4 *>(o + s) =
                        make_float4(s <= rr ? v[b][i] : 0.f, s + 1 <= rr ? v[b][i + 1] : 0.f,
                                    s + 2 <= rr ? v[b][i + 2] : 0.f, s + 3 <= rr ? v[b][i + 3] : 0.f);
                }
        }
        if (ok && !isq) { // K K^T row rr, s < rr, into the chunk's triangular tile
            float *o = kk + ((size_t)ci * Hk + j) * kTriFloats;
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                if (b == 1 && rr < 32)
                    continue; // the zero quadrant is not stored
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const int s = 32 * b + i;
                    *reinterpret_cast<float4 *>(o + 1024 * b + 32 * rr + (((i >> 2) ^ (rr & 7)) << 2)) =
                        make_float4(s < rr ? v[b][i] : 0.f, s + 1 < rr ? v[b][i + 1] : 0.f,
                                    s + 2 < rr ? v[b][i + 2] : 0.f, s + 3 < rr ? v[b][i + 3] : 0.f);
                }
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



// The sequence n that owns global chunk ci (offs[n] <= ci < offs[n+1]), and the
// chunk's first row t0 and valid rows nr.
__device__ __forceinline__ void chunk_of(const int32_t *__restrict__ cu, const int32_t *__restrict__ offs,
                                         int batch, int64_t N, int ci, int &n, int64_t &t0, int &nr) {
    int lo = 0, hi = batch - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(offs + mid) <= ci)
            lo = mid;
        else
            hi = mid - 1;
    }
    n = lo;
    int64_t s0, e0;
    seq_bounds(cu, n, N, s0, e0);
    t0 = s0 + (int64_t)(ci - __ldg(offs + n)) * kC;
    nr = (int)((e0 - t0) < kC ? (e0 - t0) : kC);
}

// One column of a 32 x 32 diagonal block T_bb = (I + A_bb)^-1 by forward
// substitution, in registers: with x[r] = T_bb[r][c], x[r] = 0 (r < c),
// x[c] = 1, x[r] = -sum_{s<r} A_bb[r][s] x[s] (r > c).  Ab points at row 32 b
// of column block b of the triangular tile (A + 2048 b), so element (r, s) of
// the block sits at Ab + 32 r + 4 ((s / 4) xor (r mod 8)) + s mod 4; every lane
// of the warp reads the same row (broadcast).
__device__ __forceinline__ void tri_diag32(const float *__restrict__ Ab, int c, float (&x)[32]) {
#pragma unroll
    for (int r = 0; r < 32; ++r)
        x[r] = 0.f;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s4 = 0; s4 < r; s4 += 4) {
            const float4 a = *reinterpret_cast<const float4 *>(Ab + 32 * r + (((s4 >> 2) ^ (r & 7)) << 2));
            const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (s4 + e < r)
                    acc[e] = fmaf(av[e], x[s4 + e], acc[e]);
        }
        const float v = -((acc[0] + acc[1]) + (acc[2] + acc[3]));
        x[r] = r < c ? 0.f : (r == c ? 1.f : v);
    }
}

// D += A B for one m16n8k8 tile on the tensor core (tf32 operands, FP32
// accumulation; A row-major, B column-major).  Lane (g, t) = (lane / 4,
// lane % 4) holds A[g][t], A[g + 8][t], A[g][t + 4], A[g + 8][t + 4],
// B[t][g], B[t + 4][g] and D[g][2t], D[g][2t + 1], D[g + 8][2t], D[g + 8][2t + 1].
__device__ __forceinline__ void mma_16x8x8_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// x = hi + lo with both parts tf32 (round to nearest): the split that lets
// three tf32 products, hi hi + hi lo + lo hi, carry about FP32 accuracy
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
    const float h = sm100::tf32_rna(x);
    hi = __float_as_uint(h);
    lo = __float_as_uint(sm100::tf32_rna(x - h));
}

// Columns j0 .. j0 + 15 of a 32 x 32 product D = X Y on the tensor core with
// about FP32 accuracy (three tf32 products a tile).  xa(i, k) and yb(k, j)
// read the operands; D comes back as two 16-row tiles x two 8-column tiles of
// m16n8 accumulators.
template <typename XA, typename YB>
__device__ __forceinline__ void mm32x16_3xtf32(XA xa, YB yb, int j0, int lane, float (&d)[2][2][4]) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                d[mt][nt][e] = 0.f;
#pragma unroll
    for (int k0 = 0; k0 < 32; k0 += 8) {
        uint32_t ah[2][4], al[2][4], bh[2][2], bl[2][2];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            const int i = 16 * mt + g;
            split_tf32(xa(i, k0 + t), ah[mt][0], al[mt][0]);
            split_tf32(xa(i + 8, k0 + t), ah[mt][1], al[mt][1]);
            split_tf32(xa(i, k0 + t + 4), ah[mt][2], al[mt][2]);
            split_tf32(xa(i + 8, k0 + t + 4), ah[mt][3], al[mt][3]);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int j = j0 + 8 * nt + g;
            split_tf32(yb(k0 + t, j), bh[nt][0], bl[nt][0]);
            split_tf32(yb(k0 + t + 4, j), bh[nt][1], bl[nt][1]);
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                mma_16x8x8_tf32(d[mt][nt], al[mt], bh[nt]);
                mma_16x8x8_tf32(d[mt][nt], ah[mt], bl[nt]);
                mma_16x8x8_tf32(d[mt][nt], ah[mt], bh[nt]);
            }
    }
}

// Two value heads a CTA (64 threads each, named barrier 1 + head): gates, A in
// shared memory, then T = (I + A)^-1 by 32 x 32 blocks, and the two B tiles
// straight to the workspace.
template <typename T>
__global__ void __launch_bounds__(128, 4)
tri_kernel(PrefillArgs p) {
    using namespace sm100;
    __shared__ __align__(16) float As[2][kTriFloats];
    __shared__ __align__(16) float Gs[2][kC], Bs[2][kC];
    // the diagonal blocks T11 (row stride 40: read as B fragments without bank
    // conflicts; later the product W = A21 T11 in the same columns) and T22
    // (row stride 36: read as A fragments)
    __shared__ __align__(16) float T1s[2][32 * 40], T2s[2][32 * 36];
    const int ci = blockIdx.x, gi = threadIdx.x >> 6, tt = threadIdx.x & 63, lane = threadIdx.x & 31;
    const int h = 2 * blockIdx.y + gi;
    if (ci >= __ldg(p.ws_offs + p.batch))
        return;
    int n, nr;
    int64_t t0;
    chunk_of(p.cu, p.ws_offs, p.batch, p.N, ci, n, t0, nr);
    const bool live = h < p.Hv;
    const int j = (live ? h : 0) / p.G;
    float *A = As[gi];
    float *G = Gs[gi], *Be = Bs[gi];
    // the K K^T tile of the chunk: thread tt of the group takes float4s tt + 64 i
    const float *kk = (const float *)p.ws_kk + ((size_t)ci * p.Hk + j) * kTriFloats;
    float4 x4[12];
#pragma unroll
    for (int i = 0; i < 12; ++i)
        x4[i] = live ? __ldg(reinterpret_cast<const float4 *>(kk) + tt + 64 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
    if (tt < 32 && live) { // gates of rows tt and tt + 32 (first warp of the group)
        const float negA = -expf(__ldg(p.A_log + h)), dtb = __ldg(p.dt_bias + h);
        float g[2], be[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int rq = tt + 32 * q;
            const bool in = rq < nr;
            const int64_t t = t0 + rq;
            g[q] = in ? negA * softplusf_(to_f(((const T *)p.a)[t * p.Hv + h]) + dtb) : 0.f;
            be[q] = in ? sigmoidf_(to_f(((const T *)p.b)[t * p.Hv + h])) : 0.f;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y0 = __shfl_up_sync(0xffffffffu, g[0], o);
            const float y1 = __shfl_up_sync(0xffffffffu, g[1], o);
            if (lane >= o) {
                g[0] += y0;
                g[1] += y1;
            }
        }
        g[1] += __shfl_sync(0xffffffffu, g[0], 31);
        G[tt] = g[0]; G[tt + 32] = g[1];
        Be[tt] = be[0]; Be[tt + 32] = be[1];
        // the chunk's gate record for the chunk kernel: G, gamma_C / gamma =
        // e^{G_C - G} and gamma = e^G (fast exponential) of every row
        const float Glast = __shfl_sync(0xffffffffu, g[1], 31);
        float *rec = p.ws_gt + ((size_t)ci * p.Hv + h) * kGateRec;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            rec[tt + 32 * q] = g[q];
            rec[kC + tt + 32 * q] = expf(Glast - g[q]);
            rec[2 * kC + tt + 32 * q] = __expf(g[q]);
        }
    }
    group_sync(1 + gi, 64);
    // A[r][s] = beta_r e^{G_r - G_s} KK[r][s] (KK is 0 for s >= r; the clamp keeps
    // the unused upper triangle finite: G_r - G_s > 0 there).  Float4 f of the
    // tile: column block f / 512, row (f % 512) / 8, 16-byte chunk f % 8 holding
    // columns 4 ((f % 8) xor (row % 8)) ..
#pragma unroll
    for (int i = 0; i < 12; ++i) {
        const int f = tt + 64 * i, blk = f >> 9, r = ((f & 511) >> 3) + (blk ? 32 : 0);
        const int c0 = 32 * blk + 4 * ((f & 7) ^ (r & 7));
        const float Gr = G[r], br = Be[r];
        const float4 Gc = *reinterpret_cast<const float4 *>(&G[c0]);
        float4 v = x4[i];
        v.x *= br * __expf(fminf(Gr - Gc.x, 0.f));
        v.y *= br * __expf(fminf(Gr - Gc.y, 0.f));
        v.z *= br * __expf(fminf(Gr - Gc.z, 0.f));
        v.w *= br * __expf(fminf(Gr - Gc.w, 0.f));
        *reinterpret_cast<float4 *>(A + 4 * f) = v;
    }
    group_sync(1 + gi, 64);
    if (!live)
        return;
    // T = (I + A)^-1 as 2 x 2 blocks of 32: each warp solves its diagonal block
    // T_ww = (I + A_ww)^-1 (lane = column); then T21 = -T22 (A21 T11), the two
    // warps taking 16 columns each, on the tensor core.  T diag(beta) and
    // -T diag(beta gamma) (the B tiles of the chunk kernel's MMA 1 and MMA 2b)
    // go out as 96 rows of 32 floats: row r of column block 0, then row r of
    // block 1 at row r + 32 (a TMA load with 128-byte swizzle turns them back
    // into the triangular tile).  gamma = e^G by the same fast exponential as the
    // gate record's.
    float *dst = (float *)p.ws_tb + ((size_t)ci * p.Hv + h) * (2 * 96 * 32);
    float *dsg = dst + 96 * 32;
    const int w = tt >> 5;
    float *T1 = T1s[gi], *T2 = T2s[gi];
    {
        float x[32];
        tri_diag32(A + 2048 * w, lane, x);
        const float bc = Be[tt], gc = __expf(G[tt]);
        float *tw = w ? T2 : T1;
        const int ts = w ? 36 : 40;
        float *db = w ? dst + 64 * 32 + lane : dst + lane; // block 1 rows 32.. / block 0 rows 0..
        float *dg = db + 96 * 32;
#pragma unroll
        for (int r = 0; r < 32; ++r) {
            tw[r * ts + lane] = x[r];
            const float tb = tf32_rna(x[r] * bc);
            db[r * 32] = tb;
            dg[r * 32] = tf32_rna(-tb * gc);
        }
    }
    group_sync(1 + gi, 64);
    const int j0 = 16 * w; // this warp's columns of W and T21
    float d[2][2][4];
    // W = A21 T11: A21 = rows 32..63, columns 0..31 of A (column block 0)
    mm32x16_3xtf32([&](int i, int k) { return A[32 * (32 + i) + (((k >> 2) ^ (i & 7)) << 2) + (k & 3)]; },
                   [&](int k, int j) { return T1[k * 40 + j]; }, j0, lane, d);
    __syncwarp();
    // W takes the place of T11's columns j0 .. j0 + 15, which only this warp reads
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int i = 16 * mt + g, j = j0 + 8 * nt + 2 * t;
            *reinterpret_cast<float2 *>(T1 + i * 40 + j) = make_float2(d[mt][nt][0], d[mt][nt][1]);
            *reinterpret_cast<float2 *>(T1 + (i + 8) * 40 + j) = make_float2(d[mt][nt][2], d[mt][nt][3]);
        }
    __syncwarp();
    // T21 = -T22 W, rows 32..63 of column block 0
    mm32x16_3xtf32([&](int i, int k) { return T2[i * 36 + k]; }, [&](int k, int j) { return T1[k * 40 + j]; },
                   j0, lane, d);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int j = j0 + 8 * nt + 2 * t;
        const float b0 = Be[j], b1 = Be[j + 1], e0 = __expf(G[j]), e1 = __expf(G[j + 1]);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int r = 32 + 16 * mt + g + 8 * hr;
                const float t0 = tf32_rna(-d[mt][nt][2 * hr] * b0), t1 = tf32_rna(-d[mt][nt][2 * hr + 1] * b1);
                *reinterpret_cast<float2 *>(dst + r * 32 + j) = make_float2(t0, t1);
                *reinterpret_cast<float2 *>(dsg + r * 32 + j) = make_float2(tf32_rna(-t0 * e0), tf32_rna(-t1 * e1));
            }
    }
}

} // namespace

cudaError_t launch_gram(const PrefillArgs &p, cudaStream_t s) {
    if (p.N == 0 || p.batch == 0)
        return cudaSuccess;
    const size_t smem = sizeof(KqSmem);
    cudaError_t e = cudaFuncSetAttribute(gram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    // upper bound on the chunk count: every sequence adds at most one partial chunk
    dim3 grid((unsigned)((p.N + kC - 1) / kC + p.batch), p.Hk);
    gram_kernel<<<grid, kKqThreads, smem, s>>>((float *)p.ws_qk, p.cu, p.batch, p.N, p.Hk, p.ws_offs,
                                               (float *)p.ws_kq, (float *)p.ws_kk, p.ws_err);
    return cudaGetLastError();
}

cudaError_t launch_tri(const PrefillArgs &p, cudaStream_t s) {
    if (p.N == 0 || p.batch == 0)
        return cudaSuccess;
    dim3 grid((unsigned)((p.N + kC - 1) / kC + p.batch), (p.Hv + 1) / 2); // two value heads a CTA
    if (p.bf16)
        tri_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(p);
    else
        tri_kernel<float><<<grid, 128, 0, s>>>(p);
    return cudaGetLastError();
}

} // namespace gdn
