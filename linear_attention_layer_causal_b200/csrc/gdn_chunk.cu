// gdn_chunk.cu -- chunked gated delta rule on the sm_100a tensor cores.
//
// The recurrence S_t = a_t S_{t-1}(I - b_t k_t k_t^T) + b_t v_t k_t^T,
// o_t = S_t q_t (the Gated DeltaNet update of "Qwen3.8-2.4T-A95B vs Inkling",
// component table, Gated DeltaNet row) is evaluated C = 64 tokens at a time.
// Inside a chunk, with G_r = sum_{i<=r} g_i (log-decay from the chunk start),
// gamma_r = exp(G_r), and S0 the state entering the chunk, the writes
// u_r = b_r (v_r - a_r S_{r-1} k_r) solve a unit lower-triangular system:
//
//   (I + A) U = diag(b) V - diag(b gamma) K S0^T,
//   A[r][s] = b_r exp(G_r - G_s) (k_r . k_s)            (s < r)
//   =>  U = T diag(b) V - T diag(b gamma) K S0^T,  T = (I + A)^-1
//   O = diag(gamma) Q S0^T + P U,  P[r][s] = exp(G_r - G_s) (q_r . k_s)  (s <= r)
//   S_next = gamma_C S0 + U^T diag(gamma_C / gamma) K.
//
// Only exp(G_r - G_s) with s <= r and exp(G_C - G_s) are ever formed, so no
// factor exceeds 1 however strong the decay.
//
// Mapping onto the tensor core (M = 128 = d_v is the TMEM lane dimension):
//   U~^T = V^T (T diag b)^T          A = V  (smem, MN-major)   B = T diag b (smem)
//   W^T  = K^T (T diag b gamma)^T    A = K  (smem, MN-major)   B = T diag b gamma
//   U^T  = U~^T + S0 (-W)^T          A = S0 (TMEM)             B = -W (smem)
//   O^T  = S0 Q^T, then column r * gamma_r     A = S0 (TMEM)   B = Q (smem)
//   O^T += U^T P^T                   A = U^T (TMEM)            B = P (smem)
//   S   <- gamma_C S + (U diag(gamma_C/gamma))^T K    A = TMEM  B = K (smem, MN-major)
// The FP32 state lives in TMEM for the whole sequence and is itself the A
// operand of the state products.  All products run as kind::tf32.  The
// operands computed here (T diag b, -W, P and both forms of U) are rounded to
// nearest before the tensor core reads them, since its own conversion
// truncates and the resulting bias in U accumulates through the state; v is
// rounded where it is produced; for S, q and k the truncation costs nothing
// measurable.  The intra-chunk Gram matrices K K^T and Q K^T, to which
// near-cancelling outputs are most sensitive, come exact in FP32 from
// kq_prep_kernel.
//
// The gated RMSNorm y = o / rms(o) * w * SiLU(z) ("Qwen3.8-2.4T-A95B vs
// Inkling", output-gate row) is fused into the output store.
#include <cuda.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_sm100.cuh"

namespace gdn {

namespace {

constexpr int kC = 64;  // chunk length
constexpr int kD = 128; // head dim (d_k = d_v)

// -------------------------------------------------------------- K K^T, Q K^T

constexpr int kKqThreads = 256;
constexpr int kTp = kC + 4; // row stride of the transposed tiles (16-byte aligned, banks staggered)

// Chunk offsets: offs[n] = number of 64-token chunks in sequences 0 .. n-1
// (offs[batch] = total).  One CTA of 1024 threads; each thread scans a run of
// consecutive sequences, then the run totals are scanned across the block.
__global__ void __launch_bounds__(1024)
chunk_offsets_kernel(const int32_t *__restrict__ cu, int batch, int64_t N, int32_t *__restrict__ offs) {
    __shared__ int32_t part[1024];
    const int tid = threadIdx.x;
    const int per = (batch + 1023) / 1024;
    const int b0 = tid * per, b1 = b0 + per < batch ? b0 + per : batch;
    int32_t sum = 0;
    for (int n = b0; n < b1; ++n) {
        int64_t s, e;
        seq_bounds(cu, n, N, s, e);
        sum += (int32_t)((e - s + kC - 1) / kC);
    }
    part[tid] = sum;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) { // inclusive scan of the run totals
        const int32_t x = tid >= o ? part[tid - o] : 0;
        __syncthreads();
        part[tid] += x;
        __syncthreads();
    }
    int32_t run = tid > 0 ? part[tid - 1] : 0;
    for (int n = b0; n < b1; ++n) {
        offs[n] = run;
        int64_t s, e;
        seq_bounds(cu, n, N, s, e);
        run += (int32_t)((e - s + kC - 1) / kC);
    }
    if (tid == 1023)
        offs[batch] = part[1023];
}

// One CTA per (chunk, q/k head j): with the chunk's rows t = t0 + r, r < nr,
//   kq[t][j][0][s] = k_t . k_{t0+s} for s < r, else 0
//   kq[t][j][1][s] = q_t . k_{t0+s} for s <= r, else 0
// from the normalised float32 q|k rows of the workspace.  Thread (tr, ts) of
// a 16 x 16 grid owns rows 4 tr .. + 3 and columns 4 ts .. + 3 of both
// products (blocks above the diagonal are zero); the chunk's q and k sit
// transposed in shared memory so that every step reads three float4s.
__global__ void __launch_bounds__(kKqThreads)
kq_prep_kernel(const float *__restrict__ qk, const int32_t *__restrict__ cu, int batch, int64_t N,
               int Hk, const int32_t *__restrict__ offs, float *__restrict__ kq) {
    extern __shared__ __align__(16) float kq_smem[];
    float *Kt = kq_smem;        // Kt[d][r] = k_{t0+r}[d]
    float *Qt = Kt + kD * kTp;  // Qt[d][r] = q_{t0+r}[d]
    const int ci = blockIdx.x, j = blockIdx.y, tid = threadIdx.x;
    if (ci >= __ldg(offs + batch))
        return;
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
    for (int e = tid; e < kC * (kD / 4); e += kKqThreads) {
        const int r = e % kC, d = (e / kC) * 4; // consecutive threads: consecutive rows
        float4 q4 = make_float4(0.f, 0.f, 0.f, 0.f), k4 = q4;
        if (r < nr) {
            const float *row = qk + (t0 + r) * QKW + j * kD + d;
            q4 = __ldg(reinterpret_cast<const float4 *>(row));
            k4 = __ldg(reinterpret_cast<const float4 *>(row + Hk * kD));
        }
        Qt[(d + 0) * kTp + r] = q4.x; Qt[(d + 1) * kTp + r] = q4.y;
        Qt[(d + 2) * kTp + r] = q4.z; Qt[(d + 3) * kTp + r] = q4.w;
        Kt[(d + 0) * kTp + r] = k4.x; Kt[(d + 1) * kTp + r] = k4.y;
        Kt[(d + 2) * kTp + r] = k4.z; Kt[(d + 3) * kTp + r] = k4.w;
    }
    __syncthreads();
    const int tr = tid >> 4, ts = tid & 15;
    float kk[4][4] = {}, qq[4][4] = {};
    if (ts <= tr) {
#pragma unroll 4
        for (int d = 0; d < kD; ++d) {
            const float4 kr = *reinterpret_cast<const float4 *>(Kt + d * kTp + 4 * tr);
            const float4 qr = *reinterpret_cast<const float4 *>(Qt + d * kTp + 4 * tr);
            const float4 ks = *reinterpret_cast<const float4 *>(Kt + d * kTp + 4 * ts);
            const float a[4] = {kr.x, kr.y, kr.z, kr.w}, b[4] = {qr.x, qr.y, qr.z, qr.w};
            const float c[4] = {ks.x, ks.y, ks.z, ks.w};
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    kk[x][y] = fmaf(a[x], c[y], kk[x][y]);
                    qq[x][y] = fmaf(b[x], c[y], qq[x][y]);
                }
        }
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const int r = 4 * tr + x;
        if (r >= nr)
            break;
        float o1[4], o2[4];
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int s = 4 * ts + y;
            o1[y] = s < r ? kk[x][y] : 0.f;
            o2[y] = s <= r ? qq[x][y] : 0.f;
        }
        float *o = kq + ((t0 + r) * Hk + j) * (2 * kC);
        *reinterpret_cast<float4 *>(o + 4 * ts) = make_float4(o1[0], o1[1], o1[2], o1[3]);
        *reinterpret_cast<float4 *>(o + kC + 4 * ts) = make_float4(o2[0], o2[1], o2[2], o2[3]);
    }
}

// ------------------------------------------------------------ chunk kernel
//
// Two warp groups work on consecutive chunks at once:
//   state group (warps 0..7): reads and rewrites TMEM (the W pass, the pass
//     that rounds U and scales O and S, the gated-RMSNorm epilogue) and issues
//     MMA 2 and MMA 3 of the current chunk; warps w and w + 4 share TMEM lanes
//     32 (w % 4) .. + 31 (lane i = value channel i) and split the columns;
//   prep group (warps 8..11): builds the next chunk's gates, A, T = (I+A)^-1,
//     T diag(beta), T diag(beta gamma) and P on the CUDA cores, issues every
//     TMA load and MMA 1.
// They hand over through mbarriers: MMA 1/2/3 completion (tcgen05.commit), a
// "prep ready" arrival, and the TMA transaction barriers of each tile.

constexpr int kStateThreads = 256;
constexpr int kPrepThreads = 128;
constexpr int kThreads = kStateThreads + kPrepThreads;
constexpr int kBarState = 1, kBarPrep = 2; // named barriers of the two groups

// TMEM columns
constexpr uint32_t kColS = 0;    // state S (FP32), 128 columns; also the A operand of S [-W; Q]^T
constexpr uint32_t kColU = 128;  // U^T (starts as U~^T), 64 columns
constexpr uint32_t kColO = 192;  // O^T, 64 columns (directly after U^T: MMA 2 writes both)
constexpr uint32_t kColW = 256;  // W^T, 64 columns
constexpr uint32_t kColUk = 320; // U^T diag(gamma_C / gamma) rounded to tf32, 64 columns
constexpr uint32_t kTmemCols = 512;

// Both operand layouts below split a tile of R rows along its contiguous
// dimension into 32-float (128-byte) column blocks of R rows each.
//
// K-major operand (rows = M or N, columns = K), 128-byte swizzle: the 16-byte
// chunks of row r are XOR-swizzled by r mod 8.
__device__ __forceinline__ int swz(int r, int c, int R) {
    return (c >> 5) * (R * 32) + r * 32 + ((((c & 31) >> 2) ^ (r & 7)) << 2) + (c & 3);
}
// MN-major tf32 operand (rows = K, columns = M or N), 128-byte swizzle on a
// 32-byte base: the 32-byte chunks of row k are XOR-swizzled by k mod 4.
__device__ __forceinline__ int swz_mn(int k, int c, int R) {
    return (c >> 5) * (R * 32) + k * 32 + ((((c & 31) >> 3) ^ (k & 3)) << 3) + (c & 7);
}

template <typename T> struct __align__(1024) ChunkSmem {
    // V and Q share 32-column blocks of 128 rows: rows 0..63 hold V (A,
    // MN-major, for MMA 1), then -W; rows 64..127 hold Q; so that [-W; Q] is
    // one K-major N = 128 operand of MMA 2
    float VQ[2 * kC * kD];
    float K[2][kC * kD];  // A / B, MN-major: K of this chunk and the next (ping-pong)
    float Tb[kC * kC];    // B, K-major: T diag(beta)
    float Tg[kC * kC];    // B, K-major: T diag(beta gamma)
    float P[kC * kC];     // B, K-major: P (lands as raw Q K^T rows)
    float A[kC * kC];     // the next chunk's A (lands as raw K K^T rows), then T; K-major swizzle
    T Z[sizeof(T) == 2 ? kC * kD : 1]; // z rows of this chunk (16-bit activations only)
    float G[2][kC], beta[2][kC];      // cumulative log-decay and beta, by chunk parity
    float gam[2][kC], kd[2][kC];      // gamma_r = e^{G_r} and gamma_C / gamma_r
    float red[4][kC];
    float rstd[kC];
    unsigned long long bar_mma1, bar_mma2, bar_mma3, bar_prep;
    unsigned long long bar_v, bar_q, bar_k[2], bar_p, bar_a, bar_z;
    uint32_t tmem;
    int abort;
    static constexpr int kVQBlk = 2 * kC * 32; // floats per 32-column block of VQ
};

constexpr long long kWaitLimit = 2000000000LL; // ~1 s of SM cycles

// The tensor maps of one call: 64-row boxes of the workspace and of z.
struct ChunkMaps {
    CUtensorMap v;  // convolved v, [N, Hv*128] fp32, 32-column boxes, MN-major tf32 swizzle
    CUtensorMap k;  // normalised k, [N, Hk*128] of the q|k rows, 32-column boxes, MN-major swizzle
    CUtensorMap q;  // normalised q, [N, Hk*128], 32-column boxes, 128-byte swizzle (K-major)
    CUtensorMap kq; // Gram rows, [N, Hk*128] fp32, 32-column boxes, 128-byte swizzle
    CUtensorMap z;  // z, [N, Hv*128] 16-bit, 128-column boxes, no swizzle
};

// Barrier over the `n` threads of one warp group (named barrier `id`).
__device__ __forceinline__ void group_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// The same, returning whether `pred` held on any of the group's threads.
__device__ __forceinline__ bool group_sync_or(int id, int n, bool pred) {
    uint32_t r;
    // operands: %0 = r (output), %1 = id, %2 = n, %3 = pred
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.u32 p, %3, 0;\n\t"
                 "bar.red.or.pred q, %1, %2, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r)
                 : "r"(id), "r"(n), "r"((uint32_t)pred)
                 : "memory");
    return r != 0;
}
// Plain arrival on an mbarrier (release); the waiter's try_wait acquires.
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
chunk_prefill_kernel(PrefillArgs p, const __grid_constant__ ChunkMaps maps) {
    using namespace sm100;
    extern __shared__ unsigned char chunk_smem_raw[];
    ChunkSmem<T> &sm = *reinterpret_cast<ChunkSmem<T> *>(
        (reinterpret_cast<uintptr_t>(chunk_smem_raw) + 1023) & ~uintptr_t(1023));

    const int h = blockIdx.x;
    const int n = blockIdx.y;
    const int j = h / p.G;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const bool is_state = tid < kStateThreads;
    int64_t start, end;
    seq_bounds(p.cu, n, p.N, start, end);
    const int64_t len = end - start;
    const int nchunks = (int)((len + kC - 1) / kC);
    const int64_t HD = (int64_t)p.Hv * kD;

    const uint32_t bar_mma1 = smem_u32(&sm.bar_mma1), bar_mma2 = smem_u32(&sm.bar_mma2);
    const uint32_t bar_mma3 = smem_u32(&sm.bar_mma3), bar_prep = smem_u32(&sm.bar_prep);
    const uint32_t bar_v = smem_u32(&sm.bar_v), bar_q = smem_u32(&sm.bar_q);
    const uint32_t bar_p = smem_u32(&sm.bar_p), bar_a = smem_u32(&sm.bar_a);
    const uint32_t bar_z = smem_u32(&sm.bar_z);
    const uint32_t bar_k0 = smem_u32(&sm.bar_k[0]), bar_k1 = smem_u32(&sm.bar_k[1]);
    if (tid == 0) {
        const uint32_t all[11] = {bar_mma1, bar_mma2, bar_mma3, bar_prep, bar_v, bar_q,
                                  bar_k0, bar_k1, bar_p, bar_a, bar_z};
        for (int b = 0; b < 11; ++b)
            mbar_init(all[b], 1);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&sm.tmem), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    const float negA = -expf(__ldg(p.A_log + h));
    const float dtb = __ldg(p.dt_bias + h);
    const int xq = j * kD, xv = h * kD, xkk = j * 2 * kC;
    auto rows_of = [&](int c) {
        const int64_t left = len - (int64_t)c * kC;
        return (int)(left < kC ? left : kC);
    };
    auto wait = [&](uint32_t bar, uint32_t &ph) {
        const bool w = mbar_wait_bounded(bar, ph, kWaitLimit);
        ph ^= 1u;
        return w;
    };
    // TMA issue by the calling thread: nb 32-column boxes of 64 rows at
    // x0 + 32 b, row t0, column block b landing at dst + b * bstride floats
    auto tma_tile = [&](float *dst, const CUtensorMap *m, int x0, int64_t t0, int nb, uint32_t bar,
                        int bstride) {
        mbar_arrive_expect_tx(bar, (uint32_t)(nb * kC * 32 * sizeof(float)));
        for (int b = 0; b < nb; ++b)
            tma_load_2d(smem_u32(dst + b * bstride), m, x0 + 32 * b, (int)t0, bar);
    };
    auto issue_z = [&](int c) { // by one thread
        if constexpr (sizeof(T) == 2) {
            mbar_arrive_expect_tx(bar_z, (uint32_t)(kC * kD * sizeof(T)));
            tma_load_2d(smem_u32(sm.Z), &maps.z, h * kD, (int)(start + (int64_t)c * kC), bar_z);
        } else { // float32 z is read straight from global memory
            mbar_arrive(bar_z);
        }
    };

    bool ok = true;
    if (!is_state) {
        // ================================================================ prep group
        const int ptid = tid - kStateThreads, pw = ptid >> 5;
        const bool leader = ptid == 0;
        auto psync = [&]() { group_sync(kBarPrep, kPrepThreads); };
        // raw gate inputs of chunk c, rows lane and lane + 32 (first prep warp);
        // converted only in gates() so that the loads overlap other work
        auto load_ab = [&](int c, T (&ra)[2], T (&rb)[2]) {
            if (pw == 0) {
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int r = lane + 32 * q;
                    ra[q] = from_f<T>(0.f);
                    rb[q] = from_f<T>(0.f);
                    if (c < nchunks && r < rows_of(c)) {
                        const int64_t t = start + (int64_t)c * kC + r;
                        ra[q] = ((const T *)p.a)[t * p.Hv + h];
                        rb[q] = ((const T *)p.b)[t * p.Hv + h];
                    }
                }
            }
        };
        // g, beta, the inclusive prefix G, gamma = e^G and gamma_C / gamma of a
        // chunk into slot `sl` (first prep warp; rows lane and lane + 32)
        auto gates = [&](int c, const T (&ra)[2], const T (&rb)[2], int sl) {
            if (pw == 0) {
                float g[2], be[2];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const bool in = c < nchunks && lane + 32 * q < rows_of(c);
                    g[q] = in ? negA * softplusf_(to_f(ra[q]) + dtb) : 0.f;
                    be[q] = in ? sigmoidf_(to_f(rb[q])) : 0.f;
                }
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float x0 = __shfl_up_sync(0xffffffffu, g[0], o);
                    const float x1 = __shfl_up_sync(0xffffffffu, g[1], o);
                    if (lane >= o) {
                        g[0] += x0;
                        g[1] += x1;
                    }
                }
                g[1] += __shfl_sync(0xffffffffu, g[0], 31);
                const float Glast = __shfl_sync(0xffffffffu, g[1], 31);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int r = lane + 32 * q;
                    sm.G[sl][r] = g[q];
                    sm.beta[sl][r] = be[q];
                    sm.gam[sl][r] = expf(g[q]);
                    sm.kd[sl][r] = expf(Glast - g[q]);
                }
            }
        };
        // Each prep thread owns the float4 at column c = 4 (ptid % 16) of rows
        // r = ptid / 16 + 8 k, k = 0..7, in the 64 x 64 tiles below.  Every
        // pass loads all its inputs before its first store, so that the
        // compiler need not order later loads behind stores it cannot
        // disambiguate.
        const int pc = 4 * (ptid & 15), pr = ptid >> 4;
        // K K^T rows -> A in place: A[r][s] = beta_r e^{G_r - G_s} KK[r][s]
        // (the kq rows are 0 for s >= r and beta is 0 on padded rows; the
        // clamp keeps the unused upper triangle finite: G_r - G_s > 0 there)
        auto build_A = [&](int sl) {
            const float4 Gc = *reinterpret_cast<const float4 *>(&sm.G[sl][pc]);
            float4 x[8];
            float Gr[8], br[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                x[k] = *reinterpret_cast<const float4 *>(sm.A + swz(pr + 8 * k, pc, kC));
                Gr[k] = sm.G[sl][pr + 8 * k];
                br[k] = sm.beta[sl][pr + 8 * k];
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                x[k].x *= br[k] * __expf(fminf(Gr[k] - Gc.x, 0.f));
                x[k].y *= br[k] * __expf(fminf(Gr[k] - Gc.y, 0.f));
                x[k].z *= br[k] * __expf(fminf(Gr[k] - Gc.z, 0.f));
                x[k].w *= br[k] * __expf(fminf(Gr[k] - Gc.w, 0.f));
            }
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<float4 *>(sm.A + swz(pr + 8 * k, pc, kC)) = x[k];
        };
        // Q K^T rows -> P in place (K-major swizzled): P[r][s] = e^{G_r - G_s} QK[r][s], tf32
        auto build_P = [&](int sl) {
            const float4 Gc = *reinterpret_cast<const float4 *>(&sm.G[sl][pc]);
            float4 x[8];
            float Gr[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                x[k] = *reinterpret_cast<const float4 *>(sm.P + swz(pr + 8 * k, pc, kC));
                Gr[k] = sm.G[sl][pr + 8 * k];
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                x[k].x = tf32_rna(x[k].x * __expf(fminf(Gr[k] - Gc.x, 0.f)));
                x[k].y = tf32_rna(x[k].y * __expf(fminf(Gr[k] - Gc.y, 0.f)));
                x[k].z = tf32_rna(x[k].z * __expf(fminf(Gr[k] - Gc.z, 0.f)));
                x[k].w = tf32_rna(x[k].w * __expf(fminf(Gr[k] - Gc.w, 0.f)));
            }
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<float4 *>(sm.P + swz(pr + 8 * k, pc, kC)) = x[k];
        };
        // T = (I + A)^-1 for the strictly lower triangular A, in place in sm.A,
        // by block doubling: invert the four 16 x 16 diagonal blocks by forward
        // substitution, then join pairs of blocks with [T1 0; X T2],
        // X = -T2 A21 T1, at 32 and at 64 rows.  Finally T diag(beta) and
        // T diag(beta gamma) are written as tf32 B operands.  sm.Tg serves as
        // scratch for A21 T1 (MMA 1 has finished reading it).
        auto solve = [&](int sl) {
            float *At = sm.A;
            float *Y = sm.Tg;
            { // 16 x 16 diagonal block pw; lane l < 16 owns column 16 pw + l
                const int c = 16 * pw + (lane & 15);
                float t[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                    for (int i = 0; i < r; ++i) {
                        const float a = At[swz(16 * pw + r, 16 * pw + i, kC)];
                        if (i & 1)
                            acc1 = fmaf(a, t[i], acc1);
                        else
                            acc0 = fmaf(a, t[i], acc0);
                    }
                    const int rr = 16 * pw + r;
                    t[r] = rr == c ? 1.f : (rr < c ? 0.f : -(acc0 + acc1));
                }
                __syncwarp();
                if (lane < 16) {
#pragma unroll
                    for (int r = 0; r < 16; ++r)
                        At[swz(16 * pw + r, c, kC)] = t[r];
                }
            }
            psync();
            { // join at 32 rows, blocks b = 0 (rows 0..31) and 1 (rows 32..63); thread:
              // rows r0, r0 + 1 of the 16 x 16 product, columns c0, c0 + 1
                const int b = ptid >> 6, q = ptid & 63;
                const int o = 32 * b, r0 = 2 * (q >> 3), c0 = 2 * (q & 7);
                float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float a0 = At[swz(o + 16 + r0, o + i, kC)];
                    const float a1 = At[swz(o + 17 + r0, o + i, kC)];
                    const float t0 = At[swz(o + i, o + c0, kC)];
                    const float t1 = At[swz(o + i, o + c0 + 1, kC)];
                    y00 = fmaf(a0, t0, y00); y01 = fmaf(a0, t1, y01);
                    y10 = fmaf(a1, t0, y10); y11 = fmaf(a1, t1, y11);
                }
                Y[b * 256 + r0 * 16 + c0] = y00;
                Y[b * 256 + r0 * 16 + c0 + 1] = y01;
                Y[b * 256 + (r0 + 1) * 16 + c0] = y10;
                Y[b * 256 + (r0 + 1) * 16 + c0 + 1] = y11;
                psync();
                float x00 = 0.f, x01 = 0.f, x10 = 0.f, x11 = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float a0 = At[swz(o + 16 + r0, o + 16 + i, kC)];
                    const float a1 = At[swz(o + 17 + r0, o + 16 + i, kC)];
                    const float t0 = Y[b * 256 + i * 16 + c0];
                    const float t1 = Y[b * 256 + i * 16 + c0 + 1];
                    x00 = fmaf(a0, t0, x00); x01 = fmaf(a0, t1, x01);
                    x10 = fmaf(a1, t0, x10); x11 = fmaf(a1, t1, x11);
                }
                // A21 was read only before the barrier above: overwrite it in place
                At[swz(o + 16 + r0, o + c0, kC)] = -x00;
                At[swz(o + 16 + r0, o + c0 + 1, kC)] = -x01;
                At[swz(o + 17 + r0, o + c0, kC)] = -x10;
                At[swz(o + 17 + r0, o + c0 + 1, kC)] = -x11;
            }
            psync();
            { // join at 64 rows: thread: rows r0, r0 + 1 of the 32 x 32 product, columns c0 .. + 3
                const int r0 = 2 * (ptid >> 3), c0 = 4 * (ptid & 7);
                float y[2][4] = {};
#pragma unroll 8
                for (int i = 0; i < 32; ++i) {
                    const float a0 = At[swz(32 + r0, i, kC)];
                    const float a1 = At[swz(33 + r0, i, kC)];
                    const float4 t4 = *reinterpret_cast<const float4 *>(At + swz(i, c0, kC));
                    y[0][0] = fmaf(a0, t4.x, y[0][0]); y[0][1] = fmaf(a0, t4.y, y[0][1]);
                    y[0][2] = fmaf(a0, t4.z, y[0][2]); y[0][3] = fmaf(a0, t4.w, y[0][3]);
                    y[1][0] = fmaf(a1, t4.x, y[1][0]); y[1][1] = fmaf(a1, t4.y, y[1][1]);
                    y[1][2] = fmaf(a1, t4.z, y[1][2]); y[1][3] = fmaf(a1, t4.w, y[1][3]);
                }
                *reinterpret_cast<float4 *>(Y + r0 * 36 + c0) =
                    make_float4(y[0][0], y[0][1], y[0][2], y[0][3]);
                *reinterpret_cast<float4 *>(Y + (r0 + 1) * 36 + c0) =
                    make_float4(y[1][0], y[1][1], y[1][2], y[1][3]);
                psync();
                float x[2][4] = {};
#pragma unroll 8
                for (int i = 0; i < 32; ++i) {
                    const float a0 = At[swz(32 + r0, 32 + i, kC)];
                    const float a1 = At[swz(33 + r0, 32 + i, kC)];
                    const float4 t4 = *reinterpret_cast<const float4 *>(Y + i * 36 + c0);
                    x[0][0] = fmaf(a0, t4.x, x[0][0]); x[0][1] = fmaf(a0, t4.y, x[0][1]);
                    x[0][2] = fmaf(a0, t4.z, x[0][2]); x[0][3] = fmaf(a0, t4.w, x[0][3]);
                    x[1][0] = fmaf(a1, t4.x, x[1][0]); x[1][1] = fmaf(a1, t4.y, x[1][1]);
                    x[1][2] = fmaf(a1, t4.z, x[1][2]); x[1][3] = fmaf(a1, t4.w, x[1][3]);
                }
                *reinterpret_cast<float4 *>(At + swz(32 + r0, c0, kC)) =
                    make_float4(-x[0][0], -x[0][1], -x[0][2], -x[0][3]);
                *reinterpret_cast<float4 *>(At + swz(33 + r0, c0, kC)) =
                    make_float4(-x[1][0], -x[1][1], -x[1][2], -x[1][3]);
            }
            psync();
            // T diag(beta), T diag(beta gamma) -> tf32 K-major operands (rows r, columns s)
            {
                const float4 b4 = *reinterpret_cast<const float4 *>(&sm.beta[sl][pc]);
                const float4 g4 = *reinterpret_cast<const float4 *>(&sm.gam[sl][pc]);
                const float4 bg = make_float4(b4.x * g4.x, b4.y * g4.y, b4.z * g4.z, b4.w * g4.w);
                float4 t4[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    t4[k] = *reinterpret_cast<const float4 *>(At + swz(pr + 8 * k, pc, kC));
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int o = swz(pr + 8 * k, pc, kC);
                    *reinterpret_cast<float4 *>(sm.Tb + o) = tf32_rna(
                        make_float4(t4[k].x * b4.x, t4[k].y * b4.y, t4[k].z * b4.z, t4[k].w * b4.w));
                    *reinterpret_cast<float4 *>(sm.Tg + o) = tf32_rna(
                        make_float4(t4[k].x * bg.x, t4[k].y * bg.y, t4[k].z * bg.z, t4[k].w * bg.w));
                }
            }
        };

        uint32_t ph1 = 0, ph2 = 0, ph3 = 0, phv = 0, phk0 = 0, phk1 = 0, php = 0, pha = 0;
        const uint64_t dV = sdesc_sw128_b32(smem_u32(sm.VQ), 2 * kC * 128, 512); // A of MMA 1
        const uint64_t dTb = sdesc_sw128(smem_u32(sm.Tb), 16, 1024);
        const uint64_t dTg = sdesc_sw128(smem_u32(sm.Tg), 16, 1024);
        const uint64_t dK0 = sdesc_sw128_b32(smem_u32(sm.K[0]), kC * 128, 512);
        const uint64_t dK1 = sdesc_sw128_b32(smem_u32(sm.K[1]), kC * 128, 512);
        constexpr int kVQBlk = ChunkSmem<T>::kVQBlk;
        T av[2], bv[2]; // raw gate inputs of the next chunk to be gated
        if (nchunks > 0) {
            // ---- prologue: all tiles of chunk 0, its gates, T and P
            if (leader) {
                tma_tile(sm.VQ, &maps.v, xv, start, 4, bar_v, kVQBlk);
                tma_tile(sm.VQ + kC * 32, &maps.q, xq, start, 4, bar_q, kVQBlk);
                tma_tile(sm.K[0], &maps.k, xq, start, 4, bar_k0, kC * 32);
                tma_tile(sm.P, &maps.kq, xkk + kC, start, 2, bar_p, kC * 32);
                tma_tile(sm.A, &maps.kq, xkk, start, 2, bar_a, kC * 32);
                issue_z(0);
            }
            load_ab(0, av, bv);
            gates(0, av, bv, 0);
            ok = wait(bar_a, pha) && ok;
            psync();
            build_A(0);
            psync();
            solve(0);
            psync(); // A is free again
            if (leader && nchunks > 1) {
                tma_tile(sm.K[1], &maps.k, xq, start + kC, 4, bar_k1, kC * 32);
                tma_tile(sm.A, &maps.kq, xkk, start + kC, 2, bar_a, kC * 32);
            }
            ok = wait(bar_p, php) && ok;
            build_P(0);
            load_ab(1, av, bv);
            fence_proxy_async_smem();
            psync();
            if (leader)
                mbar_arrive(bar_prep); // chunk 0 ready
        }
        for (int c = 0; c < nchunks; ++c) {
            const int cur = c & 1, nxt = cur ^ 1;
            const int64_t t0 = start + (int64_t)c * kC;
            const bool has_next = c + 1 < nchunks;
            // ---- MMA 1: U~^T = V^T (T diag b)^T and W^T = K^T (T diag b gamma)^T
            if (leader) {
                ok = wait(bar_v, phv) && ok;
                ok = (cur ? wait(bar_k1, phk1) : wait(bar_k0, phk0)) && ok;
                tc_fence_after();
                const uint64_t dK = cur ? dK1 : dK0;
                constexpr uint32_t id = idesc_tf32(128, kC, true, false);
#pragma unroll
                for (int s = 0; s < kC / 8; ++s) {
                    const uint64_t ks = (uint64_t)((((s >> 2) * kC * 128) + (s & 3) * 32) >> 4);
                    mma_tf32_ss(tmem + kColU, dV + s * 64, dTb + ks, id, s > 0);
                    mma_tf32_ss(tmem + kColW, dK + s * 64, dTg + ks, id, s > 0);
                }
                mma_commit(bar_mma1);
            }
            gates(c + 1, av, bv, nxt);
            ok = wait(bar_mma1, ph1) && ok; // T diag(b), T diag(b gamma) are free
            if (has_next) {
                ok = wait(bar_a, pha) && ok;
                psync();
                build_A(nxt);
                psync();
                solve(nxt);
                fence_proxy_async_smem();
                psync(); // A is free, Tb / Tg of the next chunk are written
            }
            ok = wait(bar_mma2, ph2) && ok; // V (then -W) and Q are free
            if (leader && has_next) {
                tma_tile(sm.VQ, &maps.v, xv, t0 + kC, 4, bar_v, kVQBlk);
                tma_tile(sm.VQ + kC * 32, &maps.q, xq, t0 + kC, 4, bar_q, kVQBlk);
            }
            ok = wait(bar_mma3, ph3) && ok; // P, K[cur] and the U / W columns are free
            if (leader) {
                if (has_next)
                    tma_tile(sm.P, &maps.kq, xkk + kC, t0 + kC, 2, bar_p, kC * 32);
                if (c + 2 < nchunks) {
                    tma_tile(sm.K[cur], &maps.k, xq, t0 + 2 * kC, 4, cur ? bar_k1 : bar_k0, kC * 32);
                    tma_tile(sm.A, &maps.kq, xkk, t0 + 2 * kC, 2, bar_a, kC * 32);
                }
            }
            load_ab(c + 2, av, bv);
            if (has_next) {
                ok = wait(bar_p, php) && ok;
                build_P(nxt);
                fence_proxy_async_smem();
                psync();
                if (leader)
                    mbar_arrive(bar_prep); // the next chunk is ready
            }
            if (group_sync_or(kBarPrep, kPrepThreads, !ok || *(volatile int *)&sm.abort)) {
                ok = false;
                break;
            }
        }
        if (!ok)
            *(volatile int *)&sm.abort = 1;
    } else {
        // ================================================================ state group
        const int lq = warp & 3, hf = warp >> 2; // TMEM lane quarter, column half
        const int vch = lq * 32 + lane;          // this thread's TMEM lane = value channel
        const uint32_t tl = tmem + ((uint32_t)(lq * 32) << 16);
        auto ssync = [&]() { group_sync(kBarState, kStateThreads); };
        // initial state into TMEM (row vch, this half's 64 columns); O starts at zero
        {
            const float *src = p.init_state
                                   ? p.init_state + (((size_t)n * p.Hv + h) * kD + vch) * kD + 64 * hf
                                   : nullptr;
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    float4 x = src ? *reinterpret_cast<const float4 *>(src + cb * 32 + i)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
                    v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
                }
                tmem_st32(tl + kColS + 64 * hf + 32 * cb, v);
            }
            float zero[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                zero[i] = 0.f;
            tmem_st32(tl + kColO + 32 * hf, zero); // MMA 2 accumulates onto O
            tmem_wait_st();
        }
        const float wn = __ldg(p.norm_w + vch);
        uint32_t ph1 = 0, ph2 = 0, ph3 = 0, phq = 0, phz = 0, phr = 0;
        const uint64_t dWQ = sdesc_sw128(smem_u32(sm.VQ), 16, 1024); // B of MMA 2 (N = 128)
        const uint64_t dP = sdesc_sw128(smem_u32(sm.P), 16, 1024);
        const uint64_t dK0 = sdesc_sw128_b32(smem_u32(sm.K[0]), kC * 128, 512);
        const uint64_t dK1 = sdesc_sw128_b32(smem_u32(sm.K[1]), kC * 128, 512);
        for (int c = 0; c < nchunks; ++c) {
            const int cur = c & 1;
            const int nr = rows_of(c);
            const int64_t t0 = start + (int64_t)c * kC;
            ok = wait(bar_mma1, ph1) && ok;
            tc_fence_after();
            // ---- -W into rows 0..63 of VQ (K-major: rows r, columns k = vch), tf32;
            //      this half takes rows 32 hf .. 32 hf + 31
            {
                float w[32];
                tmem_ld32(tl + kColW + 32 * hf, w);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    sm.VQ[swz(32 * hf + i, vch, 2 * kC)] = tf32_rna(-w[i]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            ssync();
            tc_fence_after();
            // ---- MMA 2: [U^T | O^T] += S0 [-W; Q]^T, one N = 128 product (A = the
            //      FP32 state in TMEM); U^T starts as U~^T, O^T as zero
            if (tid == 0) {
                ok = wait(bar_q, phq) && ok;
                constexpr uint32_t id = idesc_tf32(128, 2 * kC, false, false);
#pragma unroll
                for (int s = 0; s < kD / 8; ++s) {
                    const uint64_t ks = (uint64_t)((((s >> 2) * 2 * kC * 128) + (s & 3) * 32) >> 4);
                    mma_tf32_ts(tmem + kColU, tmem + kColS + 8 * s, dWQ + ks, id, 1);
                }
                mma_commit(bar_mma2);
            }
            ok = wait(bar_mma2, ph2) && ok;
            ok = wait(bar_prep, phr) && ok; // this chunk's gates and P
            tc_fence_after();
            // ---- TMEM pass (this half's columns): U -> tf32; U diag(gamma_C/gamma)
            //      -> tf32 copy; O columns r scaled by gamma_r; S scaled by gamma_C
            {
                float u[32], o[32], gm[32], kf[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    gm[i] = sm.gam[cur][32 * hf + i];
                    kf[i] = sm.kd[cur][32 * hf + i];
                }
                const float gC = sm.gam[cur][kC - 1]; // padded rows carry g = 0
                tmem_ld32(tl + kColU + 32 * hf, u);
                tmem_ld32(tl + kColO + 32 * hf, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    o[i] *= gm[i];
                tmem_st32(tl + kColO + 32 * hf, o);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    o[i] = tf32_rna(u[i] * kf[i]);
                    u[i] = tf32_rna(u[i]);
                }
                tmem_st32(tl + kColU + 32 * hf, u);
                tmem_st32(tl + kColUk + 32 * hf, o);
#pragma unroll
                for (int cb = 0; cb < 2; ++cb) {
                    float v[32];
                    tmem_ld32(tl + kColS + 64 * hf + 32 * cb, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        v[i] *= gC;
                    tmem_st32(tl + kColS + 64 * hf + 32 * cb, v);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            ssync();
            tc_fence_after();
            // ---- MMA 3: O^T += U^T P^T and S += (U diag(gamma_C/gamma))^T K
            if (tid == 0) {
                const uint64_t dK = cur ? dK1 : dK0;
                constexpr uint32_t idp = idesc_tf32(128, kC, false, false);
                constexpr uint32_t ids = idesc_tf32(128, kD, false, true);
#pragma unroll
                for (int s = 0; s < kC / 8; ++s) {
                    const uint64_t ks = (uint64_t)((((s >> 2) * kC * 128) + (s & 3) * 32) >> 4);
                    mma_tf32_ts(tmem + kColO, tmem + kColU + 8 * s, dP + ks, idp, 1);
                    mma_tf32_ts(tmem + kColS, tmem + kColUk + 8 * s, dK + s * 64, ids, 1);
                }
                mma_commit(bar_mma3);
            }
            ok = wait(bar_z, phz) && ok; // z rows of this chunk
            ok = wait(bar_mma3, ph3) && ok;
            tc_fence_after();
            // ---- epilogue: o[v = vch][r] for this half's rows r = 32 hf + i,
            //      RMSNorm over v, times w[v] SiLU(z), stored; then O is zeroed
            {
                float o[32], sq[32];
                tmem_ld32(tl + kColO + 32 * hf, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    sq[i] = o[i] * o[i];
                // reduce-scatter over the 32 lanes: lane l ends with row 32 hf + l
#pragma unroll
                for (int w = 16; w >= 1; w >>= 1) {
                    const bool upper = (lane & w) != 0;
#pragma unroll
                    for (int i = 0; i < w; ++i) {
                        const float send = upper ? sq[i] : sq[i + w];
                        const float keep = upper ? sq[i + w] : sq[i];
                        sq[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
                    }
                }
                sm.red[lq][32 * hf + lane] = sq[0];
                ssync();
                if (tid < kC)
                    sm.rstd[tid] = rsqrtf((sm.red[0][tid] + sm.red[1][tid] + sm.red[2][tid] +
                                           sm.red[3][tid]) * (1.0f / kD) + p.rms_eps);
                ssync();
                T *yp = (T *)p.y + (t0 + 32 * hf) * HD + (int64_t)h * kD + vch;
                const int rows = nr - 32 * hf; // valid rows of this half (may be <= 0)
                if (p.o_raw != nullptr) {
                    float *op = p.o_raw + (t0 + 32 * hf) * HD + (int64_t)h * kD + vch;
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i < rows)
                            op[i * HD] = o[i];
                }
                // all loads first, then the arithmetic, then the stores
                float zr[32], sc[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if constexpr (sizeof(T) == 2)
                        zr[i] = to_f(sm.Z[(32 * hf + i) * kD + vch]);
                    else
                        zr[i] = i < rows ? to_f(((const T *)p.z)[(t0 + 32 * hf + i) * HD +
                                                                  (int64_t)h * kD + vch])
                                         : 0.f;
                    sc[i] = sm.rstd[32 * hf + i];
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) // o * rstd * w * SiLU(z)
                    o[i] = o[i] * (sc[i] * wn) * __fdividef(zr[i], 1.0f + __expf(-zr[i]));
                if (rows >= 32) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        yp[i * HD] = from_f<T>(o[i]);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i < rows)
                            yp[i * HD] = from_f<T>(o[i]);
                }
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    o[i] = 0.f;
                tmem_st32(tl + kColO + 32 * hf, o); // MMA 2 accumulates onto O
                tmem_wait_st();
            }
            tc_fence_before();
            const bool bad = group_sync_or(kBarState, kStateThreads,
                                           !ok || *(volatile int *)&sm.abort); // Z is read
            tc_fence_after();
            if (bad) {
                ok = false;
                break;
            }
            if (tid == 0 && c + 1 < nchunks)
                issue_z(c + 1);
        }
        if (!ok)
            *(volatile int *)&sm.abort = 1;
    }

    ok = !__syncthreads_or(!ok); // one verdict for the whole CTA
    if (!ok) {
        if (tid == 0 && p.ws_err != nullptr)
            atomicOr(p.ws_err, 1u);
    } else if (is_state && p.final_state != nullptr) {
        const int lq = warp & 3, hf = warp >> 2, vch = lq * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(lq * 32) << 16);
        float *dst = p.final_state + (((size_t)n * p.Hv + h) * kD + vch) * kD + 64 * hf;
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) {
            float v[32];
            tmem_ld32(tl + kColS + 64 * hf + 32 * cb, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4 *>(dst + cb * 32 + i) =
                    make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        tmem_dealloc(tmem, kTmemCols);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime.
EncodeTiledFn encoder() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    return fn;
}

// Row-major 2-D map over `rows` rows of `cols` elements (row pitch `pitch`
// bytes), boxes of `box_cols` x 64 rows.
bool encode_2d(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t cols,
               uint64_t rows, uint64_t pitch, uint32_t box_cols, CUtensorMapSwizzle sw) {
    EncodeTiledFn enc = encoder();
    if (enc == nullptr)
        return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {pitch};
    const cuuint32_t box[2] = {box_cols, (cuuint32_t)kC};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T> cudaError_t launch_chunk_t(const PrefillArgs &p, cudaStream_t s) {
    const size_t smem = sizeof(ChunkSmem<T>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(chunk_prefill_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    ChunkMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (p.N > 0) {
        const uint64_t N = (uint64_t)p.N, F = sizeof(float);
        const uint64_t qkw = 2ull * p.Hk * kD;
        const bool okm =
            encode_2d(&maps.v, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.ws_v, (uint64_t)p.Hv * kD, N,
                      (uint64_t)p.Hv * kD * F, 32, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B) &&
            encode_2d(&maps.k, CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                      (const float *)p.ws_qk + (size_t)p.Hk * kD, (uint64_t)p.Hk * kD, N, qkw * F,
                      32, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B) &&
            encode_2d(&maps.q, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.ws_qk, (uint64_t)p.Hk * kD, N,
                      qkw * F, 32, CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_2d(&maps.kq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.ws_kq, (uint64_t)p.Hk * 2 * kC,
                      N, (uint64_t)p.Hk * 2 * kC * F, 32, CU_TENSOR_MAP_SWIZZLE_128B) &&
            (sizeof(T) != 2 ||
             encode_2d(&maps.z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.z, (uint64_t)p.Hv * kD, N,
                       (uint64_t)p.Hv * kD * sizeof(T), kD, CU_TENSOR_MAP_SWIZZLE_NONE));
        if (!okm)
            return cudaErrorInvalidValue;
    }
    dim3 grid(p.Hv, p.batch);
    chunk_prefill_kernel<T><<<grid, kThreads, smem, s>>>(p, maps);
    return cudaGetLastError();
}

} // namespace

size_t kq_workspace_bytes(int Hk, int64_t N) { return (size_t)N * Hk * 2 * kC * sizeof(float); }

cudaError_t launch_kq_prep(const PrefillArgs &p, cudaStream_t s) {
    if (p.N == 0 || p.batch == 0)
        return cudaSuccess;
    chunk_offsets_kernel<<<1, 1024, 0, s>>>(p.cu, p.batch, p.N, p.ws_offs);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    const size_t smem = sizeof(float) * 2 * kD * kTp;
    e = cudaFuncSetAttribute(kq_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    // upper bound on the chunk count: every sequence adds at most one partial chunk
    dim3 grid((unsigned)((p.N + kC - 1) / kC + p.batch), p.Hk);
    kq_prep_kernel<<<grid, kKqThreads, smem, s>>>((const float *)p.ws_qk, p.cu, p.batch, p.N, p.Hk,
                                                  p.ws_offs, (float *)p.ws_kq);
    return cudaGetLastError();
}

cudaError_t launch_chunk_prefill(const PrefillArgs &p, cudaStream_t s) {
    if (p.batch == 0)
        return cudaSuccess;
    return p.bf16 ? launch_chunk_t<__nv_bfloat16>(p, s) : launch_chunk_t<float>(p, s);
}

} // namespace gdn
