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
//   U^T  = U~^T + S0 (-W)^T          A = S0 (TMEM, tf32 copy)  B = -W (smem)
//   O^T  = S0 (diag(gamma) Q)^T      A = S0 (TMEM, tf32 copy)  B = gamma Q (smem)
//   O^T += U^T P^T                   A = U^T (TMEM)            B = P (smem)
//   S   <- gamma_C S + U^T K'        A = U^T (TMEM)            B = K' (smem, MN-major)
// The FP32 state lives in TMEM for the whole sequence; a copy rounded to tf32
// (also in TMEM) is the A operand of the state products.  All products run as
// kind::tf32 with every operand rounded to nearest beforehand (the tensor
// core's own conversion truncates, a bias that accumulates over the 128-term
// sums); the intra-chunk Gram matrices K K^T and Q K^T, to which
// near-cancelling outputs are most sensitive, come exact in FP32 from
// kq_prep_kernel.
//
// The gated RMSNorm y = o / rms(o) * w * SiLU(z) ("Qwen3.8-2.4T-A95B vs
// Inkling", output-gate row) is fused into the output store.
#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_sm100.cuh"

namespace gdn {

namespace {

constexpr int kC = 64;  // chunk length
constexpr int kD = 128; // head dim (d_k = d_v)

// -------------------------------------------------------------- K K^T, Q K^T

constexpr int kKqThreads = 256;
constexpr int kKqRows = 64;      // packed tokens per CTA
constexpr int kPad = kD + 1;     // padded smem row (conflict-free column access)

// For q/k head j and packed token t at position r = t - cs of its chunk
// (cs = sequence start + 64 * floor((t - start) / 64)):
//   kq[t][j][0][s] = k_t . k_{cs+s} for s < r, else 0
//   kq[t][j][1][s] = q_t . k_{cs+s} for s <= r, else 0
// from the normalised float32 q|k rows of the workspace.
__global__ void __launch_bounds__(kKqThreads)
kq_prep_kernel(const float *__restrict__ qk, const int32_t *__restrict__ cu, int batch, int64_t N,
               int Hk, float *__restrict__ kq) {
    extern __shared__ float ksm[];
    float *Ks = ksm;                  // [2 kC][kPad] keys of packed rows [lo, lo + 2 kC)
    float *Qs = Ks + 2 * kC * kPad;   // [kKqRows][kPad] queries of the tile's rows
    __shared__ int64_t cs_row[kKqRows];
    const int j = blockIdx.y;
    const int64_t T0 = (int64_t)blockIdx.x * kKqRows;
    const int64_t T1 = T0 + kKqRows < N ? T0 + kKqRows : N;
    const int tid = threadIdx.x;
    if (tid < kKqRows) {
        const int64_t t = T0 + tid;
        int64_t cs = t;
        if (t < N) {
            const int n = seq_of_token(cu, batch, t);
            int64_t s0 = __ldg(cu + n);
            s0 = s0 > t ? t : (s0 < 0 ? 0 : s0);
            cs = s0 + ((t - s0) / kC) * kC;
        }
        cs_row[tid] = cs;
    }
    __syncthreads();
    const int64_t lo = cs_row[0]; // chunk starts are non-decreasing in t
    const int QKW = 2 * Hk * kD;
    // keys of rows [lo, T1) and queries of rows [T0, T1)
    for (int e = tid; e < 2 * kC * (kD / 4); e += kKqThreads) {
        const int rr = e / (kD / 4), c = (e % (kD / 4)) * 4;
        const int64_t t = lo + rr;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t < T1)
            x = __ldg(reinterpret_cast<const float4 *>(qk + t * QKW + Hk * kD + j * kD + c));
        float *dst = Ks + rr * kPad + c;
        dst[0] = x.x; dst[1] = x.y; dst[2] = x.z; dst[3] = x.w;
    }
    for (int e = tid; e < kKqRows * (kD / 4); e += kKqThreads) {
        const int rr = e / (kD / 4), c = (e % (kD / 4)) * 4;
        const int64_t t = T0 + rr;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t < T1)
            x = __ldg(reinterpret_cast<const float4 *>(qk + t * QKW + j * kD + c));
        float *dst = Qs + rr * kPad + c;
        dst[0] = x.x; dst[1] = x.y; dst[2] = x.z; dst[3] = x.w;
    }
    __syncthreads();
    // warp w: tile rows 8w..8w+7; lane l: columns s = l and l + 32
    const int warp = tid >> 5, lane = tid & 31;
    for (int i = 0; i < 8; ++i) {
        const int rl = warp * 8 + i;
        const int64_t t = T0 + rl;
        if (t >= T1)
            break;
        const int64_t cs = cs_row[rl];
        const int r = (int)(t - cs);
        const float *kt = Ks + (int)(t - lo) * kPad;
        const float *qt = Qs + rl * kPad;
        const int s0 = lane, s1 = lane + 32;
        const float *k0 = Ks + (int)(cs - lo + s0) * kPad;
        const float *k1 = Ks + (int)(cs - lo + (s1 < 2 * kC ? s1 : 0)) * kPad;
        float kk0 = 0.f, kk1 = 0.f, qk0 = 0.f, qk1 = 0.f;
        if (s0 <= r) {
#pragma unroll 8
            for (int d = 0; d < kD; ++d) {
                kk0 = fmaf(kt[d], k0[d], kk0);
                qk0 = fmaf(qt[d], k0[d], qk0);
            }
        }
        if (s1 <= r) {
#pragma unroll 8
            for (int d = 0; d < kD; ++d) {
                kk1 = fmaf(kt[d], k1[d], kk1);
                qk1 = fmaf(qt[d], k1[d], qk1);
            }
        }
        float *o = kq + (t * Hk + j) * (2 * kC);
        o[s0] = s0 < r ? kk0 : 0.f;
        o[s1] = s1 < r ? kk1 : 0.f;
        o[kC + s0] = s0 <= r ? qk0 : 0.f;
        o[kC + s1] = s1 <= r ? qk1 : 0.f;
    }
}

// ------------------------------------------------------------ chunk kernel

constexpr int kThreads = 128; // 4 warps: thread i owns TMEM lane i (= value channel i)

// TMEM columns
constexpr uint32_t kColS = 0;    // state S, 128 columns
constexpr uint32_t kColU = 128;  // U^T (starts as U~^T), 64 columns
constexpr uint32_t kColO = 192;  // O^T, 64 columns
constexpr uint32_t kColW = 256;  // W^T, 64 columns
constexpr uint32_t kColSr = 320; // S rounded to tf32 (the A operand), 128 columns
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

struct __align__(1024) ChunkSmem {
    float V[kC * kD];  // A, MN-major: V^T
    float K[kC * kD];  // A, MN-major: K^T; then B, K-major: -W (same bytes, rewritten)
    float Q[kC * kD];  // B, K-major: diag(gamma) Q
    float Kp[kC * kD]; // B, MN-major: diag(gamma_C / gamma) K
    float Tb[kC * kC]; // B, K-major: T diag(beta)
    float Tg[kC * kC]; // B, K-major: T diag(beta gamma)
    float P[kC * kC];  // B, K-major: P
    float A[kC][kC + 1];
    float g[kC], beta[kC], G[kC];
    float red[4][kC];
    float rstd[kC];
    unsigned long long bar;
    uint32_t tmem;
    int abort;
};

constexpr long long kWaitLimit = 2000000000LL; // ~1 s of SM cycles

template <typename T>
__global__ void __launch_bounds__(kThreads, 1) chunk_prefill_kernel(PrefillArgs p) {
    using namespace sm100;
    extern __shared__ unsigned char chunk_smem_raw[];
    ChunkSmem &sm = *reinterpret_cast<ChunkSmem *>(
        (reinterpret_cast<uintptr_t>(chunk_smem_raw) + 1023) & ~uintptr_t(1023));

    const int h = blockIdx.x;
    const int n = blockIdx.y;
    const int j = h / p.G;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    int64_t start, end;
    seq_bounds(p.cu, n, p.N, start, end);
    const int64_t len = end - start;

    const float *qkw = (const float *)p.ws_qk;
    const float *vw = (const float *)p.ws_v;
    const float *kqw = (const float *)p.ws_kq;
    const int QKW = 2 * p.Hk * kD;
    const int64_t HD = (int64_t)p.Hv * kD;

    const uint32_t bar = smem_u32(&sm.bar);
    if (tid == 0) {
        mbar_init(bar, 1);
        sm.abort = 0;
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&sm.tmem), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16; // this warp's TMEM lanes
    const uint32_t tS = tmem + lane_base + kColS, tO = tmem + lane_base + kColO;
    const uint32_t tW = tmem + lane_base + kColW, tU = tmem + lane_base + kColU;
    const uint32_t tSr = tmem + lane_base + kColSr;

    // ---- initial state: row tid of S0 into TMEM lane tid
    {
        const float *src = p.init_state ? p.init_state + (((size_t)n * p.Hv + h) * kD + tid) * kD
                                        : nullptr;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                float4 x = src ? *reinterpret_cast<const float4 *>(src + cb * 32 + i)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
                v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
            }
            tmem_st32(tS + cb * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i)
                v[i] = tf32_rna(v[i]);
            tmem_st32(tSr + cb * 32, v);
        }
        tmem_wait_st();
    }
    const float negA = -expf(__ldg(p.A_log + h));
    const float dtb = __ldg(p.dt_bias + h);
    const float wn = __ldg(p.norm_w + tid);
    uint32_t phase = 0;
    bool ok = true;

    const uint32_t aV = smem_u32(sm.V), aK = smem_u32(sm.K), aQ = smem_u32(sm.Q);
    const uint32_t aKp = smem_u32(sm.Kp), aTb = smem_u32(sm.Tb), aTg = smem_u32(sm.Tg);
    const uint32_t aP = smem_u32(sm.P);
    constexpr uint32_t kBlk = kC * 128; // bytes per 32-column block of a 64-row tile

    for (int64_t c0 = 0; c0 < len && ok; c0 += kC) {
        const int nr = (len - c0) < kC ? (int)(len - c0) : kC;
        const int64_t t0 = start + c0;
        // ---- gates and the cumulative log-decay of the chunk
        if (tid < kC) {
            float g = 0.f, be = 0.f;
            if (tid < nr) {
                const int64_t t = t0 + tid;
                g = negA * softplusf_(to_f(((const T *)p.a)[t * p.Hv + h]) + dtb);
                be = sigmoidf_(to_f(((const T *)p.b)[t * p.Hv + h]));
            }
            sm.g[tid] = g;
            sm.beta[tid] = be;
        }
        __syncthreads();
        if (tid < kC) {
            float acc = 0.f;
            for (int i = 0; i <= tid; ++i)
                acc += sm.g[i];
            sm.G[tid] = acc;
        }
        __syncthreads();
        const float Glast = sm.G[kC - 1]; // padded rows carry g = 0
        // ---- operand tiles
        for (int e = tid; e < kC * (kD / 4); e += kThreads) {
            const int r = e / (kD / 4), c = (e % (kD / 4)) * 4;
            float4 vv = make_float4(0.f, 0.f, 0.f, 0.f), kk = vv, qq = vv;
            if (r < nr) {
                const int64_t t = t0 + r;
                vv = __ldg(reinterpret_cast<const float4 *>(vw + t * HD + (int64_t)h * kD + c));
                kk = __ldg(reinterpret_cast<const float4 *>(qkw + t * QKW + p.Hk * kD + j * kD + c));
                qq = __ldg(reinterpret_cast<const float4 *>(qkw + t * QKW + j * kD + c));
            }
            const float gam = expf(sm.G[r]);
            const float kpf = expf(Glast - sm.G[r]);
            const int o = swz(r, c, kC), om = swz_mn(r, c, kC); // 4 floats stay contiguous
            *reinterpret_cast<float4 *>(sm.V + om) = tf32_rna(vv);
            *reinterpret_cast<float4 *>(sm.K + om) = tf32_rna(kk);
            *reinterpret_cast<float4 *>(sm.Q + o) =
                tf32_rna(make_float4(qq.x * gam, qq.y * gam, qq.z * gam, qq.w * gam));
            *reinterpret_cast<float4 *>(sm.Kp + om) =
                tf32_rna(make_float4(kk.x * kpf, kk.y * kpf, kk.z * kpf, kk.w * kpf));
        }
        for (int e = tid; e < kC * kC; e += kThreads) {
            const int r = e / kC, s = e % kC;
            float a = 0.f, pv = 0.f;
            if (r < nr && s <= r) {
                const float *row = kqw + ((t0 + r) * p.Hk + j) * (2 * kC);
                const float dec = expf(sm.G[r] - sm.G[s]);
                pv = dec * __ldg(row + kC + s);
                if (s < r)
                    a = sm.beta[r] * dec * __ldg(row + s);
            }
            sm.A[r][s] = a;
            sm.P[swz(r, s, kC)] = tf32_rna(pv);
        }
        __syncthreads();
        // ---- T = (I + A)^-1 by forward substitution, one column per thread
        if (tid < kC) {
            const int c = tid;
            float Tc[kC];
#pragma unroll
            for (int r = 0; r < kC; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < r; ++i)
                    acc = fmaf(sm.A[r][i], Tc[i], acc);
                Tc[r] = r == c ? 1.f : (r < c ? 0.f : -acc);
            }
            const float bc = sm.beta[c];
            const float bgc = bc * expf(sm.G[c]);
#pragma unroll
            for (int r = 0; r < kC; ++r) {
                sm.Tb[swz(r, c, kC)] = tf32_rna(Tc[r] * bc);
                sm.Tg[swz(r, c, kC)] = tf32_rna(Tc[r] * bgc);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- MMA 1: U~^T and W^T
        if (tid == 0) {
            const uint32_t id = idesc_tf32(128, kC, true, false);
#pragma unroll
            for (int s = 0; s < kC / 8; ++s) {
                const uint64_t b1 = sdesc_sw128(aTb + (s >> 2) * kBlk + (s & 3) * 32, 16, 1024);
                const uint64_t b2 = sdesc_sw128(aTg + (s >> 2) * kBlk + (s & 3) * 32, 16, 1024);
                mma_tf32_ss(tmem + kColU, sdesc_sw128_b32(aV + s * 1024, kBlk, 512), b1, id, s > 0);
                mma_tf32_ss(tmem + kColW, sdesc_sw128_b32(aK + s * 1024, kBlk, 512), b2, id, s > 0);
            }
            mma_commit(bar);
        }
        ok = mbar_wait_bounded(bar, phase, kWaitLimit);
        phase ^= 1;
        if (__syncthreads_or(!ok))
            break;
        tc_fence_after();
        // ---- -W into the (now free) K tile, K-major: rows r, columns k = tid
        {
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                float w[32];
                tmem_ld32(tW + cb * 32, w);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    sm.K[swz(cb * 32 + i, tid, kC)] = tf32_rna(-w[i]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- MMA 2: U^T = U~^T - S0 W^T and O^T = S0 (gamma Q)^T
        if (tid == 0) {
            const uint32_t id = idesc_tf32(128, kC, false, false);
#pragma unroll
            for (int s = 0; s < kD / 8; ++s) {
                const uint64_t bw = sdesc_sw128(aK + (s >> 2) * kBlk + (s & 3) * 32, 16, 1024);
                mma_tf32_ts(tmem + kColU, tmem + kColSr + 8 * s, bw, id, 1);
            }
#pragma unroll
            for (int s = 0; s < kD / 8; ++s) {
                const uint64_t bq = sdesc_sw128(aQ + (s >> 2) * kBlk + (s & 3) * 32, 16, 1024);
                mma_tf32_ts(tmem + kColO, tmem + kColSr + 8 * s, bq, id, s > 0);
            }
            mma_commit(bar);
        }
        ok = mbar_wait_bounded(bar, phase, kWaitLimit);
        phase ^= 1;
        if (__syncthreads_or(!ok))
            break;
        tc_fence_after();
        // ---- S <- gamma_C S, and U rounded to tf32 in place (A operand of MMA 3)
        {
            const float gC = expf(Glast);
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float v[32];
                tmem_ld32(tS + cb * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    v[i] *= gC;
                tmem_st32(tS + cb * 32, v);
            }
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                float v[32];
                tmem_ld32(tU + cb * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    v[i] = tf32_rna(v[i]);
                tmem_st32(tU + cb * 32, v);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- MMA 3: O^T += U^T P^T and S += U^T K'
        if (tid == 0) {
            const uint32_t idp = idesc_tf32(128, kC, false, false);
            const uint32_t ids = idesc_tf32(128, kD, false, true);
#pragma unroll
            for (int s = 0; s < kC / 8; ++s) {
                const uint64_t bp = sdesc_sw128(aP + (s >> 2) * kBlk + (s & 3) * 32, 16, 1024);
                mma_tf32_ts(tmem + kColO, tmem + kColU + 8 * s, bp, idp, 1);
                const uint64_t bk = sdesc_sw128_b32(aKp + s * 1024, kBlk, 512);
                mma_tf32_ts(tmem + kColS, tmem + kColU + 8 * s, bk, ids, 1);
            }
            mma_commit(bar);
        }
        ok = mbar_wait_bounded(bar, phase, kWaitLimit);
        phase ^= 1;
        if (__syncthreads_or(!ok))
            break;
        tc_fence_after();
        // ---- the next chunk's A operand: S rounded to tf32
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            float v[32];
            tmem_ld32(tS + cb * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i)
                v[i] = tf32_rna(v[i]);
            tmem_st32(tSr + cb * 32, v);
        }
        tmem_wait_st();
        // ---- epilogue: o[v = tid][r], gated RMSNorm over v, store
        float oa[32], ob[32];
        tmem_ld32(tO, oa);
        tmem_ld32(tO + 32, ob);
        tmem_wait_ld();
        {
            float sq[kC];
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                sq[r] = oa[r] * oa[r];
                sq[r + 32] = ob[r] * ob[r];
            }
            // reduce-scatter over the 32 lanes: lane l ends with two sums
            const int lane = tid & 31;
#pragma unroll
            for (int w = 32; w >= 2; w >>= 1) {
                const int off = w >> 1;
                const bool upper = (lane & off) != 0;
#pragma unroll
                for (int i = 0; i < w; ++i) {
                    const float send = upper ? sq[i] : sq[i + w];
                    const float keep = upper ? sq[i + w] : sq[i];
                    sq[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
            // lane bits (4..0) select, from the top, which half was kept at each step
            const int rb = ((lane >> 4) & 1) * 32 + ((lane >> 3) & 1) * 16 + ((lane >> 2) & 1) * 8 +
                           ((lane >> 1) & 1) * 4 + (lane & 1) * 2;
            sm.red[warp][rb] = sq[0];
            sm.red[warp][rb + 1] = sq[1];
        }
        __syncthreads();
        if (tid < kC)
            sm.rstd[tid] = rsqrtf((sm.red[0][tid] + sm.red[1][tid] + sm.red[2][tid] +
                                   sm.red[3][tid]) / (float)kD + p.rms_eps);
        __syncthreads();
        {
            const T *zz = (const T *)p.z;
            T *yy = (T *)p.y;
#pragma unroll
            for (int r = 0; r < kC; ++r) {
                if (r < nr) {
                    const float ov = r < 32 ? oa[r] : ob[r - 32];
                    const int64_t idx = (t0 + r) * HD + (int64_t)h * kD + tid;
                    const float zv = to_f(zz[idx]);
                    yy[idx] = from_f<T>(ov * sm.rstd[r] * wn * siluf_(zv));
                    if (p.o_raw != nullptr)
                        p.o_raw[idx] = ov;
                }
            }
        }
        tc_fence_before();
        __syncthreads(); // tiles and TMEM regions are reused by the next chunk
        tc_fence_after();
    }

    if (!ok) {
        if (tid == 0 && p.ws_err != nullptr)
            atomicOr(p.ws_err, 1u);
    } else if (p.final_state != nullptr) {
        float *dst = p.final_state + (((size_t)n * p.Hv + h) * kD + tid) * kD;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            float v[32];
            tmem_ld32(tS + cb * 32, v);
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

template <typename T> cudaError_t launch_chunk_t(const PrefillArgs &p, cudaStream_t s) {
    const size_t smem = sizeof(ChunkSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(chunk_prefill_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    dim3 grid(p.Hv, p.batch);
    chunk_prefill_kernel<T><<<grid, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

} // namespace

size_t kq_workspace_bytes(int Hk, int64_t N) { return (size_t)N * Hk * 2 * kC * sizeof(float); }

cudaError_t launch_kq_prep(const PrefillArgs &p, cudaStream_t s) {
    if (p.N == 0)
        return cudaSuccess;
    const size_t smem = sizeof(float) * (2 * kC + kKqRows) * kPad;
    cudaError_t e = cudaFuncSetAttribute(kq_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess)
        return e;
    dim3 grid((unsigned)((p.N + kKqRows - 1) / kKqRows), p.Hk);
    kq_prep_kernel<<<grid, kKqThreads, smem, s>>>((const float *)p.ws_qk, p.cu, p.batch, p.N, p.Hk,
                                                  (float *)p.ws_kq);
    return cudaGetLastError();
}

cudaError_t launch_chunk_prefill(const PrefillArgs &p, cudaStream_t s) {
    if (p.batch == 0)
        return cudaSuccess;
    return p.bf16 ? launch_chunk_t<__nv_bfloat16>(p, s) : launch_chunk_t<float>(p, s);
}

} // namespace gdn
