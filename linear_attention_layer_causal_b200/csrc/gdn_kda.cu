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
//     s <- s * alpha;  u = beta (v - s . k);  s <- s + u k;  o = s . q
// (the last equal to (s * alpha) . q + u (k . q)).
// Each head has its own q and k (no sharing).  Both kernels run the update on
// CUDA cores in FP32: the prefill (D / 32 CTAs of 32 state rows per (head,
// sequence), two tokens per step; the conv, SiLU and L2 norm come from the
// shared front kernel; the gated RMSNorm is a separate pass over the raw
// output) and the one-token decode (one CTA per (sequence, head), conv from
// the cache).
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

constexpr int kTB = 16;  // tokens staged per batch
constexpr int kRows = 32; // state rows (value channels) per CTA
constexpr int kLaneRows = 4; // state rows per lane (2 or 4; 2 measured slower)
// 16 lanes share a row group, two groups per warp
constexpr int kPfThreads = 32 * kRows / (2 * kLaneRows);

// Double-buffered token batches: q, k, z and this CTA's v rows arrive by
// cp.async while the previous batch runs.  Per pair of tokens (t0, t1) of the
// current batch, with a0, a1 their decay vectors, the vectors the pair step
// reads are formed once:
//     pv[0] = a0 k0,  pv[1] = a0 q0,  pv[2] = a0 a1 k1,  pv[3] = a0 a1 q1,
//     pv[4] = a0 a1,  pv[5] = a1 k0,
// and the scalars pc = (k0 . a1 k1, k0 . a1 q1, k0 . q0, k1 . q1).
template <typename T, int D> struct KdaSmem {
    float q[2][kTB][D];
    float k[2][kTB][D];
    T z[2][kTB][D];
    float v[2][kTB][kRows];
    float beta[2][kTB];
    float pv[kTB / 2][6][D];
    float4 pc[kTB / 2];
};

// -5 sigmoid(e^A z): the bounded per-channel log-decay, and its exponential
__device__ __forceinline__ float kda_log_decay(float eA, float z) { return -5.0f * sigmoidf_(eA * z); }
__device__ __forceinline__ float kda_decay(float eA, float z) {
    return __expf(-5.0f * __fdividef(1.0f, 1.0f + __expf(-eA * z)));
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Columns held by lane cg (of 16) of a row group: C = D / 16 of them, taken as
// float4s at 4 cg + 64 j (D = 64, 128) or as one float2 at 2 cg (D = 32), so
// that the 16 lanes of a load phase read consecutive shared-memory words.
template <int D> struct KdaCols {
    static constexpr int C = D / 16;
    static_assert(C == 2 || C % 4 == 0, "head dim 32, 64 or 128");
    __device__ static __forceinline__ void load(const float *row, int cg, float (&x)[C]) {
        if constexpr (C == 2) {
            const float2 t = reinterpret_cast<const float2 *>(row)[cg];
            x[0] = t.x; x[1] = t.y;
        } else {
#pragma unroll
            for (int j = 0; j < C / 4; ++j) {
                const float4 t = reinterpret_cast<const float4 *>(row + 64 * j)[cg];
                x[4 * j] = t.x; x[4 * j + 1] = t.y; x[4 * j + 2] = t.z; x[4 * j + 3] = t.w;
            }
        }
    }
    __device__ static __forceinline__ void store(float *row, int cg, const float (&x)[C]) {
        if constexpr (C == 2) {
            reinterpret_cast<float2 *>(row)[cg] = make_float2(x[0], x[1]);
        } else {
#pragma unroll
            for (int j = 0; j < C / 4; ++j)
                reinterpret_cast<float4 *>(row + 64 * j)[cg] =
                    make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
        }
    }
};

// The rows of a head's state evolve independently given each token's k, decay
// and beta, so a head is split over D / 32 CTAs of 32 rows (blockIdx.z), which
// fills the SMs and runs several token chains per SM.  A warp holds 2 R rows
// (R = kLaneRows) as two groups of 16 lanes; each lane keeps R rows x D/16
// columns of the FP32 state, so the shared vectors are read once per R rows.
//
// Tokens go two at a time.  From the row s entering the pair, with
// s0' = a0 s and s1' = a1 (s0' + u0 k0):
//     s0' . k0 = s . pv[0],   s0' . q0 = s . pv[1],
//     s1' . k1 = s . pv[2] + u0 (k0 . a1 k1),
//     s1' . q1 = s . pv[3] + u0 (k0 . a1 q1),
// so the four projections of the pair come from one pass over s, and
//     u0 = beta0 (v0 - s0' . k0),        o0 = s0' . q0 + u0 (k0 . q0),
//     u1 = beta1 (v1 - s1' . k1),        o1 = s1' . q1 + u1 (k1 . q1),
//     s <- (a0 a1) s + u0 (a1 k0) + u1 k1.
// The 4 R partial sums of a lane (R rows x 4 projections) are reduced over its
// 16 lanes by a butterfly that halves the values it carries at each exchange
// (a plain add once one is left), so that group lane cg ends with projection
// d = cg >> 2 of row r, r the next log2(R) bits of cg; u0 and u1 then go back
// to the group by shuffles.  A lane holds its rows and projections in the
// order i ^ r and e ^ d (register slot i holds row lrow0 + (i ^ r); slot group
// e holds projection e ^ d), so that at every exchange it keeps the lower half
// of its values and sends the upper half.  An odd last token is paired with a
// neutral one (decay 1, beta 0, zero q, k, v) whose output is not written.
// Each CTA writes its 32 channels of the raw output o (FP32) to `ob` (the
// call's o_raw, or the workspace); kda_norm_kernel then applies the gated
// RMSNorm, which needs all D channels of a token.
template <typename T, int D>
__global__ void __launch_bounds__(kPfThreads)
kda_prefill_kernel(PrefillArgs p, float *__restrict__ ob) {
    constexpr int NT = kPfThreads;
    constexpr int R = kLaneRows;
    static_assert(R == 2 || R == 4, "2 or 4 rows per lane");
    constexpr int RS = R == 4 ? 0 : 1; // row r = (cg >> RS) & (R - 1)
    constexpr int C = KdaCols<D>::C;  // columns per lane
    constexpr int ZV = 16 / (int)sizeof(T); // z elements per 16-byte copy
    constexpr unsigned FULL = 0xffffffffu;
    extern __shared__ __align__(16) unsigned char kda_smem_raw[];
    KdaSmem<T, D> &sm = *reinterpret_cast<KdaSmem<T, D> *>(kda_smem_raw);
    const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31, cg = lane & 15, gl = lane & 16;
    const int lrow0 = warp * 2 * R + (lane >> 4) * R; // first of this lane's rows within the CTA's 32
    const int row0 = (int)blockIdx.z * kRows + lrow0;
    // after the butterfly: projection d of row r of the group
    const int r = (cg >> RS) & (R - 1), d = cg >> 2;
    int64_t start, end;
    seq_bounds(p.cu, n, p.N, start, end);
    const int64_t len = end - start;
    const float *qk = (const float *)p.ws_qk;
    const float *vv = (const float *)p.ws_v;
    const T *zd = (const T *)p.kda_zdec;
    const int QK = 2 * p.Hk * D;
    const int64_t HD = (int64_t)p.Hv * D;

    // batch [b0, b0 + kTB) into buffer `buf`; rows past the sequence are zero-filled
    auto stage = [&](int buf, int64_t t0) {
        const int nb = (len - t0) < kTB ? (int)(len - t0) : kTB;
        for (int e = tid; e < kTB * (D / 4); e += NT) {
            const int tk = e / (D / 4), c = (e % (D / 4)) * 4;
            const int64_t t = start + t0 + (tk < nb ? tk : 0);
            cp_async16(&sm.q[buf][tk][c], qk + t * QK + h * D + c, tk < nb);
            cp_async16(&sm.k[buf][tk][c], qk + t * QK + p.Hk * D + h * D + c, tk < nb);
        }
        for (int e = tid; e < kTB * (D / ZV); e += NT) {
            const int tk = e / (D / ZV), c = (e % (D / ZV)) * ZV;
            const int64_t t = start + t0 + (tk < nb ? tk : 0);
            cp_async16(&sm.z[buf][tk][c], zd + t * HD + (int64_t)h * D + c, tk < nb);
        }
        for (int e = tid; e < kTB * (kRows / 4); e += NT) {
            const int tk = e / (kRows / 4), c = (e % (kRows / 4)) * 4;
            const int64_t t = start + t0 + (tk < nb ? tk : 0);
            cp_async16(&sm.v[buf][tk][c], vv + t * HD + (int64_t)h * D + (int)blockIdx.z * kRows + c, tk < nb);
        }
        cp_async_commit();
        if (tid < kTB)
            sm.beta[buf][tid] = tid < nb ? sigmoidf_(to_f(((const T *)p.b)[(start + t0 + tid) * p.Hv + h])) : 0.f;
    };

    float s[R][C];
    float *const srow = p.final_state == nullptr ? nullptr
                                                 : p.final_state + (((size_t)n * p.Hv + h) * D + row0) * D;
    {
        const float *irow = p.init_state == nullptr ? nullptr
                                                    : p.init_state + (((size_t)n * p.Hv + h) * D + row0) * D;
#pragma unroll
        for (int i = 0; i < R; ++i) {
            if (irow != nullptr)
                KdaCols<D>::load(irow + (size_t)(i ^ r) * D, cg, s[i]);
            else
#pragma unroll
                for (int c = 0; c < C; ++c)
                    s[i][c] = 0.f;
        }
    }
    const float eA = expf(__ldg(p.A_log + h));
    if (len > 0)
        stage(0, 0);
    int buf = 0;
    for (int64_t tb = 0; tb < len; tb += kTB, buf ^= 1) {
        const int nb = (len - tb) < kTB ? (int)(len - tb) : kTB;
        const int np = (nb + 1) / 2;
        cp_async_wait_all();
        __syncthreads(); // batch tb has landed; the previous batch's tokens are done
        if (tb + kTB < len)
            stage(buf ^ 1, tb + kTB);
        for (int pp = warp; pp < np; pp += NT / 32) {
            const int t0 = 2 * pp, t1 = t0 + 1;
            const bool has1 = t1 < nb;
            float ckk = 0.f, ckq = 0.f, kq0 = 0.f, kq1 = 0.f;
            for (int c = lane; c < D; c += 32) {
                const float a0 = kda_decay(eA, to_f(sm.z[buf][t0][c]));
                const float a1 = has1 ? kda_decay(eA, to_f(sm.z[buf][t1][c])) : 1.0f;
                const float k0 = sm.k[buf][t0][c], q0 = sm.q[buf][t0][c];
                const float k1 = sm.k[buf][t1][c], q1 = sm.q[buf][t1][c];
                const float a01 = a0 * a1, a1k0 = a1 * k0;
                sm.pv[pp][0][c] = a0 * k0;
                sm.pv[pp][1][c] = a0 * q0;
                sm.pv[pp][2][c] = a01 * k1;
                sm.pv[pp][3][c] = a01 * q1;
                sm.pv[pp][4][c] = a01;
                sm.pv[pp][5][c] = a1k0;
                ckk = fmaf(a1k0, k1, ckk);
                ckq = fmaf(a1k0, q1, ckq);
                kq0 = fmaf(k0, q0, kq0);
                kq1 = fmaf(k1, q1, kq1);
            }
            ckk = group_sum<32>(ckk);
            ckq = group_sum<32>(ckq);
            kq0 = group_sum<32>(kq0);
            kq1 = group_sum<32>(kq1);
            if (lane == 0)
                sm.pc[pp] = make_float4(ckk, ckq, kq0, kq1);
        }
        __syncthreads();
        for (int pp = 0; pp < np; ++pp) {
            const int t0 = 2 * pp;
            float a[4 * R];
            {
                float x0[C], x1[C], x2[C], x3[C];
                KdaCols<D>::load(sm.pv[pp][d], cg, x0);
                KdaCols<D>::load(sm.pv[pp][1 ^ d], cg, x1);
                KdaCols<D>::load(sm.pv[pp][2 ^ d], cg, x2);
                KdaCols<D>::load(sm.pv[pp][3 ^ d], cg, x3);
#pragma unroll
                for (int i = 0; i < R; ++i) {
                    float y0 = 0.f, y1 = 0.f, y2 = 0.f, y3 = 0.f;
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        y0 = fmaf(s[i][c], x0[c], y0);
                        y1 = fmaf(s[i][c], x1[c], y1);
                        y2 = fmaf(s[i][c], x2[c], y2);
                        y3 = fmaf(s[i][c], x3[c], y3);
                    }
                    a[i] = y0;
                    a[R + i] = y1;
                    a[2 * R + i] = y2;
                    a[3 * R + i] = y3;
                }
            }
            // butterfly over the 16 lanes: 4 R values halved at each exchange
#pragma unroll
            for (int m = 8, nv = 4 * R; m >= 1; m >>= 1) {
                if (nv > 1) {
#pragma unroll
                    for (int j = 0; j < nv / 2; ++j)
                        a[j] += __shfl_xor_sync(FULL, a[j + nv / 2], m);
                    nv /= 2;
                } else {
                    a[0] += __shfl_xor_sync(FULL, a[0], m);
                }
            }
            const float pr = a[0];
            // every lane of row r: the two u of the pair
            const float pk0 = __shfl_sync(FULL, pr, gl | (r << RS));
            const float xk1 = __shfl_sync(FULL, pr, gl | 8 | (r << RS));
            const float4 sc = sm.pc[pp];
            const float u0 = sm.beta[buf][t0] * (sm.v[buf][t0][lrow0 + r] - pk0);
            const float u1 = sm.beta[buf][t0 + 1] * (sm.v[buf][t0 + 1][lrow0 + r] - fmaf(u0, sc.x, xk1));
            const int64_t ot = (start + tb + t0) * HD + (int64_t)h * D + row0 + r;
            const bool lead = (cg & ((1 << RS) - 1)) == 0; // one lane per (d, r)
            if (d == 1 && lead)
                ob[ot] = fmaf(u0, sc.z, pr);
            else if (d == 3 && lead && t0 + 1 < nb)
                ob[ot + HD] = fmaf(u1, sc.w, fmaf(u0, sc.y, pr));
            float w2[C], w1[C], w0[C];
            KdaCols<D>::load(sm.pv[pp][4], cg, w2);
            KdaCols<D>::load(sm.pv[pp][5], cg, w1);
            KdaCols<D>::load(sm.k[buf][t0 + 1], cg, w0);
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const float u0i = __shfl_sync(FULL, u0, gl | ((i ^ r) << RS));
                const float u1i = __shfl_sync(FULL, u1, gl | ((i ^ r) << RS));
#pragma unroll
                for (int c = 0; c < C; ++c)
                    s[i][c] = fmaf(u1i, w0[c], fmaf(u0i, w1[c], s[i][c] * w2[c]));
            }
        }
    }
    if (srow != nullptr) {
#pragma unroll
        for (int i = 0; i < R; ++i)
            KdaCols<D>::store(srow + (size_t)(i ^ r) * D, cg, s[i]);
    }
}

// y = o / rms(o) * w * sigmoid(gate) for each (token, head): one warp each,
// D / 32 channels a lane
template <typename T, int D>
__global__ void __launch_bounds__(256)
kda_norm_kernel(PrefillArgs p, const float *__restrict__ ob) {
    constexpr int PER = D / 32;
    const int64_t unit = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (unit >= p.N * p.Hv)
        return;
    const int64_t base = unit * D + lane * PER; // [N, H, D] row-major: unit = t * H + h
    float ov[PER];
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        ov[e] = ob[base + e];
        ss = fmaf(ov[e], ov[e], ss);
    }
    ss = group_sum<32>(ss);
    const float r = rsqrtf(ss / (float)D + p.rms_eps);
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        const float gt = to_f(((const T *)p.z)[base + e]);
        ((T *)p.y)[base + e] = from_f<T>(ov[e] * r * __ldg(p.norm_w + lane * PER + e) * sigmoidf_(gt));
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
    // four rows per warp in flight: their loads are issued before any of them is used
    constexpr int KU = 4;
    for (int r0 = warp * RPI + lr; r0 < D; r0 += NW * RPI * KU) {
        float4 sv[KU];
#pragma unroll
        for (int uu = 0; uu < KU; ++uu) {
            const int r = r0 + uu * NW * RPI;
            sv[uu] = r < D ? __ldcs(reinterpret_cast<const float4 *>(Sg + (size_t)r * D + c4))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int uu = 0; uu < KU; ++uu) {
            const int r = r0 + uu * NW * RPI;
            float pk = sv[uu].x * ka[0] + sv[uu].y * ka[1] + sv[uu].z * ka[2] + sv[uu].w * ka[3];
            float pq = sv[uu].x * qa[0] + sv[uu].y * qa[1] + sv[uu].z * qa[2] + sv[uu].w * qa[3];
#pragma unroll
            for (int o = L / 2; o > 0; o >>= 1) {
                pk += __shfl_xor_sync(0xffffffffu, pk, o);
                pq += __shfl_xor_sync(0xffffffffu, pq, o);
            }
            if (r < D) {
                const float u = beta * (vs[r] - pk);
                float4 nv;
                nv.x = fmaf(u, kr[0], al[0] * sv[uu].x);
                nv.y = fmaf(u, kr[1], al[1] * sv[uu].y);
                nv.z = fmaf(u, kr[2], al[2] * sv[uu].z);
                nv.w = fmaf(u, kr[3], al[3] * sv[uu].w);
                __stcs(reinterpret_cast<float4 *>(Sg + (size_t)r * D + c4), nv);
                if ((lane % L) == 0)
                    os[r] = pq + u * kq; // o = (S D) q + u (k . q)
            }
        }
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
    const size_t smem = sizeof(KdaSmem<T, D>);
    cudaError_t e = cudaFuncSetAttribute(kda_prefill_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    float *ob = p.o_raw != nullptr ? p.o_raw : p.ws_o;
    kda_prefill_kernel<T, D><<<dim3(p.Hv, p.batch, D / kRows), kPfThreads, smem, s>>>(p, ob);
    if ((e = cudaGetLastError()) != cudaSuccess || p.N == 0)
        return e;
    const int64_t units = p.N * p.Hv;
    kda_norm_kernel<T, D><<<(unsigned)((units + 7) / 8), 256, 0, s>>>(p, ob);
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
