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
// Mapping onto the tensor core (M = 128 = d_v is the TMEM lane dimension),
// with X = K S0^T:
//   MMA 1   U~^T = V^T (T diag b)^T        A = V (smem, MN-major), B = T diag b
//   MMA 2   [X^T | O^T] = S0 [K ; Q]^T     (one N = 128 product; A = the FP32
//           state in TMEM, B = K and Q, K-major); then, in FP32 on the CUDA
//           cores, O^T *= diag(gamma) and S *= gamma_C
//   MMA 2b  U^T = U~^T + X^T (-T diag b gamma)^T     (A = X^T from TMEM)
//   MMA 3   O^T += U^T P^T  and  S += U^T (diag(gamma_C/gamma) K)   (K MN-major)
// The state lives in TMEM for the whole sequence.  All products run as
// kind::tf32 on operands rounded to nearest beforehand (the tensor core's own
// conversion truncates, a bias that would accumulate through the state): q
// and k leave the front kernel rounded, V leaves the conv rounded, and every
// operand formed here (T diag b, -T diag b gamma, P, diag(gamma_C/gamma) K, U)
// is rounded where it is formed; only S0 and X, which the tensor core reads
// straight from TMEM, are truncated.  The Gram matrices K K^T and Q K^T come
// exact in FP32 from the front kernel (gdn_front.cu): the near-cancelling
// outputs are sensitive to them.
//
// The gated RMSNorm y = o / rms(o) * w * SiLU(z) ("Qwen3.8-2.4T-A95B vs
// Inkling", output-gate row) is fused into the output store.
#include <cuda.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_sm100.cuh"
#include "gdn_tmap.h"
#include "gdn_tri.cuh"

namespace gdn {

namespace {

constexpr int kC = 64;  // chunk length
constexpr int kD = 128; // head dim (d_k = d_v)
// The waits that let this CTA's own TMA copies and MMAs finish before it
// releases shared memory and TMEM always get the default bound (~1 s of SM
// cycles); the waits between roles get the call's bound (p.wait_limit).
constexpr long long kWaitLimit = kDefaultWaitLimit;

// ------------------------------------------------------------ chunk offsets

// Chunk offsets: offs[n] = number of 64-token chunks in sequences 0 .. n-1
// (offs[batch] = total).  One CTA of 1024 threads; each thread scans a run of
// consecutive sequences, then the run totals are scanned across the block.
// It is the first kernel of a chunked prefill call, so it also clears the
// call's status words.
__global__ void __launch_bounds__(1024)
chunk_offsets_kernel(const int32_t *__restrict__ cu, int batch, int64_t N, int32_t *__restrict__ offs,
                     unsigned int *__restrict__ err) {
    __shared__ int32_t part[1024];
    const int tid = threadIdx.x;
    if (tid == 0 && err != nullptr) {
        err[0] = 0u; // status word of this call; later kernels only set bits
        err[1] = 0u; // where the first timed-out wait gave up
    }
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

// ------------------------------------------------------------ chunk kernel
//
// One CTA per (value head, sequence) (or per segment of a split sequence),
// four roles that run consecutive chunks at once and hand over through
// mbarriers:
//   state group (warps 0..7): once MMA 2 is done, S *= gamma_C and O^T *=
//     diag(gamma); once MMA 2b is done, U rounded to tf32 in place and
//     U diag(gamma_C / gamma) into the X columns; then the gated-RMSNorm
//     epilogue.  Warps w and w + 4 share TMEM lanes 32 (w % 4) .. + 31
//     (lane = value channel) and split the columns.  X/O and U are
//     double-buffered in TMEM, so the epilogue of chunk c overlaps MMA 2 of
//     chunk c + 1;
//   prep team (warps 8..11): P of chunk c from the Q K^T rows, then for chunk
//     c + 1 the gate record (written by the inverse kernel) and, with 16-bit
//     activations, the v conv into V^T;
//   MMA warp (warp 12): the whole warp runs the issue loop, one elected lane
//     issues;
//   TMA warp (warp 13): one lane reloads each buffer once its last reader is
//     done.
// The per-chunk critical path is MMA 2 -> MMA 2b -> U pass -> MMA 3 -> MMA 2;
// MMA 1 of the next chunk runs beside the U pass.  The roles' loops are
// rolled where that measured faster: the SMs fetch the kernel's code from L2,
// and smaller hot code runs faster.

constexpr int kSG = 256;                          // state group threads
constexpr int kTeam = 128;                        // prep team threads
constexpr int kThreads = kSG + kTeam + 64;        // + MMA warp + TMA warp: 14 warps
constexpr int kWarpMma = (kSG + kTeam) / 32;      // 12
constexpr int kBarSG = 1, kBarT = 2;              // named barriers

// TMEM columns: the state, two [X^T | O^T] pairs (MMA 2 writes one pair with a
// single N = 128 product), two U^T buffers.  All by chunk parity.
constexpr uint32_t kColS = 0;
constexpr uint32_t kColX0 = 128, kColX1 = 256; // O of each pair sits 64 columns on
constexpr uint32_t kColU0 = 384, kColU1 = 448;
constexpr uint32_t kTmemCols = 512;

// Operand layouts.  Both split a tile along its contiguous dimension into
// 32-float (128-byte) column blocks.
//
// K-major operands (rows = M or N, columns = K): 128-byte swizzle, the
// 16-byte chunks of row r XOR-swizzled by r mod 8; element (r, c) of a tile of
// R-row blocks at (c / 32) R 32 + 32 r + 4 (((c mod 32) / 4) xor (r mod 8)) + c mod 4.
// MN-major tf32 operands (V, K) use the 128-byte swizzle on a 32-byte base,
// written only by TMA: 32-byte chunks of row k XOR-swizzled by k mod 4.
// Lower-triangular 64 x 64 tiles use the triangular-tile layout of gdn_tri.cuh.

struct __align__(1024) ChunkSmem {
    // B of MMA 2 (K-major, N = 128 rows): rows 0..63 = K, rows 64..127 = Q
    float KQ[2 * kC * kD];
    // A of MMA 1: V by TMA, MN-major (fp32 activations), or V^T (rows = value
    // channels) written by the prep team, K-major (16-bit activations)
    float V[kC * kD];
    float K[kC * kD];          // B of MMA 3 (MN-major): lands as K, becomes diag(gamma_C/gamma) K
    float Tb[2][kTriFloats];   // B of MMA 1: T diag(beta) (from the inverse kernel, by TMA), by chunk parity
    float Tg[2][kTriFloats];   // B of MMA 2b: -T diag(beta gamma) (the same), by chunk parity
    float P[kTriFloats];       // B of MMA 3: lands as Q K^T rows, becomes P
    // z rows of the chunk (16-bit activations).  Once the state group has formed
    // the gate from it, it stages the chunk's y rows for one TMA store.
    __nv_bfloat16 Z[kC * kD];
    // pre-conv v rows t0 - 3 .. t0 + 63 of the head (16-bit activations), from
    // which the prep team convolves V
    __nv_bfloat16 Vx[(kC + 3) * kD];
    float red[4][kC];          // epilogue: partial sums of o^2 per TMEM lane quarter
    float rstd[kC];            // epilogue: reciprocal RMS of each row
    float G[4][kC], kd[4][kC]; // log-decay prefix and gamma_C / gamma by chunk index mod 4
    float gam[4][kC];          // gamma = e^G (fast exponential), by chunk index mod 4
    unsigned long long bar_v, bar_q, bar_k, bar_kmaj, bar_qk, bar_z; // TMA landings
    unsigned long long bar_tb[2];                               // TMA landing of T diag(beta), by parity
    unsigned long long bar_m1, bar_m2, bar_m2b[2], bar_m3;      // MMA completions
    unsigned long long bar_u, bar_of[2];                        // state group -> MMA
    unsigned long long bar_zf;                                  // state group -> TMA: z tile free
    unsigned long long bar_pT[4], bar_pP;                       // prep team -> MMA, TMA, state group
    unsigned long long bar_fin;                                 // MMA drain on abort
    unsigned long long bar_vx, bar_vxf;                         // TMA landing of Vx; prep team -> TMA: Vx read
    uint32_t tmem;
    int abort;
};
static_assert(sizeof(ChunkSmem) <= 227 * 1024, "the chunk kernel's shared memory exceeds a CTA's 227 KB");


// The tensor maps of one call: 64-row boxes (32-row for the lower half of
// the Gram tiles' second column block) of the workspace.
struct ChunkMaps {
    CUtensorMap v;    // convolved v, [N, Hv*128] fp32, 32-column boxes, MN-major tf32 swizzle (fp32 activations)
    CUtensorMap vx;   // pre-conv qkv rows, [N, conv_dim] bf16, 128 x 67 boxes, no swizzle (bf16 activations)
    CUtensorMap k;    // normalised k, [N, Hk*128] of the q|k rows, MN-major tf32 swizzle
    CUtensorMap q;    // normalised q, [N, Hk*128], 128-byte swizzle (K-major)
    CUtensorMap kmaj; // normalised k, [N, Hk*128], 128-byte swizzle (K-major)
    CUtensorMap kq;   // Q K^T rows, [N, Hk*64] fp32, 32 x 64 boxes, 128-byte swizzle
    CUtensorMap kq32; // the same with 32 x 32 boxes
    CUtensorMap tb;   // T diag(beta) tiles, [chunks * Hv * 96, 32] fp32, 32 x 96 boxes, 128-byte swizzle
    CUtensorMap z;    // z, [N, Hv*128] bf16, 128 x 64 boxes, no swizzle (bf16 activations)
    CUtensorMap y;    // y, the same layout (bf16 activations): the store of a full chunk
};

// The rest of a bounded wait whose first try failed: polls until the phase
// completes, another role aborts, or `limit` SM cycles pass (about 1 s by
// default); on a time-out records `diag` (the first one only) in err[1].  Out
// of line: every wait site shares it.
__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t ph, volatile int *abort_flag,
                                       unsigned int *err, uint32_t diag, long long limit) {
    const long long t0 = clock64();
    while (!sm100::mbar_try_wait_spin(bar, ph)) {
        if (*abort_flag)
            return false;
        if (clock64() - t0 > limit) {
            if (err != nullptr)
                atomicCAS(err + 1, 0u, diag);
            return false;
        }
    }
    return true;
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
    extern __shared__ __align__(1024) unsigned char chunk_smem_raw[];
    // the swizzled tiles need 1024-byte alignment, which the dynamic shared
    // memory window provides when the kernel has no static shared memory; a
    // misaligned window fails the call instead of corrupting the tiles
    if ((smem_u32(chunk_smem_raw) & 1023u) != 0) {
        if (threadIdx.x == 0 && p.ws_err != nullptr)
            atomicOr(p.ws_err, 2u);
        return;
    }
    ChunkSmem &sm = *reinterpret_cast<ChunkSmem *>(chunk_smem_raw);

    const int h = blockIdx.x;
    const int n = blockIdx.y;
    const int j = h / p.G;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    // The segment of sequence n this CTA scans: chunks [cb, ce) of its nc, the
    // sequence cut into p.segments equal runs.  The output pass has one CTA per
    // segment (blockIdx.z); the summary pass two per segment but the last
    // (blockIdx.z = 2 seg + which), which run the segment from S0 = 0 (R) and
    // from S0 = I with the values taken as zero (M), and write no outputs.
    const bool summary = p.seg_pass != 0;
    const int seg = summary ? (int)(blockIdx.z >> 1) : (int)blockIdx.z;
    const bool mpart = summary && (blockIdx.z & 1) != 0;
    int64_t start, end;
    seq_bounds(p.cu, n, p.N, start, end);
    const int nc = (int)((end - start + kC - 1) / kC);
    const int cb = (int)((int64_t)nc * seg / p.segments);
    const int ce = (int)((int64_t)nc * (seg + 1) / p.segments);
    start += (int64_t)cb * kC;
    const int64_t len = (int64_t)(ce - cb) * kC < end - start ? (int64_t)(ce - cb) * kC : end - start;
    const int nchunks = ce - cb;
    const int64_t HD = (int64_t)p.Hv * kD;
    // one 128 x 128 state of the split's workspace: region r (0 = R, 1 = M,
    // 2 = start states, indexed by seg - 1), segment sg
    const int64_t seg_units = (int64_t)p.batch * (p.segments - 1) * p.Hv;
    auto seg_state = [&](int r, int sg) {
        return p.ws_seg + (((int64_t)r * seg_units + ((int64_t)n * (p.segments - 1) + sg) * p.Hv + h) * kD) * kD;
    };

    const uint32_t bar_v = smem_u32(&sm.bar_v), bar_q = smem_u32(&sm.bar_q);
    const uint32_t bar_k = smem_u32(&sm.bar_k), bar_kmaj = smem_u32(&sm.bar_kmaj);
    const uint32_t bar_qk = smem_u32(&sm.bar_qk);
    // T diag(beta) of chunk c landed, by chunk parity
    auto bar_tb = [&](int c) { return smem_u32(&sm.bar_tb[c & 1]); };
    const uint32_t bar_z = smem_u32(&sm.bar_z);
    constexpr bool kZTile = sizeof(T) == 2; // z comes by TMA (16-bit) or from global (fp32)
    constexpr bool kVConv = sizeof(T) == 2; // the prep team convolves v from the pre-conv rows (16-bit)
    const uint32_t bar_m1 = smem_u32(&sm.bar_m1), bar_m2 = smem_u32(&sm.bar_m2);
    const uint32_t bar_m3 = smem_u32(&sm.bar_m3);
    // MMA 2b done, by chunk parity (its waiters are a chunk apart)
    auto bar_m2b = [&](int c) { return smem_u32(&sm.bar_m2b[c & 1]); };
    const uint32_t bar_u = smem_u32(&sm.bar_u);
    const uint32_t bar_of0 = smem_u32(&sm.bar_of[0]), bar_of1 = smem_u32(&sm.bar_of[1]);
    const uint32_t bar_zf = smem_u32(&sm.bar_zf);
    // T tiles + gates of chunk c ready, by chunk index mod 4: a waiter for chunk c
    // must see that phase before the barrier can move on, and the T team may run
    // up to two chunks ahead of the state group
    auto bar_pT = [&](int c) { return smem_u32(&sm.bar_pT[c & 3]); };
    const uint32_t bar_pP = smem_u32(&sm.bar_pP);
    if (tid == 0) {
        const uint32_t one[] = {bar_v,  bar_q,  bar_k,   bar_kmaj, bar_qk,  bar_z,  bar_m1,
                                bar_m2, bar_m3, bar_u,   bar_of0,  bar_of1, bar_pP, bar_zf,
                                smem_u32(&sm.bar_fin), smem_u32(&sm.bar_vx), smem_u32(&sm.bar_vxf)};
#pragma unroll
        for (int b = 0; b < (int)(sizeof(one) / sizeof(one[0])); ++b)
            mbar_init(one[b], 1);
#pragma unroll
        for (int b = 0; b < 4; ++b)
            mbar_init(smem_u32(&sm.bar_pT[b]), 1);
        mbar_init(smem_u32(&sm.bar_m2b[0]), 1);
        mbar_init(smem_u32(&sm.bar_m2b[1]), 1);
        mbar_init(smem_u32(&sm.bar_tb[0]), 1);
        mbar_init(smem_u32(&sm.bar_tb[1]), 1);
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
    volatile int *abort_flag = &sm.abort;
    const int xq = j * kD, xv = h * kD, xkk = j * kC;
    auto rows_of = [&](int c) {
        const int64_t left = len - (int64_t)c * kC;
        return (int)(left < kC ? left : kC);
    };
    // bounded wait on phase `ph` of `bar` (then flips ph); false on time-out or
    // abort.  The first wait of the call that times out records, in the second
    // word of the workspace header, which warp gave up on which barrier:
    // 0x80000000 | warp << 24 | barrier index << 16 | phases this thread had
    // seen on it (low 16 bits); the status word then gets bit 0.
    const uint32_t bar_base = smem_u32(&sm.bar_v);
    uint32_t waits_seen = 0;
    // every wait polls: sleeping on the barrier (a suspend hint) measured slower
    auto waitp = [&](uint32_t bar, uint32_t &ph) {
        bool done = mbar_try_wait_spin(bar, ph);
        if (!done)
            done = wait_slow(bar, ph, abort_flag, p.ws_err,
                             0x80000000u | ((uint32_t)warp << 24) | (((bar - bar_base) / 8) << 16) |
                                 (waits_seen & 0xffffu),
                             p.wait_limit);
        ph ^= 1u;
        ++waits_seen;
        return done;
    };
    // the same for an explicit phase parity (barriers split by chunk index)
    auto waitq = [&](uint32_t bar, uint32_t parity) {
        uint32_t ph = parity;
        return waitp(bar, ph);
    };
    bool ok = true;

    if (warp < kSG / 32) {
        // ==================================================== state group
        const int lq = warp & 3, hf = warp >> 2; // TMEM lane quarter, column half
        const int vch = lq * 32 + lane;          // this thread's TMEM lane = value channel
        const uint32_t tl = tmem + ((uint32_t)(lq * 32) << 16);
        // initial state into TMEM (row vch, this half's 64 columns): the call's
        // (first segment), the chained start state (later segments of the output
        // pass), zero (R) or the identity (M)
        {
            const float *src = nullptr;
            if (!summary && seg > 0)
                src = seg_state(2, seg - 1) + (size_t)vch * kD + 64 * hf;
            else if (!summary && p.init_state != nullptr)
                src = p.init_state + (((size_t)n * p.Hv + h) * kD + vch) * kD + 64 * hf;
#pragma unroll
            for (int bk = 0; bk < 2; ++bk) {
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    float4 x = src ? *reinterpret_cast<const float4 *>(src + bk * 32 + i)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
                    v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
                }
                if (mpart) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        v[i] = vch == 64 * hf + 32 * bk + i ? 1.f : 0.f;
                }
                tmem_st32(tl + kColS + 64 * hf + 32 * bk, v);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        if (group_sync_or(kBarSG, kSG, *abort_flag))
            ok = false;
        if (ok && tid == 0)
            mbar_arrive(bar_u); // phase 0 of the U barrier: the initial state is in TMEM
        const float wn = __ldg(p.norm_w + vch);
        uint32_t ph3 = 0, phz = 0;
        float *red = &sm.red[0][0];
        float *rstd = sm.rstd;
        bool zpend = false; // a y store from the z tile is in flight (uniform over the group)
        // once the y store has read the z tile, the tile may take the next chunk's z
        auto release_z = [&]() {
            if (zpend && tid == 0) {
                bulk_wait_read();
                mbar_arrive(bar_zf);
            }
            zpend = false;
        };
        for (int c = 0; ok && c < nchunks; ++c) {
            release_z();
            const int sl = c & 3;
            const uint32_t cU = (c & 1) ? kColU1 : kColU0, cX = (c & 1) ? kColX1 : kColX0;
            const uint32_t cO = cX + 64;
            // ---- once MMA 2 is done: S *= gamma_C and O^T *= diag(gamma) (MMA 2 left
            //      S0 Q^T there; MMA 3 adds U^T P^T), beside MMA 2b, which touches
            //      neither; then, once MMA 2b is done, the U pass
            {
                bool good = waitq(bar_pT(c), (c >> 2) & 1); // this chunk's gates
                good = waitq(bar_m2, c & 1) && good;
                good = __all_sync(0xffffffffu, good); // TMEM loads are warp-wide
                tc_fence_after();
                if (good) {
                    const float gC = expf(sm.G[sl][kC - 1]); // padded rows carry g = 0
                    // three rounds of two TMEM loads in flight: S columns 0..31 and
                    // 32..63 of this half, then O rows r = 32 hf + 16 q + i
                    const int nrd = summary ? 2 : 3; // the summary pass forms no O
#pragma unroll 1
                    for (int rd = 0; rd < nrd; ++rd) {
                        float v[2][16];
                        const uint32_t col = rd < 2 ? kColS + 64 * hf + 32 * rd : cO + 32 * hf;
                        tmem_ld16(tl + col, v[0]);
                        tmem_ld16(tl + col + 16, v[1]);
                        tmem_wait_ld();
                        if (rd < 2) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                v[0][i] *= gC;
                                v[1][i] *= gC;
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < 2; ++q)
#pragma unroll
                                for (int i = 0; i < 16; i += 4) {
                                    const float4 g4 = *reinterpret_cast<const float4 *>(&sm.gam[sl][32 * hf + 16 * q + i]);
                                    v[q][i] *= g4.x; v[q][i + 1] *= g4.y;
                                    v[q][i + 2] *= g4.z; v[q][i + 3] *= g4.w;
                                }
                        }
                        tmem_st16(tl + col, v[0]);
                        tmem_st16(tl + col + 16, v[1]);
                    }
                }
                good = waitq(bar_m2b(c), (c >> 1) & 1) && good;
                good = __all_sync(0xffffffffu, good);
                tc_fence_after();
                if (good) {
                    // U -> tf32 in place (A of MMA 3's O part) and U diag(gamma_C / gamma)
                    // -> tf32 into the X columns, which MMA 2b has read (A of its state part)
                    float u[2][16];
                    tmem_ld16(tl + cU + 32 * hf, u[0]);
                    tmem_ld16(tl + cU + 32 * hf + 16, u[1]);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        float uk[16];
#pragma unroll
                        for (int i = 0; i < 16; i += 4) {
                            const float4 k4 = *reinterpret_cast<const float4 *>(&sm.kd[sl][32 * hf + 16 * q + i]);
                            uk[i] = tf32_rna(u[q][i] * k4.x);
                            uk[i + 1] = tf32_rna(u[q][i + 1] * k4.y);
                            uk[i + 2] = tf32_rna(u[q][i + 2] * k4.z);
                            uk[i + 3] = tf32_rna(u[q][i + 3] * k4.w);
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            u[q][i] = tf32_rna(u[q][i]);
                        tmem_st16(tl + cU + 32 * hf + 16 * q, u[q]);
                        tmem_st16(tl + cX + 32 * hf + 16 * q, uk);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                if (group_sync_or(kBarSG, kSG, !good || *abort_flag)) {
                    ok = false;
                    break;
                }
                if (tid == 0)
                    mbar_arrive(bar_u);
            }
            if (summary)
                continue; // no outputs
            // ---- epilogue: o[v = vch][r] for this half's rows r = 32 hf + i,
            //      RMSNorm over v, times w[v] SiLU(z), stored
            {
                const int64_t t0 = start + (int64_t)c * kC;
                const int rows = rows_of(c) - 32 * hf; // valid rows of this half (may be <= 0)
                const bool full = rows_of(c) == kC;
                // the gate w[v] SiLU(z) does not depend on the state: form it while
                // MMA 3 runs
                float gt[32];
                bool zok = true;
                if constexpr (kZTile) {
                    zok = __all_sync(0xffffffffu, waitp(bar_z, phz));
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        gt[i] = to_f(sm.Z[(32 * hf + i) * kD + vch]);
                } else {
                    const T *zp = (const T *)p.z + (t0 + 32 * hf) * HD + (int64_t)h * kD + vch;
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        gt[i] = i < rows ? ld_cg(zp + i * HD) : 0.f;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    gt[i] = wn * __fdividef(gt[i], 1.0f + __expf(-gt[i]));
                group_sync(kBarSG, kSG); // the z tile is read: it takes the y rows below
                bool good = zok && __all_sync(0xffffffffu, waitp(bar_m3, ph3));
                tc_fence_after();
                float o[32];
                if (good) {
                    float sq[32];
                    tmem_ld32(tl + cO + 32 * hf, o);
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
                    red[lq * kC + 32 * hf + lane] = sq[0];
                }
                group_sync(kBarSG, kSG);
                if (tid < kC)
                    rstd[tid] = rsqrtf((red[tid] + red[kC + tid] + red[2 * kC + tid] +
                                        red[3 * kC + tid]) * (1.0f / kD) + p.rms_eps);
                group_sync(kBarSG, kSG);
                if (good) {
                    if (p.o_raw != nullptr) {
                        float *op = p.o_raw + (t0 + 32 * hf) * HD + (int64_t)h * kD + vch;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i < rows)
                                st_cg(op + i * HD, o[i]);
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) // o * rstd * w * SiLU(z)
                        o[i] = o[i] * rstd[32 * hf + i] * gt[i];
                    if (kZTile && full) { // y rows into the z tile, then one TMA store
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            reinterpret_cast<__nv_bfloat16 *>(sm.Z)[(32 * hf + i) * kD + vch] =
                                __float2bfloat16_rn(o[i]);
                    } else {
                        T *yp = (T *)p.y + (t0 + 32 * hf) * HD + (int64_t)h * kD + vch;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i < rows)
                                st_cg(yp + i * HD, o[i]);
                    }
                }
                if (kZTile && full) {
                    fence_proxy_async_smem();
                    group_sync(kBarSG, kSG);
                    if (tid == 0 && good) {
                        tma_store_2d(&maps.y, h * kD, (int)t0, smem_u32(sm.Z));
                        bulk_commit();
                    }
                    zpend = true; // released at the top of the next chunk
                } else if (kZTile && tid == 0) {
                    mbar_arrive(bar_zf); // read by the gate step (before the sums above)
                }
                tc_fence_before();
                if (group_sync_or(kBarSG, kSG, !good || *abort_flag)) {
                    ok = false;
                    break;
                }
                if (tid == 0)
                    mbar_arrive((c & 1) ? bar_of1 : bar_of0);
            }
        }
        release_z();
        if (!ok)
            *abort_flag = 1;
    } else if (warp < (kSG + kTeam) / 32) {
        // ==================================================== prep team
        // Per chunk: the gate record; P from the Q K^T rows (tf32, in the
        // triangular-tile layout); with 16-bit activations the v conv.
        const int tt = tid - kSG;
        const TriThread tr(tt);
        // The gate record of chunk c, formed by the inverse kernel: G, gamma_C /
        // gamma and gamma of its 64 rows (padded rows carry g = 0), 48 float4s
        // that threads tt < 48 load one chunk ahead and store into slot c mod 4.
        // (a call without tokens has no workspace: nothing is read then)
        const float *grec =
            nchunks > 0 ? p.ws_gt + ((size_t)(__ldg(p.ws_offs + n) + cb) * p.Hv + h) * kGateRec : nullptr;
        auto load_gt = [&](int c) {
            return tt < kGateRec / 4 && c < nchunks
                       ? __ldg(reinterpret_cast<const float4 *>(grec + (size_t)c * p.Hv * kGateRec) + tt)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
        };
        auto put_gt = [&](const float4 &v, int sl) {
            if (tt < kGateRec / 4) {
                const int arr = tt >> 4, e = 4 * (tt & 15);
                float *d = (arr == 0 ? sm.G[sl] : (arr == 1 ? sm.kd[sl] : sm.gam[sl])) + e;
                *reinterpret_cast<float4 *>(d) = v;
            }
        };
        // ---- (16-bit activations) V of chunk c: thread tt convolves value channel tt
        //      of the head over the chunk's rows (kernel 4, SiLU, tf32 rounding, the
        //      front end's arithmetic for q and k) from the staged pre-conv rows and, in
        //      the first chunk of a sequence, the initial conv window.  Written as V^T
        //      (rows = value channels, columns = tokens) in the K-major 128-byte-swizzled
        //      layout, four tokens per float4; rows past the chunk's end are zero.
        //      M of the summary pass ignores V and skips the arithmetic.
        const int Cd = (2 * p.Hk + p.Hv) * kD;
        const int cv = 2 * p.Hk * kD + h * kD + tt; // this thread's qkv channel
        float4 cw = make_float4(0.f, 0.f, 0.f, 0.f);
        if constexpr (kVConv)
            cw = __ldg(reinterpret_cast<const float4 *>(p.conv_w) + cv);
        uint32_t phvx = 0;
        auto vconv = [&](int c) {
            bool good = waitp(smem_u32(&sm.bar_vx), phvx);       // the pre-conv rows of chunk c
            good = (c < 1 || waitq(bar_m1, (c - 1) & 1)) && good; // MMA 1 of chunk c - 1 has read V
            if (good && !mpart) {
                // four quarters of 16 tokens: the quarter's 19 staged rows are loaded
                // before any arithmetic and its 16 outputs are independent; then four
                // float4 stores
                const __nv_bfloat16 *x = sm.Vx + tt;
                const int rows = rows_of(c);
                const T *iw = (const T *)p.init_conv + (int64_t)n * 3 * Cd + cv;
                float *vt = sm.V + 32 * tt;
#pragma unroll 1
                for (int qt = 0; qt < kC / 16; ++qt) {
                    float xr[19]; // rows t - 3 .. t + 15 of the quarter's tokens t
#pragma unroll
                    for (int i = 0; i < 19; ++i)
                        xr[i] = to_f(x[(16 * qt + i) * kD]);
                    if (qt == 0 && cb + c == 0) { // taps before the sequence: the initial window
#pragma unroll
                        for (int i = 0; i < 3; ++i)
                            xr[i] = p.init_conv ? to_f(iw[i * Cd]) : 0.f;
                    }
                    float o[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float acc = cw.x * xr[i];
                        acc = fmaf(cw.y, xr[i + 1], acc);
                        acc = fmaf(cw.z, xr[i + 2], acc);
                        acc = fmaf(cw.w, xr[i + 3], acc);
                        o[i] = tf32_rna(siluf_(acc));
                        // rows past the end of a partial chunk: zero (a branch uniform
                        // over the CTA; a select around the SiLU measured far slower)
                        if (rows < kC && 16 * qt + i >= rows)
                            o[i] = 0.f;
                    }
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) { // tokens 16 qt + 4 q4 .. + 3
                        const int t4 = 16 * qt + 4 * q4;
                        *reinterpret_cast<float4 *>(vt + (t4 >> 5) * (kD * 32) + 4 * (((t4 & 31) >> 2) ^ (tt & 7))) =
                            make_float4(o[4 * q4], o[4 * q4 + 1], o[4 * q4 + 2], o[4 * q4 + 3]);
                    }
                }
            }
            fence_proxy_async_smem();
            if (group_sync_or(kBarT, kTeam, !good || *abort_flag))
                return false;
            if (tt == 0) {
                mbar_arrive(bar_v);                  // V of chunk c, for MMA 1
                mbar_arrive(smem_u32(&sm.bar_vxf)); // the staged rows may take chunk c + 1
            }
            return true;
        };
        uint32_t phqk = 0;
        float4 gv = load_gt(0);
        // ---- the gate record of chunk c into slot c mod 4 (the state group's
        //      S *= gamma_C, O *= gamma and U pass and P read it).  Slot c mod 4 last
        //      held chunk c - 4, whose readers are all done: this runs after P of
        //      chunk c - 1, which waited for MMA 3 of chunk c - 2 and so for the
        //      state group's U pass of that chunk.
        auto gates = [&](int c) {
            put_gt(gv, c & 3);
            gv = load_gt(c + 1);
            group_sync(kBarT, kTeam); // the gates are in
            if (tt == 0)
                mbar_arrive(bar_pT(c)); // gates of chunk c
        };
        // Order: the gates of chunk c + 1, then its V, as soon as P of chunk c is
        // out.  The state group's S *= gamma_C of a chunk needs only its gates, so
        // the v conv never delays it; MMA 1 of chunk c + 1 waits for V only at
        // MMA 2b, a whole MMA 2 later.
        if (nchunks > 0) {
            gates(0);
            if constexpr (kVConv)
                ok = vconv(0);
        }
        for (int c = 0; ok && c < nchunks; ++c) {
            const int sl = c & 3;
            // ---- P[r][s] = e^{G_r - G_s} QK[r][s] in place, tf32 (the Q K^T rows are
            //      0 for s > r; the clamp keeps the unused upper triangle finite); the
            //      summary pass has no O and no P
            bool good = summary || waitp(bar_qk, phqk);
            if (good && !summary) {
                float4 x[6];
#pragma unroll
                for (int jj = 0; jj < 6; ++jj)
                    x[jj] = *reinterpret_cast<const float4 *>(sm.P + tr.o(jj));
#pragma unroll
                for (int jj = 0; jj < 6; ++jj) {
                    const float Gr = sm.G[sl][tr.r(jj)];
                    const float4 Gc = *reinterpret_cast<const float4 *>(&sm.G[sl][tr.c(jj)]);
                    *reinterpret_cast<float4 *>(sm.P + tr.o(jj)) =
                        tf32_rna(make_float4(x[jj].x * __expf(fminf(Gr - Gc.x, 0.f)),
                                             x[jj].y * __expf(fminf(Gr - Gc.y, 0.f)),
                                             x[jj].z * __expf(fminf(Gr - Gc.z, 0.f)),
                                             x[jj].w * __expf(fminf(Gr - Gc.w, 0.f))));
                }
            }
            fence_proxy_async_smem();
            if (group_sync_or(kBarT, kTeam, !good || *abort_flag)) {
                ok = false;
                break;
            }
            if (tt == 0 && !summary)
                mbar_arrive(bar_pP); // P of chunk c
            if (c + 1 < nchunks) {
                gates(c + 1);
                if constexpr (kVConv) {
                    if (!vconv(c + 1)) {
                        ok = false;
                        break;
                    }
                }
            }
        }
        if (!ok)
            *abort_flag = 1;
    } else if (warp == kWarpMma) {
        // ==================================================== MMA issue
        // The whole warp runs this loop in uniform control flow (so the
        // descriptor arithmetic stays warp-uniform) and the elected lane issues
        // the MMAs and commits; every decision is taken by all lanes alike.
        if (nchunks > 0) {
            const uint32_t is = elect_one();
            auto all = [&](bool g) { return __all_sync(0xffffffffu, g) != 0; };
            // V: MN-major from TMA, or V^T K-major from the prep team (128 rows a block)
            const uint64_t dV = kVConv ? sdesc_sw128(smem_u32(sm.V), 16, 1024)
                                       : sdesc_sw128_b32(smem_u32(sm.V), kC * 128, 512);
            auto aV = [&](int s) -> uint64_t {
                return kVConv ? dV + (uint64_t)((((s >> 2) * kD * 128) + (s & 3) * 32) >> 4) : dV + s * 64;
            };
            const uint64_t dK = sdesc_sw128_b32(smem_u32(sm.K), kC * 128, 512);
            const uint64_t dKQ = sdesc_sw128(smem_u32(sm.KQ), 16, 1024);
            const uint64_t dP0 = sdesc_sw128(smem_u32(sm.P), 16, 1024);
            const uint64_t dP1 = sdesc_sw128(smem_u32(sm.P + 2048), 16, 1024);
            auto tb0 = [&](int c) { return sdesc_sw128(smem_u32(sm.Tb[c & 1]), 16, 1024); };
            auto tb1 = [&](int c) { return sdesc_sw128(smem_u32(sm.Tb[c & 1] + 2048), 16, 1024); };
            auto tg0 = [&](int c) { return sdesc_sw128(smem_u32(sm.Tg[c & 1]), 16, 1024); };
            auto tg1 = [&](int c) { return sdesc_sw128(smem_u32(sm.Tg[c & 1] + 2048), 16, 1024); };
            constexpr uint32_t id64 = idesc_tf32(128, 64, true, false);    // MMA 1 (A MN-major)
            constexpr uint32_t id32 = idesc_tf32(128, 32, true, false);
            constexpr uint32_t id128 = idesc_tf32(128, 128, false, false); // MMA 2
            constexpr uint32_t idT64 = idesc_tf32(128, 64, false, false);  // MMA 2b, MMA 3 O
            constexpr uint32_t idT32 = idesc_tf32(128, 32, false, false);
            constexpr uint32_t idS = idesc_tf32(128, 128, false, true);    // MMA 3 S (B MN-major)
            constexpr uint32_t idV64 = kVConv ? idT64 : id64, idV32 = kVConv ? idT32 : id32; // MMA 1
            uint32_t phv = 0, phkm = 0, phq = 0, phu = 0, phP = 0, ph2 = 0, phk = 0;
            // MMA 1 of chunk c: U~^T into U_(c%2).  K steps 0..3 run over column
            // block 0 of the T tile (N = 64), 4..7 over block 1 (rows 32..63)
            auto mma1 = [&](int c) {
                const uint32_t dU = tmem + ((c & 1) ? kColU1 : kColU0);
                const uint64_t b0 = tb0(c), b1 = tb1(c);
#pragma unroll 1
                for (int s = 0; s < 4; ++s)
                    mma_tf32_ss_if(dU, aV(s), b0 + 2 * s, idV64, s > 0, is);
#pragma unroll 1
                for (int s = 4; s < 8; ++s)
                    mma_tf32_ss_if(dU + 32, aV(s), b1 + 2 * (s - 4), idV32, 1, is);
                mma_commit_if(bar_m1, is);
            };
            // the inputs of MMA 1 of chunk c: its T diag(beta) tile and V (both by TMA);
            // the non-blocking form takes lane 0's view, so that all lanes agree
            auto m1_ready = [&](int c, bool block) {
                if (!block)
                    return __shfl_sync(0xffffffffu,
                                       (int)(mbar_test_wait(bar_tb(c), (c >> 1) & 1) &&
                                             mbar_test_wait(bar_v, phv)),
                                       0) != 0;
                bool g = waitq(bar_tb(c), (c >> 1) & 1);
                g = g && waitq(bar_v, phv);
                return all(g);
            };
            // MMA 1 of chunk c runs any time between MMA 3 of chunk c - 2 (the last
            // reader of its U buffer) and MMA 2b of chunk c (its first consumer): it is
            // issued as soon as its T diag(beta) tile and V are in, at the latest
            // (waiting for them) just before MMA 2b, so that neither the V loads nor
            // the prep team's v conv hold up MMA 2
            int m1_next = 0; // the chunk whose MMA 1 is issued next
            auto issue_m1 = [&](bool block) {
                if (!m1_ready(m1_next, block))
                    return false;
                phv ^= 1u;
                tc_fence_after();
                mma1(m1_next++);
                return true;
            };
            bool good = all(waitp(bar_u, phu)); // phase 0 of U: the initial state
            if (good)
                issue_m1(false);
            for (int c = 0; good && c < nchunks; ++c) {
                const uint32_t dXO = tmem + ((c & 1) ? kColX1 : kColX0);
                const uint32_t dU = tmem + ((c & 1) ? kColU1 : kColU0);
                // ---- MMA 2: [X^T | O^T] = S [K; Q]^T (A = the state in TMEM); the
                //      summary pass takes X^T alone (N = 64: the K rows of each block)
                good = summary || waitp(bar_q, phq);
                good = waitp(bar_kmaj, phkm) && good;
                if (c >= 2 && !summary)
                    good = ((c & 1) ? waitq(bar_of1, ((c >> 1) - 1) & 1)
                                    : waitq(bar_of0, ((c >> 1) - 1) & 1)) && good;
                if (!all(good))
                    break;
                tc_fence_after();
                const uint32_t id2 = summary ? idT64 : id128;
#pragma unroll 1
                for (int s = 0; s < kD / 8; ++s) {
                    const uint64_t ks = (uint64_t)((((s >> 2) * 2 * kC * 128) + (s & 3) * 32) >> 4);
                    mma_tf32_ts_if(dXO, tmem + kColS + 8 * s, dKQ + ks, id2, s > 0, is);
                }
                mma_commit_if(bar_m2, is);
                if (m1_next == c && !issue_m1(true)) {
                    good = false;
                    break;
                }
                // ---- MMA 2b: U^T = U~^T + X^T (-T diag(b gamma))^T (A = X^T in TMEM);
                //      its B tile landed with T diag(beta), which MMA 1 waited for
                good = waitp(bar_m2, ph2);
                if (!all(good))
                    break;
                tc_fence_after();
                {
                    // M of the summary pass has no values: U^T = X^T (-T diag(b gamma))^T
                    // alone, its first product overwriting U~^T
                    const uint64_t g0 = tg0(c), g1 = tg1(c);
#pragma unroll 1
                    for (int s = 0; s < 4; ++s)
                        mma_tf32_ts_if(dU, dXO + 8 * s, g0 + 2 * s, idT64, !mpart || s > 0, is);
#pragma unroll 1
                    for (int s = 4; s < 8; ++s)
                        mma_tf32_ts_if(dU + 32, dXO + 8 * s, g1 + 2 * (s - 4), idT32, 1, is);
                }
                mma_commit_if(bar_m2b(c), is);
                // ---- MMA 1 of the next chunk beside the U pass, if its inputs are in
                //      (its U buffer was last read by MMA 3 of chunk c - 1)
                if (m1_next == c + 1 && c + 1 < nchunks)
                    issue_m1(false);
                // ---- MMA 3: O^T += U^T P^T, S += (U diag(gamma_C/gamma))^T K (K MN-major)
                good = waitp(bar_u, phu);
                good = (summary || waitp(bar_pP, phP)) && good;
                good = waitp(bar_k, phk) && good;
                if (!all(good))
                    break;
                tc_fence_after();
                {
                    const uint32_t dO = dXO + 64;
                    if (!summary) {
#pragma unroll 1
                        for (int s = 0; s < 4; ++s)
                            mma_tf32_ts_if(dO, dU + 8 * s, dP0 + 2 * s, idT64, 1, is);
#pragma unroll 1
                        for (int s = 4; s < 8; ++s)
                            mma_tf32_ts_if(dO + 32, dU + 8 * s, dP1 + 2 * (s - 4), idT32, 1, is);
                    }
#pragma unroll 1
                    for (int s = 0; s < kC / 8; ++s)
                        mma_tf32_ts_if(tmem + kColS, dXO + 8 * s, dK + s * 64, idS, 1, is);
                }
                mma_commit_if(bar_m3, is);
                if (m1_next == c + 1 && c + 1 < nchunks)
                    issue_m1(false);
            }
            ok = good;
            // let every MMA issued so far finish before the CTA releases TMEM
            if (!ok) {
                *abort_flag = 1;
                uint32_t phx = 0;
                const uint32_t bar_x = smem_u32(&sm.bar_fin);
                mma_commit_if(bar_x, is);
                mbar_wait_bounded(bar_x, phx, kWaitLimit);
            }
        }
    } else {
        // ==================================================== TMA issue
        if (lane == 0 && nchunks > 0) {
            // loads armed on v, q, k, kmaj, tb (parity 0, 1), qk, z, vx
            uint32_t cnt[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
            const uint32_t bar_vx = smem_u32(&sm.bar_vx), bar_vxf = smem_u32(&sm.bar_vxf);
            const uint32_t lbar[9] = {bar_v,  bar_q,  bar_k, bar_kmaj, bar_tb(0),
                                      bar_tb(1), bar_qk, bar_z, bar_vx};
            // nb 32-column boxes of 64 rows at x0 + 32 b, row t0, block b landing at dst + b * bstride
            // (each load also asks L2 for the next chunk's boxes of the same stream, so
            // that a long sequence's loads, which miss L2, do not wait on DRAM)
            auto tile = [&](int which, float *dst, const CUtensorMap *m, int x0, int64_t t0, int nb,
                            int bstride) {
                mbar_arrive_expect_tx(lbar[which], (uint32_t)(nb * kC * 32 * sizeof(float)));
                for (int b = 0; b < nb; ++b)
                    tma_load_2d(smem_u32(dst + b * bstride), m, x0 + 32 * b, (int)t0, lbar[which]);
                if (t0 + kC < end)
                    for (int b = 0; b < nb; ++b)
                        tma_prefetch_2d(m, x0 + 32 * b, (int)(t0 + kC));
                ++cnt[which];
            };
            auto t_of = [&](int c) { return start + (int64_t)c * kC; };
            // the Q K^T rows of chunk c as a triangular tile: block 0 (64 rows) and the
            // lower half of block 1
            auto qktile = [&](int c) {
                if (summary)
                    return;
                mbar_arrive_expect_tx(bar_qk, (uint32_t)(kTriFloats * sizeof(float)));
                tma_load_2d(smem_u32(sm.P), &maps.kq, xkk, (int)t_of(c), bar_qk);
                tma_load_2d(smem_u32(sm.P + 2048), &maps.kq32, xkk + 32, (int)(t_of(c) + 32), bar_qk);
                if (c + 1 < nchunks) {
                    tma_prefetch_2d(&maps.kq, xkk, (int)t_of(c + 1));
                    tma_prefetch_2d(&maps.kq32, xkk + 32, (int)(t_of(c + 1) + 32));
                }
                ++cnt[6];
            };
            // T diag(beta) and -T diag(beta gamma) of chunk c: one box of 96 rows each
            // (triangular tiles), one barrier
            const int chunk0 = __ldg(p.ws_offs + n) + cb; // global index of this segment's first chunk
            auto tbtile = [&](int c) {
                mbar_arrive_expect_tx(bar_tb(c), (uint32_t)(2 * kTriFloats * sizeof(float)));
                const int row = (int)(((int64_t)(chunk0 + c) * p.Hv + h) * 2 * 96);
                tma_load_2d(smem_u32(sm.Tb[c & 1]), &maps.tb, 0, row, bar_tb(c));
                tma_load_2d(smem_u32(sm.Tg[c & 1]), &maps.tb, 0, row + 96, bar_tb(c));
                ++cnt[4 + (c & 1)];
            };
            // the z rows of a chunk: one 128-column box of 64 rows
            auto ztile = [&](int c) {
                if (kZTile && !summary) {
                    mbar_arrive_expect_tx(bar_z, (uint32_t)(kC * kD * sizeof(T)));
                    tma_load_2d(smem_u32(sm.Z), &maps.z, h * kD, (int)t_of(c), bar_z);
                    if (c + 1 < nchunks)
                        tma_prefetch_2d(&maps.z, h * kD, (int)t_of(c + 1));
                    ++cnt[7];
                }
            };
            // the pre-conv v rows t0 - 3 .. t0 + 63 of a chunk (16-bit activations;
            // rows before the first token read as zero and are not used)
            auto vxtile = [&](int c) {
                mbar_arrive_expect_tx(bar_vx, (uint32_t)((kC + 3) * kD * sizeof(T)));
                tma_load_2d(smem_u32(sm.Vx), &maps.vx, 2 * p.Hk * kD + h * kD, (int)(t_of(c) - 3), bar_vx);
                if (c + 1 < nchunks)
                    tma_prefetch_2d(&maps.vx, 2 * p.Hk * kD + h * kD, (int)(t_of(c + 1) - 3));
                ++cnt[8];
            };
            constexpr int kBlkV = kC * 32, kBlkQ = 2 * kC * 32;
            tbtile(0);
            if (kVConv)
                vxtile(0);
            else
                tile(0, sm.V, &maps.v, xv, t_of(0), 4, kBlkV);
            tile(3, sm.KQ, &maps.kmaj, xq, t_of(0), 4, kBlkQ);        // rows 0..63 of KQ
            if (!summary)
                tile(1, sm.KQ + kC * 32, &maps.q, xq, t_of(0), 4, kBlkQ); // rows 64..127
            qktile(0);
            tile(2, sm.K, &maps.k, xq, t_of(0), 4, kBlkV);
            ztile(0);
            if (nchunks > 1)
                tbtile(1);
            // six event streams, each served in chunk order as it completes
            // Every stream polls a barrier whose next phase cannot complete before
            // the reload it triggers: a parity test cannot then miss a phase.  (MMA 1
            // completions are polled only where the TMA warp feeds V; with the v conv
            // on the prep team two MMA 1 phases can complete between two polls.)
            int ib = 0, i1 = kVConv ? nchunks : 0, i2 = 0, i3 = 0, iz = kZTile && !summary ? 0 : nchunks;
            int ix = kVConv ? 0 : nchunks;
            long long t_last = clock64();
            while (ib < nchunks || i1 < nchunks || i2 < nchunks || i3 < nchunks || iz < nchunks ||
                   ix < nchunks) {
                bool prog = false;
                // the prep team has convolved chunk ix from the staged rows
                if (ix < nchunks && mbar_test_wait(bar_vxf, ix & 1)) {
                    if (ix + 1 < nchunks)
                        vxtile(ix + 1);
                    ++ix;
                    prog = true;
                }
                // the epilogue of chunk iz has released the z tile
                if (iz < nchunks && mbar_test_wait(bar_zf, iz & 1)) {
                    if (iz + 1 < nchunks)
                        ztile(iz + 1);
                    ++iz;
                    prog = true;
                }
                // MMA 2b of chunk ib is done, so MMA 1 (issued before it) and the prep
                // team (whose -T diag(beta gamma) MMA 2b waited for) have read T diag(beta)
                // of chunk ib: its slot takes chunk ib + 2
                if (ib < nchunks && mbar_test_wait(bar_m2b(ib), (ib >> 1) & 1)) {
                    if (ib + 2 < nchunks)
                        tbtile(ib + 2);
                    ++ib;
                    prog = true;
                }
                if (i1 < nchunks && mbar_test_wait(bar_m1, i1 & 1)) { // V is free
                    if (i1 + 1 < nchunks && !kVConv)
                        tile(0, sm.V, &maps.v, xv, t_of(i1 + 1), 4, kBlkV);
                    ++i1;
                    prog = true;
                }
                if (i2 < nchunks && mbar_test_wait(bar_m2, i2 & 1)) { // K (K-major) and Q are free
                    if (i2 + 1 < nchunks) {
                        tile(3, sm.KQ, &maps.kmaj, xq, t_of(i2 + 1), 4, kBlkQ);
                        if (!summary)
                            tile(1, sm.KQ + kC * 32, &maps.q, xq, t_of(i2 + 1), 4, kBlkQ);
                    }
                    ++i2;
                    prog = true;
                }
                if (i3 < nchunks && mbar_test_wait(bar_m3, i3 & 1)) { // P and K (MN-major) are free
                    if (i3 + 1 < nchunks) {
                        qktile(i3 + 1);
                        tile(2, sm.K, &maps.k, xq, t_of(i3 + 1), 4, kBlkV);
                    }
                    ++i3;
                    prog = true;
                }
                if (prog) {
                    t_last = clock64();
                } else if (clock64() - t_last > p.wait_limit || *abort_flag) {
                    ok = false;
                    break;
                } else {
                    __nanosleep(16); // leave the issue slots to the working warps
                }
            }
            // every armed load lands before the CTA exits
#pragma unroll
            for (int b = 0; b < 9; ++b)
                if (cnt[b] > 0)
                    mbar_wait_bounded(lbar[b], (cnt[b] - 1) & 1, kWaitLimit);
            if (!ok)
                *abort_flag = 1;
        }
    }

    if (tid == 0)
        bulk_wait_all(); // the epilogue's y stores are complete
    ok = !__syncthreads_or(!ok); // one verdict for the whole CTA
    if (!ok) {
        if (tid == 0 && p.ws_err != nullptr)
            atomicOr(p.ws_err, 1u);
    } else if (warp < kSG / 32 &&
               (summary || (seg == p.segments - 1 && p.final_state != nullptr))) {
        // the final state (last segment of the output pass) or the segment's R or M
        const int lq = warp & 3, hf = warp >> 2, vch = lq * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(lq * 32) << 16);
        float *dst = (summary ? seg_state(mpart ? 1 : 0, seg) + (size_t)vch * kD
                              : p.final_state + (((size_t)n * p.Hv + h) * kD + vch) * kD) + 64 * hf;
        // the summary pass has not waited for the last MMA 3 here (the TMA warp has,
        // before the barrier above)
        tc_fence_after();
#pragma unroll
        for (int bk = 0; bk < 2; ++bk) {
            float v[32];
            tmem_ld32(tl + kColS + 64 * hf + 32 * bk, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4 *>(dst + bk * 32 + i) =
                    make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------ segment chain
//
// The state entering each segment of a split sequence: with S(0) the call's
// initial state (zero if none), S(s) = S(s - 1) M(s - 1) + R(s - 1) for
// s = 1 .. P - 1, the affine map of segment s - 1 applied to the state entering
// it.  FP32 on the CUDA cores: one CTA per (value head, sequence), each of its
// 256 threads an 8 x 8 block of every 128 x 128 x 128 product; the left factor
// sits transposed in shared memory so that both operands load as float4.
constexpr int kCombThreads = 256;
constexpr size_t kCombSmem = 2 * kD * kD * sizeof(float);

__global__ void __launch_bounds__(kCombThreads)
seg_combine_kernel(PrefillArgs p) {
    extern __shared__ __align__(16) float comb_smem[];
    float *At = comb_smem;           // At[k][i] = S(s - 1)[i][k]
    float *Ms = comb_smem + kD * kD; // M(s - 1)[k][j]
    const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x;
    const int ty = tid >> 4, tx = tid & 15; // rows 8 ty .. 8 ty + 7, columns 8 tx .. 8 tx + 7
    const int64_t units = (int64_t)p.batch * (p.segments - 1) * p.Hv;
    auto st = [&](int r, int sg) {
        return p.ws_seg + (((int64_t)r * units + ((int64_t)n * (p.segments - 1) + sg) * p.Hv + h) * kD) * kD;
    };
    const float *S0 = p.init_state ? p.init_state + ((int64_t)n * p.Hv + h) * kD * kD : nullptr;
    for (int e = tid; e < kD * kD; e += kCombThreads)
        At[(e % kD) * kD + e / kD] = S0 ? S0[e] : 0.f;
    for (int sg = 1; sg < p.segments; ++sg) {
        const float *M = st(1, sg - 1), *R = st(0, sg - 1);
        float *out = st(2, sg - 1);
        for (int e = 4 * tid; e < kD * kD; e += 4 * kCombThreads)
            *reinterpret_cast<float4 *>(Ms + e) = *reinterpret_cast<const float4 *>(M + e);
        __syncthreads(); // Ms and At (the previous step's result) are in
        float acc[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 r0 = *reinterpret_cast<const float4 *>(R + (8 * ty + i) * kD + 8 * tx);
            const float4 r1 = *reinterpret_cast<const float4 *>(R + (8 * ty + i) * kD + 8 * tx + 4);
            acc[i][0] = r0.x; acc[i][1] = r0.y; acc[i][2] = r0.z; acc[i][3] = r0.w;
            acc[i][4] = r1.x; acc[i][5] = r1.y; acc[i][6] = r1.z; acc[i][7] = r1.w;
        }
#pragma unroll 4
        for (int k = 0; k < kD; ++k) {
            const float4 a0 = *reinterpret_cast<const float4 *>(At + k * kD + 8 * ty);
            const float4 a1 = *reinterpret_cast<const float4 *>(At + k * kD + 8 * ty + 4);
            const float4 b0 = *reinterpret_cast<const float4 *>(Ms + k * kD + 8 * tx);
            const float4 b1 = *reinterpret_cast<const float4 *>(Ms + k * kD + 8 * tx + 4);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    acc[i][jj] = fmaf(a[i], b[jj], acc[i][jj]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float *o = out + (8 * ty + i) * kD + 8 * tx;
            *reinterpret_cast<float4 *>(o) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
            *reinterpret_cast<float4 *>(o + 4) = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
        }
        __syncthreads(); // every thread is done reading At and Ms
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
                At[(8 * tx + jj) * kD + 8 * ty + i] = acc[i][jj];
    }
}

template <typename T> cudaError_t launch_chunk_t(const PrefillArgs &p, cudaStream_t s) {
    const size_t smem = sizeof(ChunkSmem);
    cudaError_t e = cudaFuncSetAttribute(chunk_prefill_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    ChunkMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (p.N > 0) {
        const uint64_t N = (uint64_t)p.N, F = sizeof(float);
        const uint64_t qkw = 2ull * p.Hk * kD, kqw = (uint64_t)p.Hk * kC;
        const uint64_t tb_rows = (uint64_t)((p.N + kC - 1) / kC + p.batch) * p.Hv * 2 * 96;
        const uint64_t Cd = (uint64_t)(2 * p.Hk + p.Hv) * kD;
        const bool okm =
            (sizeof(T) == 2
                 ? encode_2d(&maps.vx, p.qkv, Cd, N, Cd * sizeof(T), kD, kC + 3, CU_TENSOR_MAP_SWIZZLE_NONE,
                             CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)
                 : encode_2d(&maps.v, p.ws_v, (uint64_t)p.Hv * kD, N, (uint64_t)p.Hv * kD * F, 32, kC,
                             CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B)) &&
            encode_2d(&maps.k, (const float *)p.ws_qk + (size_t)p.Hk * kD, (uint64_t)p.Hk * kD, N,
                      qkw * F, 32, kC, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B) &&
            encode_2d(&maps.q, p.ws_qk, (uint64_t)p.Hk * kD, N, qkw * F, 32, kC,
                      CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_2d(&maps.kmaj, (const float *)p.ws_qk + (size_t)p.Hk * kD, (uint64_t)p.Hk * kD, N,
                      qkw * F, 32, kC, CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_2d(&maps.kq, p.ws_kq, kqw, N, kqw * F, 32, kC, CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_2d(&maps.kq32, p.ws_kq, kqw, N, kqw * F, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_2d(&maps.tb, p.ws_tb, 32, tb_rows, 32 * F, 32, 96, CU_TENSOR_MAP_SWIZZLE_128B) &&
            (sizeof(T) != 2 ||
             (encode_2d(&maps.z, p.z, (uint64_t)p.Hv * kD, N, (uint64_t)p.Hv * kD * sizeof(T), kD, kC,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) &&
              encode_2d(&maps.y, p.y, (uint64_t)p.Hv * kD, N, (uint64_t)p.Hv * kD * sizeof(T), kD, kC,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)));
        if (!okm)
            return cudaErrorInvalidValue;
    }
    if (p.segments > 1) {
        // the split: (M, R) of every segment but the last, then the chained start
        // states, then the output pass over all segments
        PrefillArgs ps = p;
        ps.seg_pass = 1;
        chunk_prefill_kernel<T><<<dim3(p.Hv, p.batch, 2 * (p.segments - 1)), kThreads, smem, s>>>(ps, maps);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
        if ((e = cudaFuncSetAttribute(seg_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kCombSmem)) != cudaSuccess)
            return e;
        seg_combine_kernel<<<dim3(p.Hv, p.batch), kCombThreads, kCombSmem, s>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
    }
    chunk_prefill_kernel<T><<<dim3(p.Hv, p.batch, p.segments), kThreads, smem, s>>>(p, maps);
    return cudaGetLastError();
}

} // namespace

size_t kq_workspace_bytes(int Hk, int64_t N) { return (size_t)N * Hk * kC * sizeof(float); }

// T diag(beta) and -T diag(beta gamma) tiles: two per (chunk, value head), 96
// rows of 32 floats each; every sequence adds at most one partial chunk to the
// N / 64 full ones.
size_t tb_workspace_bytes(int Hv, int64_t N, int batch) {
    return (size_t)((N + kC - 1) / kC + batch) * Hv * 2 * 96 * 32 * sizeof(float);
}

// Gate records: one per (chunk, value head).
size_t gt_workspace_bytes(int Hv, int64_t N, int batch) {
    return (size_t)((N + kC - 1) / kC + batch) * Hv * kGateRec * sizeof(float);
}

// K K^T triangular tiles: one per (chunk, q/k head).
size_t kk_workspace_bytes(int Hk, int64_t N, int batch) {
    return (size_t)((N + kC - 1) / kC + batch) * Hk * kTriFloats * sizeof(float);
}

cudaError_t launch_chunk_offsets(const PrefillArgs &p, cudaStream_t s) {
    // no tokens: no workspace (the offsets and status words have no home) and
    // no chunk to count; the chunk kernel then only passes the states through
    if (p.batch == 0 || p.N == 0)
        return cudaSuccess;
    chunk_offsets_kernel<<<1, 1024, 0, s>>>(p.cu, p.batch, p.N, p.ws_offs, p.ws_err);
    return cudaGetLastError();
}

cudaError_t launch_chunk_prefill(const PrefillArgs &p, cudaStream_t s) {
    if (p.batch == 0)
        return cudaSuccess;
    return p.bf16 ? launch_chunk_t<__nv_bfloat16>(p, s) : launch_chunk_t<float>(p, s);
}

} // namespace gdn
