// gdn_tri.cuh -- the 64 x 64 unit lower-triangular inverse T = (I + A)^-1 of
// the chunked gated delta rule (A[r][s] = beta_r exp(G_r - G_s) k_r . k_s for
// s < r; the chunked form of the Gated DeltaNet recurrence, "Qwen3.8-2.4T-A95B
// vs Inkling", component table, Gated DeltaNet row), in FP32 on the CUDA cores
// of 128 threads, in place in a shared-memory tile.
//
// Tile layout ("triangular tile"): the K-major, 128-byte-swizzled layout of a
// 64 x 64 tile in 32-float column blocks with its zero quadrant (rows 0..31,
// columns 32..63) left out: column block 0 holds rows 0..63 (2048 floats),
// block 1 rows 32..63 only (1024 floats).  Element (r, c) sits at
// 32 r + 4 ((c / 4) xor (r mod 8)) + c mod 4 for c < 32 and at
// 1024 + 32 r + 4 (((c - 32) / 4) xor (r mod 8)) + c mod 4 for c >= 32.  Read as
// 96 rows of 128 bytes (block 0 rows, then block 1 rows 32..63), each row's
// 16-byte chunks are XOR-swizzled by the row index mod 8: the pattern a TMA
// load with 128-byte swizzle writes.
#pragma once

#include <stdint.h>

namespace gdn {

constexpr int kTriFloats = 3 * 1024;

// Barrier over the `n` threads of one group (named barrier `id`).
__device__ __forceinline__ void group_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// The six float4s of a triangular tile that thread tt (0..127) of a group
// handles in an elementwise pass: rows tt / 8 + 16 jj (jj = 0..3, column block
// 0, columns 4 (tt % 8) .. + 3) and 32 + tt / 8 + 16 (jj - 4) (jj = 4, 5, block
// 1, columns 32 + 4 (tt % 8) .. + 3).  16 jj keeps r mod 8, so the swizzle term
// is one constant per thread.
struct TriThread {
    int trow, tcol, tbase;
    __device__ __forceinline__ explicit TriThread(int tt)
        : trow(tt >> 3), tcol(4 * (tt & 7)), tbase((tt >> 3) * 32 + (((tt & 7) ^ ((tt >> 3) & 7)) << 2)) {}
    __device__ __forceinline__ int r(int jj) const { return jj < 4 ? trow + 16 * jj : 32 + trow + 16 * (jj - 4); }
    __device__ __forceinline__ int c(int jj) const { return jj < 4 ? tcol : 32 + tcol; }
    __device__ __forceinline__ int o(int jj) const { return tbase + (jj < 4 ? 512 * jj : 1024 + 512 * (jj - 2)); }
};

// Wk holds A (strictly lower triangular; the diagonal and above are ignored)
// and receives T = (I + A)^-1, by block doubling: the four 16 x 16 diagonal
// blocks by forward substitution, then the joins at 32 and at 64
// (T21 = -T22 A21 T11).  Threads tt = 0..127 of a group whose named barrier
// is `bar`; every thread of the group calls it.  The loops are unrolled: each
// step is a short dependency chain, so the latency of one hides the next.
__device__ __forceinline__ void tri_invert(float *Wk, int tt, int bar) {
    // ---- T = (I + A)^-1 in place, by block doubling.  Level 1: the four
    //      16 x 16 diagonal blocks by forward substitution, one column per
    //      thread (threads 0..63)
    {
        // warp 0: blocks 0, 1 (column block 0); warp 1: blocks 2, 3 (block 1,
        // whose rows 32.. sit at 1024 + 32 r); lanes 0..15 / 16..31 take the
        // two blocks, R' = 0 / 16 within the column block
        const int cl = tt & 15, Rp = 16 * ((tt >> 4) & 1), R = 32 * (tt >> 5) + Rp;
        const float *blk = Wk + 1024 * (tt >> 5) + R * 32;
        float x[16];
        if (tt < 64) {
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                for (int m = 0; m < (r + 3) / 4; ++m) {
                    const float4 a = *reinterpret_cast<const float4 *>(
                        blk + r * 32 + ((((Rp >> 2) + m) ^ (r & 7)) << 2));
                    const float av4[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (4 * m + e < r) {
                            if (e & 1)
                                acc1 = fmaf(av4[e], x[4 * m + e], acc1);
                            else
                                acc0 = fmaf(av4[e], x[4 * m + e], acc0);
                        }
                }
                x[r] = r < cl ? 0.f : (r == cl ? 1.f : -(acc0 + acc1));
            }
        }
        group_sync(bar, 128); // every diagonal block of A has been read
        if (tt < 64) {
            float *dst = Wk + 1024 * (tt >> 5) + R * 32 + ((Rp + cl) & 3);
#pragma unroll
            for (int r = 0; r < 16; ++r)
                dst[r * 32 + ((((Rp + cl) >> 2) ^ (r & 7)) << 2)] = x[r];
        }
    }
    group_sync(bar, 128);
    // ---- level 2: join the 16-blocks of each 32-block p (warps 0, 1: p = 0
    //      in column block 0; warps 2, 3: p = 1 in block 1):
    //      T21 = -T22 (A21 T11); thread: rows r0, r0 + 1, columns c0, c0 + 1;
    //      element (32 p + i, 32 p + j) at base + i * 32 + swizzle(i, j)
    {
        const int pb = tt >> 6, q = tt & 63;
        const int r0 = 2 * (q >> 3), c0 = 2 * (q & 7);
        float *base = Wk + 1024 * pb + 32 * pb * 32;
        auto at = [&](int i, int jc) { return base + i * 32 + (((jc >> 2) ^ (i & 7)) << 2) + (jc & 3); };
        float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 a0 = *reinterpret_cast<const float4 *>(at(16 + r0, 4 * m));
            const float4 a1 = *reinterpret_cast<const float4 *>(at(17 + r0, 4 * m));
            const float a0v[4] = {a0.x, a0.y, a0.z, a0.w}, a1v[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 t2 = *reinterpret_cast<const float2 *>(at(4 * m + e, c0));
                y00 = fmaf(a0v[e], t2.x, y00); y01 = fmaf(a0v[e], t2.y, y01);
                y10 = fmaf(a1v[e], t2.x, y10); y11 = fmaf(a1v[e], t2.y, y11);
            }
        }
        group_sync(bar, 128); // A21 is read: Y takes its place
        *reinterpret_cast<float2 *>(at(16 + r0, c0)) = make_float2(y00, y01);
        *reinterpret_cast<float2 *>(at(17 + r0, c0)) = make_float2(y10, y11);
        group_sync(bar, 128);
        float x00 = 0.f, x01 = 0.f, x10 = 0.f, x11 = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 a0 = *reinterpret_cast<const float4 *>(at(16 + r0, 16 + 4 * m));
            const float4 a1 = *reinterpret_cast<const float4 *>(at(17 + r0, 16 + 4 * m));
            const float a0v[4] = {a0.x, a0.y, a0.z, a0.w}, a1v[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 t2 = *reinterpret_cast<const float2 *>(at(16 + 4 * m + e, c0));
                x00 = fmaf(a0v[e], t2.x, x00); x01 = fmaf(a0v[e], t2.y, x01);
                x10 = fmaf(a1v[e], t2.x, x10); x11 = fmaf(a1v[e], t2.y, x11);
            }
        }
        group_sync(bar, 128); // Y is read: T21 takes its place
        *reinterpret_cast<float2 *>(at(16 + r0, c0)) = make_float2(-x00, -x01);
        *reinterpret_cast<float2 *>(at(17 + r0, c0)) = make_float2(-x10, -x11);
    }
    group_sync(bar, 128);
    // ---- level 3: join the two 32-blocks: T21 = -T22 (A21 T11); thread:
    //      rows r0, r0 + 1, columns c0 .. + 3 of the 32 x 32 products.  A21,
    //      T11 and Y sit in column block 0 (offset r * 32 + chunk ^ (r & 7)),
    //      T22 in block 1 (rows 32..63)
    {
        const int r0 = 2 * (tt >> 3), q0 = tt & 7; // columns c0 = 4 q0
        const float *Ar0 = Wk + (32 + r0) * 32, *Ar1 = Ar0 + 32;   // rows 32 + r0, + 1
        const float *Br0 = Wk + 2048 + r0 * 32, *Br1 = Br0 + 32;   // block 1 rows
        const int x0 = r0 & 7, x1 = (r0 + 1) & 7;
        float y[2][4] = {};
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const float4 a0 = *reinterpret_cast<const float4 *>(Ar0 + ((m ^ x0) << 2));
            const float4 a1 = *reinterpret_cast<const float4 *>(Ar1 + ((m ^ x1) << 2));
            const float a0v[4] = {a0.x, a0.y, a0.z, a0.w}, a1v[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = 4 * m + e; // T11 row i, columns c0 .. + 3
                const float4 t4 =
                    *reinterpret_cast<const float4 *>(Wk + i * 32 + ((q0 ^ (i & 7)) << 2));
                y[0][0] = fmaf(a0v[e], t4.x, y[0][0]); y[0][1] = fmaf(a0v[e], t4.y, y[0][1]);
                y[0][2] = fmaf(a0v[e], t4.z, y[0][2]); y[0][3] = fmaf(a0v[e], t4.w, y[0][3]);
                y[1][0] = fmaf(a1v[e], t4.x, y[1][0]); y[1][1] = fmaf(a1v[e], t4.y, y[1][1]);
                y[1][2] = fmaf(a1v[e], t4.z, y[1][2]); y[1][3] = fmaf(a1v[e], t4.w, y[1][3]);
            }
        }
        group_sync(bar, 128); // A21 is read: Y takes its place
        float *Yr0 = Wk + (32 + r0) * 32 + ((q0 ^ x0) << 2);
        float *Yr1 = Wk + (33 + r0) * 32 + ((q0 ^ x1) << 2);
        *reinterpret_cast<float4 *>(Yr0) = make_float4(y[0][0], y[0][1], y[0][2], y[0][3]);
        *reinterpret_cast<float4 *>(Yr1) = make_float4(y[1][0], y[1][1], y[1][2], y[1][3]);
        group_sync(bar, 128);
        float x[2][4] = {};
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const float4 a0 = *reinterpret_cast<const float4 *>(Br0 + ((m ^ x0) << 2));
            const float4 a1 = *reinterpret_cast<const float4 *>(Br1 + ((m ^ x1) << 2));
            const float a0v[4] = {a0.x, a0.y, a0.z, a0.w}, a1v[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = 32 + 4 * m + e; // Y row i - 32, columns c0 .. + 3
                const float4 t4 =
                    *reinterpret_cast<const float4 *>(Wk + i * 32 + ((q0 ^ (i & 7)) << 2));
                x[0][0] = fmaf(a0v[e], t4.x, x[0][0]); x[0][1] = fmaf(a0v[e], t4.y, x[0][1]);
                x[0][2] = fmaf(a0v[e], t4.z, x[0][2]); x[0][3] = fmaf(a0v[e], t4.w, x[0][3]);
                x[1][0] = fmaf(a1v[e], t4.x, x[1][0]); x[1][1] = fmaf(a1v[e], t4.y, x[1][1]);
                x[1][2] = fmaf(a1v[e], t4.z, x[1][2]); x[1][3] = fmaf(a1v[e], t4.w, x[1][3]);
            }
        }
        group_sync(bar, 128); // Y is read: T21 takes its place
        *reinterpret_cast<float4 *>(Yr0) = make_float4(-x[0][0], -x[0][1], -x[0][2], -x[0][3]);
        *reinterpret_cast<float4 *>(Yr1) = make_float4(-x[1][0], -x[1][1], -x[1][2], -x[1][3]);
    }
}

} // namespace gdn
