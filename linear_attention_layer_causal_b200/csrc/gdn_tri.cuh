// gdn_tri.cuh -- the shared-memory layout of the 64 x 64 lower-triangular
// tiles of the chunked gated delta rule (A[r][s] = beta_r exp(G_r - G_s)
// k_r . k_s for s < r, its inverse T = (I + A)^-1, and P; the chunked form of
// the Gated DeltaNet recurrence, "Qwen3.8-2.4T-A95B vs Inkling", component
// table, Gated DeltaNet row), and the helpers that walk them.
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

} // namespace gdn
