// gdn_common.cuh -- small device helpers shared by the library's kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

// Activation element <-> float.
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// 16-byte vector of activations: 8 bf16 or 4 floats.
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    uint4 raw;
    __device__ __forceinline__ float get(int i) const {
        const __nv_bfloat16 *p = reinterpret_cast<const __nv_bfloat16 *>(&raw);
        return __bfloat162float(p[i]);
    }
    __device__ __forceinline__ void set(int i, float x) {
        __nv_bfloat16 *p = reinterpret_cast<__nv_bfloat16 *>(&raw);
        p[i] = __float2bfloat16_rn(x);
    }
};
template <> struct Vec16<float> {
    static constexpr int N = 4;
    uint4 raw;
    __device__ __forceinline__ float get(int i) const {
        return reinterpret_cast<const float *>(&raw)[i];
    }
    __device__ __forceinline__ void set(int i, float x) { reinterpret_cast<float *>(&raw)[i] = x; }
};

// 8-byte vector of 4 bf16 activations: a lighter unit for the prefill conv
// (half the registers per thread of Vec16, so more warps fit on an SM).
struct Vec8bf {
    static constexpr int N = 4;
    uint2 raw;
    // element i: the high or low half of word i / 2 (a bf16 is the top 16 bits
    // of the float with the same value)
    __device__ __forceinline__ float get(int i) const {
        const uint32_t w = i < 2 ? raw.x : raw.y;
        return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
    }
};

template <typename T> __device__ __forceinline__ Vec16<T> ld16(const T *p) {
    Vec16<T> v;
    v.raw = *reinterpret_cast<const uint4 *>(p);
    return v;
}
template <typename T> __device__ __forceinline__ Vec16<T> ld16_nc(const T *p) {
    Vec16<T> v;
    v.raw = __ldg(reinterpret_cast<const uint4 *>(p));
    return v;
}
template <typename T> __device__ __forceinline__ void st16(T *p, const Vec16<T> &v) {
    *reinterpret_cast<uint4 *>(p) = v.raw;
}
template <typename T> __device__ __forceinline__ Vec16<T> zero16() {
    Vec16<T> v;
    v.raw = make_uint4(0u, 0u, 0u, 0u);
    return v;
}

// Loads and stores cached in L2 only: a kernel whose shared memory takes most
// of the L1/shared store leaves little L1, and strided element accesses that
// allocate L1 lines then serialise.
__device__ __forceinline__ float ld_cg(const float *p) { return __ldcg(p); }
__device__ __forceinline__ float ld_cg(const __nv_bfloat16 *p) {
    return __bfloat162float(__ushort_as_bfloat16(__ldcg(reinterpret_cast<const unsigned short *>(p))));
}
__device__ __forceinline__ void st_cg(float *p, float x) { __stcg(p, x); }
__device__ __forceinline__ void st_cg(__nv_bfloat16 *p, float x) {
    __stcg(reinterpret_cast<unsigned short *>(p), __bfloat16_as_ushort(__float2bfloat16_rn(x)));
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + __expf(-x)); }
__device__ __forceinline__ float siluf_(float x) { return __fdividef(x, 1.0f + __expf(-x)); }
// log(1 + e^x) = max(x, 0) + log1p(e^{-|x|}), finite for every x.
__device__ __forceinline__ float softplusf_(float x) {
    return fmaxf(x, 0.0f) + log1pf(__expf(-fabsf(x)));
}

// Index of the sequence that owns packed token t: the n with cu[n] <= t < cu[n+1]
// (the last such n when empty sequences share a boundary).
__device__ __forceinline__ int seq_of_token(const int32_t *__restrict__ cu, int batch, int64_t t) {
    int lo = 0, hi = batch - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((int64_t)__ldg(cu + mid) <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Rows [start, end) of sequence n, clamped to [0, N) so that a malformed
// cu_seqlens array can never move an access outside the packed tensors.
__device__ __forceinline__ void seq_bounds(const int32_t *__restrict__ cu, int n, int64_t N,
                                           int64_t &start, int64_t &end) {
    int64_t s = __ldg(cu + n), e = __ldg(cu + n + 1);
    s = s < 0 ? 0 : (s > N ? N : s);
    e = e < s ? s : (e > N ? N : e);
    start = s;
    end = e;
}

template <int W> __device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = W / 2; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

} // namespace gdn
