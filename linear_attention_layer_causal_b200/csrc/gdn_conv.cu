// gdn_conv.cu -- prefill front end: conv + SiLU + L2 norm of every q|k|v
// channel (the per-thread body is in gdn_conv.cuh), and the final conv window
// of every sequence.
#include "gdn_conv.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

constexpr int kConvThreads = 256;

// One CTA: kConvTokens consecutive packed tokens x kConvThreads channel
// vectors (8 bytes = 4 channels for bf16 at head dim 128, whose lighter
// threads fit four CTAs on an SM; 16 bytes otherwise).  The lanes covering one head are consecutive and the head
// width d / V divides 32, so the L2 reduction is a shuffle within an aligned
// lane group.
template <typename T, int D, typename VecT = Vec16<T>>
__global__ void __launch_bounds__(kConvThreads, sizeof(VecT) == 8 ? 4 : 1) // 8-byte units: 64 registers
conv_prep_kernel(ConvIO<T> io, unsigned int *__restrict__ err) {
    constexpr int V = VecT::N;
    const int C = (2 * io.Hk + io.Hv) * D;
    // the first kernel of a token-serial call clears the call's status words
    if (err != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
        err[0] = 0u; // status word of this call; later kernels only set bits
        err[1] = 0u; // where the first timed-out wait gave up
    }
    const int by = (int)blockIdx.y + io.block_y0;
    const int c0 = (by * kConvThreads + threadIdx.x) * V;
    const bool active = c0 < C;
    const int64_t t0 = (int64_t)blockIdx.x * kConvTokens;
    const int64_t tend = t0 + kConvTokens < io.N ? t0 + kConvTokens : io.N;
    const int n = seq_of_token(io.cu, io.batch, t0 < io.N ? t0 : io.N - 1);
    // a block whose channels all lie in v skips the norm code (uniform branch)
    if (by * kConvThreads * V >= 2 * io.Hk * D)
        conv_thread<T, D, true, VecT>(io, active ? c0 : 2 * io.Hk * D, active, t0, tend, n);
    else
        conv_thread<T, D, false, VecT>(io, active ? c0 : 0, active, t0, tend, n);
}

// final_conv[n] = the last 3 pre-conv rows of [init_conv[n]; sequence n].
// Each thread reads all three source rows of its channels before writing, so
// final_conv may alias init_conv.
template <typename T>
__global__ void final_conv_kernel(const T *__restrict__ qkv, const int32_t *__restrict__ cu,
                                  int batch, int64_t N, const T *init_conv, T *final_conv, int C) {
    constexpr int V = Vec16<T>::N;
    const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * V;
    const int n = blockIdx.y;
    if (c0 >= C || n >= batch)
        return;
    int64_t start, end;
    seq_bounds(cu, n, N, start, end);
    Vec16<T> r[3];
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const int64_t src = end - 3 + i;
        if (src >= start)
            r[i] = ld16_nc(qkv + src * C + c0);
        else if (init_conv != nullptr)
            r[i] = ld16(init_conv + ((int64_t)n * 3 + (3 + (src - start))) * C + c0);
        else
            r[i] = zero16<T>();
    }
#pragma unroll
    for (int i = 0; i < 3; ++i)
        st16(final_conv + ((int64_t)n * 3 + i) * C + c0, r[i]);
}

template <typename T>
ConvIO<T> conv_io(const PrefillArgs &p) {
    ConvIO<T> io;
    io.qkv = (const T *)p.qkv;
    io.cu = p.cu;
    io.batch = p.batch;
    io.N = p.N;
    io.init_conv = (const T *)p.init_conv;
    io.conv_w = p.conv_w;
    io.Hk = p.Hk;
    io.Hv = p.Hv;
    io.l2_eps = p.l2_eps;
    io.q_scale = p.q_scale;
    io.qk_out = (float *)p.ws_qk;
    io.v_out = (float *)p.ws_v;
    io.round_v = p.chunked;
    io.block_y0 = 0;
    return io;
}

template <typename T, int D, typename VecT = Vec16<T>>
cudaError_t launch_conv_prep_t(const PrefillArgs &p, ConvPart part, cudaStream_t s) {
    constexpr int V = VecT::N;
    const int C = (2 * p.Hk + p.Hv) * D;
    ConvIO<T> io = conv_io<T>(p);
    // channel blocks: those holding any q or k channel come first (a block that
    // straddles the q/k | v boundary belongs to them and writes its v channels too)
    const int nb = (C / V + kConvThreads - 1) / kConvThreads;
    const int nqk = (2 * p.Hk * D / V + kConvThreads - 1) / kConvThreads;
    io.block_y0 = part == ConvPart::kV ? nqk : 0;
    const int nby = part == ConvPart::kAll ? nb : (part == ConvPart::kQK ? nqk : nb - nqk);
    if (nby <= 0)
        return cudaSuccess;
    dim3 grid((unsigned)((p.N + kConvTokens - 1) / kConvTokens), nby);
    // the chunked path's offsets kernel clears the status words; the token-serial
    // path's single conv launch does
    conv_prep_kernel<T, D, VecT><<<grid, kConvThreads, 0, s>>>(io, p.chunked ? nullptr : p.ws_err);
    return cudaGetLastError();
}

template <typename T> cudaError_t launch_final_conv_t(const PrefillArgs &p, cudaStream_t s) {
    constexpr int V = Vec16<T>::N;
    const int C = (2 * p.Hk + p.Hv) * p.D;
    dim3 grid((C / V + 255) / 256, p.batch);
    final_conv_kernel<T><<<grid, 256, 0, s>>>((const T *)p.qkv, p.cu, p.batch, p.N,
                                              (const T *)p.init_conv, (T *)p.final_conv, C);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_conv_prep(const PrefillArgs &p, ConvPart part, cudaStream_t s) {
    if (p.N == 0)
        return cudaSuccess;
    if (p.bf16)
        return p.D == 128 ? launch_conv_prep_t<__nv_bfloat16, 128, Vec8bf>(p, part, s)
                          : launch_conv_prep_t<__nv_bfloat16, 32>(p, part, s);
    return p.D == 128 ? launch_conv_prep_t<float, 128>(p, part, s)
                      : launch_conv_prep_t<float, 32>(p, part, s);
}

cudaError_t launch_final_conv(const PrefillArgs &p, cudaStream_t s) {
    if (p.final_conv == nullptr || p.batch == 0)
        return cudaSuccess;
    return p.bf16 ? launch_final_conv_t<__nv_bfloat16>(p, s) : launch_final_conv_t<float>(p, s);
}

} // namespace gdn
