// s6_conv.cuh -- standalone causal depthwise conv + SiLU, sm_100a.
//
// "mamba, live" (what is actually running): xc = SiLU(depthwise_conv4(xin)),
// 4-tap causal, per channel.  "Carry context through a selective state"
// (manifest step "local"): the conv is left-padded, reading the current and
// the K-1 earlier inputs.
//
//     out[b,t,c] = SiLU(conv_b[c] + sum_{k<K} conv_w[c,k] * x[b, t-K+1+k, c]),  x[b,<0,c] = 0
//
// HBM-bound: every input element is read once (plus 3 halo rows per run of
// tokens) and every output written once.  A thread owns VEC = 16/sizeof(io)
// consecutive channels, so each token is one 16-byte load and one 16-byte
// store; a warp covers 32*VEC contiguous channels of one token row (512 B
// coalesced).  The warps of a CTA walk different runs of TS tokens.
#pragma once

#include "s6_common.cuh"

namespace s6 {

constexpr int kConvWarps = 4;
constexpr int kConvRun = 64;  // tokens per thread

template <typename IO>
struct ConvVec {
    static constexpr int VEC = 16 / sizeof(IO);
    union U {
        uint4 raw;
        IO v[VEC];
    };
};

struct ConvArgs {
    int Bt, L, d, K;
    const void *x;
    const float *conv_w;  // [d, K]
    const float *conv_b;  // [d] or null
    void *out;
};

template <typename IO>
__global__ void __launch_bounds__(32 * kConvWarps) s6_conv_silu_kernel(const ConvArgs a) {
    using V = ConvVec<IO>;
    using tr = io_traits<IO>;
    constexpr int VEC = V::VEC;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int c_base = (blockIdx.x * 32 + lane) * VEC;
    const int t_begin = (blockIdx.y * kConvWarps + warp) * kConvRun;
    const int b = blockIdx.z;
    if (c_base >= a.d || t_begin >= a.L)
        return;
    const int t_end = min(a.L, t_begin + kConvRun);

    // taps right-aligned into 4 slots (missing oldest taps are zero)
    float w[VEC][4], cb[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
        const int c = c_base + j;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int src = k - (4 - a.K);
            w[j][k] = (src >= 0) ? a.conv_w[static_cast<size_t>(c) * a.K + src] : 0.0f;
        }
        cb[j] = a.conv_b ? a.conv_b[c] : 0.0f;
    }

    const IO *xp = static_cast<const IO *>(a.x) + (static_cast<size_t>(b) * a.L) * a.d + c_base;
    IO *op = static_cast<IO *>(a.out) + (static_cast<size_t>(b) * a.L) * a.d + c_base;

    auto load_row = [&](int t, float (&dst)[VEC]) {
        typename V::U u;
        if (t >= 0) {
            u.raw = __ldg(reinterpret_cast<const uint4 *>(xp + static_cast<size_t>(t) * a.d));
#pragma unroll
            for (int j = 0; j < VEC; ++j)
                dst[j] = tr::to_f(u.v[j]);
        } else {
#pragma unroll
            for (int j = 0; j < VEC; ++j)
                dst[j] = 0.0f;
        }
    };

    float h3[VEC], h2[VEC], h1[VEC];  // x[t-3], x[t-2], x[t-1]
    load_row(t_begin - 3, h3);
    load_row(t_begin - 2, h2);
    load_row(t_begin - 1, h1);

    constexpr int U = 4;  // tokens loaded ahead of their use
    int t = t_begin;
    for (; t + U <= t_end; t += U) {
        float xr[U][VEC];
#pragma unroll
        for (int i = 0; i < U; ++i)
            load_row(t + i, xr[i]);
#pragma unroll
        for (int i = 0; i < U; ++i) {
            typename V::U o;
#pragma unroll
            for (int j = 0; j < VEC; ++j) {
                float pre = fmaf(w[j][0], h3[j], cb[j]);
                pre = fmaf(w[j][1], h2[j], pre);
                pre = fmaf(w[j][2], h1[j], pre);
                pre = fmaf(w[j][3], xr[i][j], pre);
                o.v[j] = tr::from_f(silu_f(pre));
                h3[j] = h2[j];
                h2[j] = h1[j];
                h1[j] = xr[i][j];
            }
            *reinterpret_cast<uint4 *>(op + static_cast<size_t>(t + i) * a.d) = o.raw;
        }
    }
    for (; t < t_end; ++t) {
        float xr[VEC];
        load_row(t, xr);
        typename V::U o;
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            float pre = fmaf(w[j][0], h3[j], cb[j]);
            pre = fmaf(w[j][1], h2[j], pre);
            pre = fmaf(w[j][2], h1[j], pre);
            pre = fmaf(w[j][3], xr[j], pre);
            o.v[j] = tr::from_f(silu_f(pre));
            h3[j] = h2[j];
            h2[j] = h1[j];
            h1[j] = xr[j];
        }
        *reinterpret_cast<uint4 *>(op + static_cast<size_t>(t) * a.d) = o.raw;
    }
}

}  // namespace s6
