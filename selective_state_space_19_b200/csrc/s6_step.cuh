// s6_step.cuh -- batched single-token streaming step, state in place, sm_100a.
//
// "mamba, live" (what is actually running): one token in, one token out,
// constant work; the whole memory of a block is h_ssm (d_inner x N floats per
// sequence) plus a (K-1)-token conv history per channel.  One step applies the
// block's scan body to one token:
//     pre  = conv_b + sum_{k<K-1} w[k] hist[k] + w[K-1] u_t ;  u = SiLU(pre)
//     hist <- (hist[1..K-2], u_t)
//     Delta = softplus(dt_t + dt_bias);  A_bar = 2^(Delta A log2 e)
//     h    <- A_bar h + write;  y = (<h, C_t> + D u) * SiLU(z_t)
//
// HBM-bound: each (sequence, channel) reads and writes its N float32 states
// and its conv history once.  NS/4 threads share a channel, each owning four
// consecutive states (one 16-byte load and store), so a warp moves a
// contiguous 2 KiB of h per instruction at NS = 16; the readout is summed
// across those threads with shuffles.
#pragma once

#include "s6_common.cuh"

namespace s6 {

constexpr int kStepThreads = 128;

struct StepArgs {
    int Bt, d, N, K, zoh, has_z;
    const float *A_log, *D, *dt_bias, *conv_w, *conv_b;
    const void *u, *dt, *B, *C, *z;
    float *h;
    void *conv_state;
    void *y;
};

template <typename IO, int NS, bool ZOH>
__global__ void __launch_bounds__(kStepThreads) s6_step_kernel(const StepArgs a) {
    using tr = io_traits<IO>;
    constexpr int TPC = NS / 4;  // threads per channel
    const int gid = blockIdx.x * kStepThreads + threadIdx.x;
    const int q = gid % TPC;               // which 4 states
    const long long g = gid / TPC;         // (sequence, channel)
    const long long total = static_cast<long long>(a.Bt) * a.d;
    const bool live = g < total;
    const long long gc = live ? g : 0;
    const int b = static_cast<int>(gc / a.d);
    const int c = static_cast<int>(gc - static_cast<long long>(b) * a.d);

    const IO *u_p = static_cast<const IO *>(a.u);
    const IO *dt_p = static_cast<const IO *>(a.dt);
    const IO *B_p = static_cast<const IO *>(a.B);
    const IO *C_p = static_cast<const IO *>(a.C);
    IO *cs = static_cast<IO *>(a.conv_state) + gc * (a.K - 1);

    float u = 0.f, delta = 0.f, zg = 1.f;
    float hist[3] = {0.f, 0.f, 0.f};
    float xt = 0.f;
    if (live) {
        xt = tr::to_f(u_p[gc]);
        float pre = a.conv_b ? a.conv_b[c] : 0.0f;
        for (int k = 0; k < a.K - 1; ++k) {
            hist[k] = tr::to_f(cs[k]);
            pre = fmaf(a.conv_w[static_cast<size_t>(c) * a.K + k], hist[k], pre);
        }
        pre = fmaf(a.conv_w[static_cast<size_t>(c) * a.K + a.K - 1], xt, pre);
        u = silu_f(pre);
        delta = softplus_f(tr::to_f(dt_p[gc]) + (a.dt_bias ? a.dt_bias[c] : 0.0f));
        if (a.has_z)
            zg = silu_f(tr::to_f(static_cast<const IO *>(a.z)[gc]));
    }

    float acc = 0.0f;
    if (live) {
        float *hp = a.h + gc * a.N;
        const float *alp = a.A_log + static_cast<size_t>(c) * a.N;
        const IO *Bp = B_p + static_cast<size_t>(b) * a.N;
        const IO *Cp = C_p + static_cast<size_t>(b) * a.N;
        const int n0 = 4 * q;
        float hv[4], al[4], Bv[4], Cv[4];
        const bool vec = (a.N == NS);
        if (vec) {
            const float4 h4 = *reinterpret_cast<const float4 *>(hp + n0);
            const float4 a4 = __ldg(reinterpret_cast<const float4 *>(alp + n0));
            hv[0] = h4.x; hv[1] = h4.y; hv[2] = h4.z; hv[3] = h4.w;
            al[0] = a4.x; al[1] = a4.y; al[2] = a4.z; al[3] = a4.w;
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const bool in = n0 + j < a.N;
                hv[j] = in ? hp[n0 + j] : 0.0f;
                al[j] = in ? alp[n0 + j] : 0.0f;
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const bool in = n0 + j < a.N;
            Bv[j] = in ? tr::to_f(Bp[n0 + j]) : 0.0f;
            Cv[j] = in ? tr::to_f(Cp[n0 + j]) : 0.0f;
        }
        const float du = delta * u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (n0 + j < a.N) {
                const float A = -ex2_approx(al[j] * kLog2e);  // A = -exp(A_log)
                const float abar = ex2_approx(delta * A * kLog2e);
                if (ZOH) {
                    const float k = (Bv[j] * u) / A;
                    hv[j] = fmaf(abar, hv[j] + k, -k);
                } else {
                    hv[j] = fmaf(abar, hv[j], du * Bv[j]);
                }
                acc = fmaf(hv[j], Cv[j], acc);
            }
        }
        if (vec) {
            *reinterpret_cast<float4 *>(hp + n0) = make_float4(hv[0], hv[1], hv[2], hv[3]);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (n0 + j < a.N)
                    hp[n0 + j] = hv[j];
        }
    }
    // readout: sum the TPC partial dot products of this channel
#pragma unroll
    for (int off = 1; off < TPC; off <<= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, off);

    if (live && q == 0) {
        const float yv = fmaf(a.D[c], u, acc) * zg;
        static_cast<IO *>(a.y)[gc] = tr::from_f(yv);
        for (int k = 0; k + 1 < a.K - 1; ++k)
            cs[k] = tr::from_f(hist[k + 1]);
        cs[a.K - 2] = tr::from_f(xt);
    }
}

}  // namespace s6
