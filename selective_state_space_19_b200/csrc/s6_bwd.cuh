// s6_bwd.cuh -- backward pass of the selective scan (no conv: u given), sm_100a.
//
// Gradients of the loss sum_t dy[t] * y[t] through the scan of s6_scan.cuh
// ("Carry context through a selective state": the recurrence is what makes
// training slow, every timestep touching N states).  Per (sequence b,
// channel c), with Delta_t = softplus(v_t), v_t = dt_t + dt_bias,
// a_t = exp(Delta_t A), gain_t = Delta_t (simplified) or (a_t - 1)/A (ZOH):
//
//     s_t   = <h_t, C_t> + D u_t,  y_t = s_t * SiLU(z_t)
//     ds_t  = dy_t SiLU(z_t);  dz_t = dy_t s_t SiLU'(z_t)
//     dh_t  = ds_t C_t + a_{t+1} dh_{t+1}               (reverse recurrence)
//     dC_t += ds_t h_t;  dB_t += dh_t gain_t u_t;  du_t = ds_t D + <dh_t, gain_t B_t>
//     dDelta_t = <dh_t h_{t-1}, a_t A> + <dh_t B_t u_t, dgain/dDelta>
//     dA      += dh_t h_{t-1} a_t Delta_t (+ ZOH: dh_t B_t u_t dgain/dA)
//     ddt_t = dDelta_t sigmoid(v_t);  dA_log = dA * A;  dD += ds_t u_t
//
// One thread owns one (sequence, channel) and all of its N states.  The
// reverse pass needs h_{t-1} at every t: a first forward pass saves the state
// at the start of every chunk of kBwdChunk tokens (checkpoints), then the
// chunks are walked last to first, each recomputed forward from its
// checkpoint into a scratch buffer and then walked backwards.  Scratch layouts
// put consecutive threads at consecutive addresses.  dB and dC are shared by
// all channels of a sequence: a warp whose lanes all belong to one sequence
// sums its 32 channels' shares with shuffles and adds them with one atomic
// per value, otherwise every lane adds its own.  The parameter gradients
// (dA_log, dD, ddt_bias) are summed over the sequences with atomics.
#pragma once

#include "s6_common.cuh"

namespace s6 {

constexpr int kBwdThreads = 128;
constexpr int kBwdChunk = 64;  // tokens between checkpoints

struct BwdArgs {
    int Bt, L, d, N, has_z, nck;
    const void *u, *dt, *B, *C, *z, *dy;
    const float *A_log, *D, *dt_bias, *h_init;
    float *du, *ddt, *dz, *dB, *dC, *dA_log, *dD, *ddt_bias, *dh_init;
    float *ck;  // [nck][NS][Bt*d] state at the start of each chunk
    float *hb;  // [kBwdChunk][NS][Bt*d] the states of the chunk being reversed
};

// ZOH write gain (e^x - 1)/A with x = Delta*A, and its derivative in A at
// fixed Delta, (x e^x - (e^x - 1))/A^2 = Delta^2 f(x)/x^2 with
// f(x) = e^x (x - 1) + 1 = x^2 (1/2 + x/3 + x^2/8 + x^3/30 + x^4/144 + ...);
// the series is used for |x| < 1/4 (truncation below 3e-6 relative), where
// the closed form cancels in float32.
__device__ __forceinline__ float zoh_gain(float x, float A) { return expm1f(x) / A; }
__device__ __forceinline__ float zoh_dgain_dA(float x, float delta, float A) {
    if (fabsf(x) < 0.25f) {
        const float p = fmaf(fmaf(fmaf(fmaf(x, 1.0f / 144.0f, 1.0f / 30.0f), x, 0.125f), x, 1.0f / 3.0f), x, 0.5f);
        return delta * delta * p;
    }
    return (x * expf(x) - expm1f(x)) / (A * A);
}

template <typename IO, int NS, bool ZOH>
__global__ void __launch_bounds__(kBwdThreads) s6_scan_bwd_kernel(const BwdArgs a) {
    using tr = io_traits<IO>;
    constexpr int T = kBwdChunk;
    const long long G = static_cast<long long>(a.Bt) * a.d;
    const long long g = static_cast<long long>(blockIdx.x) * kBwdThreads + threadIdx.x;
    const bool live = g < G;
    const long long gc = live ? g : 0;
    const int b = static_cast<int>(gc / a.d);
    const int c = static_cast<int>(gc - static_cast<long long>(b) * a.d);
    const unsigned full = 0xffffffffu;
    // every lane of the warp in the same sequence: dB/dC can be summed in the warp
    const bool one_seq = __all_sync(full, b == __shfl_sync(full, b, 0));

    float A[NS], A2[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) {
        const float Av = (n < a.N) ? -expf(a.A_log[static_cast<size_t>(c) * a.N + n]) : 0.0f;  // A = -exp(A_log)
        A[n] = Av;
        A2[n] = Av * kLog2e;
    }
    const float Dd = a.D[c];
    const float bias = a.dt_bias ? a.dt_bias[c] : 0.0f;

    auto seq = [&](const void *p, int t) -> float {
        return tr::to_f(static_cast<const IO *>(p)[(static_cast<size_t>(b) * a.L + t) * a.d + c]);
    };
    auto row = [&](const void *p, int t, int n) -> float {
        return (n < a.N) ? tr::to_f(static_cast<const IO *>(p)[(static_cast<size_t>(b) * a.L + t) * a.N + n]) : 0.0f;
    };
    auto slot = [&](float *base, int i, int n) -> float * {
        return base + (static_cast<size_t>(i) * NS + n) * G + gc;
    };
    // one forward token: h <- a h + gain B u
    auto step = [&](int t, float (&h)[NS]) {
        const float delta = softplus_f(seq(a.dt, t) + bias);
        const float uu = seq(a.u, t);
#pragma unroll
        for (int n = 0; n < NS; ++n) {
            const float ab = ex2_approx(delta * A2[n]);
            const float gain = ZOH ? ((n < a.N) ? zoh_gain(delta * A[n], A[n]) : 0.0f) : delta;
            h[n] = fmaf(ab, h[n], gain * row(a.B, t, n) * uu);
        }
    };

    // ---- pass 1: forward, checkpoint at every chunk start
    float h[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n)
        h[n] = (live && a.h_init && n < a.N) ? a.h_init[gc * a.N + n] : 0.0f;
    for (int k = 0; k < a.nck; ++k) {
        if (live) {
#pragma unroll
            for (int n = 0; n < NS; ++n)
                *slot(a.ck, k, n) = h[n];
        }
        const int t1 = min(a.L, (k + 1) * T);
        for (int t = k * T; t < t1; ++t)
            step(t, h);
    }

    // ---- pass 2: chunks last to first
    float gcar[NS], dA[NS];  // dLoss/dh from later tokens (times their decay); dLoss/dA
#pragma unroll
    for (int n = 0; n < NS; ++n)
        gcar[n] = dA[n] = 0.0f;
    float dDa = 0.0f, dba = 0.0f;
    for (int k = a.nck - 1; k >= 0; --k) {
        const int t0 = k * T, t1 = min(a.L, t0 + T);
        float hc[NS];
#pragma unroll
        for (int n = 0; n < NS; ++n)
            hc[n] = live ? *slot(a.ck, k, n) : 0.0f;
        for (int t = t0; t < t1; ++t) {
            step(t, hc);
            if (live) {
#pragma unroll
                for (int n = 0; n < NS; ++n)
                    *slot(a.hb, t - t0, n) = hc[n];
            }
        }
        for (int t = t1 - 1; t >= t0; --t) {
            float ht[NS], hp[NS];
#pragma unroll
            for (int n = 0; n < NS; ++n) {
                ht[n] = live ? *slot(a.hb, t - t0, n) : 0.0f;
                hp[n] = live ? (t > t0 ? *slot(a.hb, t - t0 - 1, n) : *slot(a.ck, k, n)) : 0.0f;
            }
            const float v = seq(a.dt, t) + bias;
            const float delta = softplus_f(v);
            const float uu = seq(a.u, t);
            const float dyv = live ? seq(a.dy, t) : 0.0f;
            float s = Dd * uu;
#pragma unroll
            for (int n = 0; n < NS; ++n)
                s = fmaf(ht[n], row(a.C, t, n), s);
            float gate = 1.0f;
            if (a.has_z) {
                const float zv = seq(a.z, t);
                const float sg = 1.0f / (1.0f + expf(-zv));
                gate = zv * sg;
                if (live)
                    a.dz[(static_cast<size_t>(b) * a.L + t) * a.d + c] = dyv * s * sg * (1.0f + zv * (1.0f - sg));
            }
            const float ds = dyv * gate;
            dDa = fmaf(ds, uu, dDa);
            float dut = ds * Dd, ddelta = 0.0f;
            float dBn[NS], dCn[NS];
#pragma unroll
            for (int n = 0; n < NS; ++n) {
                const float ab = ex2_approx(delta * A2[n]);
                const float Bn = row(a.B, t, n), Cn = row(a.C, t, n);
                const float gain = ZOH ? ((n < a.N) ? zoh_gain(delta * A[n], A[n]) : 0.0f) : delta;
                dCn[n] = ds * ht[n];
                const float dh = fmaf(ds, Cn, gcar[n]);
                const float da = dh * hp[n];
                const float dgain = dh * Bn * uu;
                dBn[n] = dh * gain * uu;
                dut = fmaf(dh * gain, Bn, dut);
                ddelta = fmaf(da * ab, A[n], ddelta);
                float dAn = da * ab * delta;
                if (ZOH) {
                    ddelta = fmaf(dgain, ab, ddelta);
                    if (n < a.N)
                        dAn += dgain * zoh_dgain_dA(delta * A[n], delta, A[n]);
                } else {
                    ddelta += dgain;
                }
                dA[n] += dAn;
                gcar[n] = dh * ab;
            }
            const float dv = ddelta / (1.0f + expf(-v));  // softplus'(v) = sigmoid(v)
            dba += dv;
            if (live) {
                const size_t o = (static_cast<size_t>(b) * a.L + t) * a.d + c;
                a.du[o] = dut;
                a.ddt[o] = dv;
            }
            // dB, dC rows of (b, t): sum over the channels
            float *dBr = a.dB + (static_cast<size_t>(b) * a.L + t) * a.N;
            float *dCr = a.dC + (static_cast<size_t>(b) * a.L + t) * a.N;
            if (one_seq) {
#pragma unroll
                for (int n = 0; n < NS; ++n) {
                    float vb = dBn[n], vc = dCn[n];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) {
                        vb += __shfl_xor_sync(full, vb, off);
                        vc += __shfl_xor_sync(full, vc, off);
                    }
                    if ((threadIdx.x & 31) == 0 && n < a.N) {
                        atomicAdd(dBr + n, vb);
                        atomicAdd(dCr + n, vc);
                    }
                }
            } else if (live) {
#pragma unroll
                for (int n = 0; n < NS; ++n)
                    if (n < a.N) {
                        atomicAdd(dBr + n, dBn[n]);
                        atomicAdd(dCr + n, dCn[n]);
                    }
            }
        }
    }
    if (!live)
        return;
    if (a.dh_init) {
#pragma unroll
        for (int n = 0; n < NS; ++n)
            if (n < a.N)
                a.dh_init[gc * a.N + n] = gcar[n];
    }
#pragma unroll
    for (int n = 0; n < NS; ++n)
        if (n < a.N)
            atomicAdd(a.dA_log + static_cast<size_t>(c) * a.N + n, dA[n] * A[n]);  // dA/dA_log = A
    atomicAdd(a.dD + c, dDa);
    if (a.ddt_bias)
        atomicAdd(a.ddt_bias + c, dba);
}

}  // namespace s6
