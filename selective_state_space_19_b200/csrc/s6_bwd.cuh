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
// Four threads share a (sequence, channel), each owning N/4 of its states;
// the sums over the states (readout, du, dDelta) go through two shuffles.
// The reverse pass needs h_{t-1} at every t: a first forward pass saves the state
// at the start of every chunk of kBwdChunk tokens (checkpoints), then the
// chunks are walked last to first, each recomputed forward from its
// checkpoint into a scratch buffer and then walked backwards.  Scratch layouts
// put consecutive threads at consecutive addresses.  dB and dC are shared by
// all channels of a sequence: a warp whose lanes all belong to one sequence
// sums its 8 channels' shares with shuffles and adds them with one atomic
// per value, otherwise every lane adds its own.  The parameter gradients
// (dA_log, dD, ddt_bias) are summed over the sequences with atomics.
#pragma once

#include "s6_common.cuh"

namespace s6 {

constexpr int kBwdThreads = 128;
constexpr int kBwdChunk = 64;  // tokens between checkpoints
constexpr int kBwdTPC = 4;     // threads per channel (N/4 states each)

struct BwdArgs {
    int Bt, L, d, N, K, has_z, nck;
    const void *u, *dt, *B, *C, *z, *dy;  // u: the pre-conv x in the fused form
    const float *A_log, *D, *dt_bias, *h_init;
    const float *conv_w, *conv_b;          // fused form: [d, K] taps oldest first, [d] or null
    float *du, *ddt, *dz, *dB, *dC, *dA_log, *dD, *ddt_bias, *dh_init;  // du: dx in the fused form
    float *dconv_w, *dconv_b;              // fused form: [d, K], [d] or null
    float *ck;  // [nck][NS/4][Bt*d*4] state at the start of each chunk
    float *hb;  // [kBwdChunk][NS/4][Bt*d*4] the states of the chunk being reversed
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

// CONV: the fused path -- u_t = SiLU(pre_t), pre_t = conv_b + sum_k w[k] x[t-K+1+k]
// recomputed from x wherever it is needed; on the way back dpre_t =
// du_t SiLU'(pre_t), and dx[s] = sum_k w[k] dpre_{s+K-1-k} collects the next
// K-1 tokens' dpre from a sliding window, so each dx is final when written.
template <typename IO, int NS, bool ZOH, bool CONV>
__global__ void __launch_bounds__(kBwdThreads) s6_scan_bwd_kernel(const BwdArgs a) {
    using tr = io_traits<IO>;
    constexpr int T = kBwdChunk;
    constexpr int TPC = kBwdTPC;      // threads per channel
    constexpr int NH = NS / TPC;      // states per thread
    const long long G = static_cast<long long>(a.Bt) * a.d;  // channels
    const long long GT = G * TPC;                            // threads with work
    const long long gt = static_cast<long long>(blockIdx.x) * kBwdThreads + threadIdx.x;
    const bool live = gt < GT;
    const long long gtc = live ? gt : 0;
    const long long gc = gtc / TPC;  // channel
    const int q = static_cast<int>(gtc - gc * TPC);
    const int n0 = q * NH;           // this thread's first state
    const int b = static_cast<int>(gc / a.d);
    const int c = static_cast<int>(gc - static_cast<long long>(b) * a.d);
    const unsigned full = 0xffffffffu;
    // every lane of the warp in the same sequence: dB/dC can be summed in the warp
    const bool one_seq = __all_sync(full, b == __shfl_sync(full, b, 0));
    // sum over the TPC threads of a channel
    auto chan_sum = [&](float v) {
#pragma unroll
        for (int off = 1; off < TPC; off <<= 1)
            v += __shfl_xor_sync(full, v, off);
        return v;
    };

    float A[NH], A2[NH];
#pragma unroll
    for (int j = 0; j < NH; ++j) {
        const int n = n0 + j;
        const float Av = (n < a.N) ? -expf(a.A_log[static_cast<size_t>(c) * a.N + n]) : 0.0f;  // A = -exp(A_log)
        A[j] = Av;
        A2[j] = Av * kLog2e;
    }
    const float Dd = a.D[c];
    const float bias = a.dt_bias ? a.dt_bias[c] : 0.0f;
    // conv taps right-aligned into 4 slots (missing oldest taps are zero)
    float w[4] = {0.f, 0.f, 0.f, 0.f}, cbv = 0.f;
    if (CONV) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int src = k - (4 - a.K);
            w[k] = src >= 0 ? a.conv_w[static_cast<size_t>(c) * a.K + src] : 0.0f;
        }
        cbv = a.conv_b ? a.conv_b[c] : 0.0f;
    }

    auto seq = [&](const void *p, int t) -> float {
        return tr::to_f(static_cast<const IO *>(p)[(static_cast<size_t>(b) * a.L + t) * a.d + c]);
    };
    auto row = [&](const void *p, int t, int j) -> float {
        const int n = n0 + j;
        return (n < a.N) ? tr::to_f(static_cast<const IO *>(p)[(static_cast<size_t>(b) * a.L + t) * a.N + n]) : 0.0f;
    };
    // the pre-conv input at token t (zero before the sequence)
    auto xin = [&](int t) -> float { return t >= 0 ? seq(a.u, t) : 0.0f; };
    // scratch slot of this thread's state j at checkpoint / chunk row i
    auto slot = [&](float *base, int i, int j) -> float * {
        return base + (static_cast<size_t>(i) * NH + j) * GT + gtc;
    };
    // one forward token: h <- a h + gain B u
    // A token's inputs: raw dt, the conv window x[t-3..t] (x[3] alone is u
    // without the conv), dy, z, and this thread's B and C values.  In the
    // fused form (PF) they are read one token ahead of their use, so that the
    // window's loads overlap the previous token's arithmetic; without the conv
    // the extra registers cost more than the overlap gains (measured), and each
    // token's inputs are read when it starts.
    constexpr bool PF = CONV;
    struct Tok {
        float dt, x[4], dy, z, B[NH], C[NH];
    };
    auto load_tok = [&](int t, Tok &k, bool rev) {
        k.dt = seq(a.dt, t);
        if (CONV) {
#pragma unroll
            for (int i = 0; i < 3; ++i)
                k.x[i] = xin(t - 3 + i);
        }
        k.x[3] = seq(a.u, t);
#pragma unroll
        for (int j = 0; j < NH; ++j)
            k.B[j] = row(a.B, t, j);
        if (rev) {
            k.dy = live ? seq(a.dy, t) : 0.0f;
            k.z = a.has_z ? seq(a.z, t) : 0.0f;
#pragma unroll
            for (int j = 0; j < NH; ++j)
                k.C[j] = row(a.C, t, j);
        }
    };
    auto pre_of = [&](const Tok &k) {
        float p = cbv;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            p = fmaf(w[i], k.x[i], p);
        return p;
    };
    auto u_of = [&](const Tok &k) {
        if (CONV) {
            const float p = pre_of(k);
            return p / (1.0f + expf(-p));  // SiLU
        }
        return k.x[3];
    };
    auto step = [&](const Tok &k, float (&h)[NH]) {
        const float delta = softplus_f(k.dt + bias);
        const float uu = u_of(k);
#pragma unroll
        for (int j = 0; j < NH; ++j) {
            const float ab = ex2_approx(delta * A2[j]);
            const float gain = ZOH ? ((n0 + j < a.N) ? zoh_gain(delta * A[j], A[j]) : 0.0f) : delta;
            h[j] = fmaf(ab, h[j], gain * k.B[j] * uu);
        }
    };
    // forward over tokens [ta, tb) from h; `keep` stores each state in the chunk buffer
    auto walk = [&](int ta, int tb, float (&h)[NH], bool keep) {
        Tok cur, nxt;
        if (PF)
            load_tok(ta, cur, false);
        for (int t = ta; t < tb; ++t) {
            if (!PF)
                load_tok(t, cur, false);
            else if (t + 1 < tb)
                load_tok(t + 1, nxt, false);
            step(cur, h);
            if (keep && live) {
#pragma unroll
                for (int j = 0; j < NH; ++j)
                    *slot(a.hb, t - ta, j) = h[j];
            }
            if (PF)
                cur = nxt;
        }
    };

    // ---- pass 1: forward, checkpoint at every chunk start
    float h[NH];
#pragma unroll
    for (int j = 0; j < NH; ++j)
        h[j] = (live && a.h_init && n0 + j < a.N) ? a.h_init[gc * a.N + n0 + j] : 0.0f;
    for (int k = 0; k < a.nck; ++k) {
        if (live) {
#pragma unroll
            for (int j = 0; j < NH; ++j)
                *slot(a.ck, k, j) = h[j];
        }
        walk(k * T, min(a.L, (k + 1) * T), h, false);
    }

    // ---- pass 2: chunks last to first
    float gcar[NH], dA[NH];  // dLoss/dh from later tokens (times their decay); dLoss/dA
#pragma unroll
    for (int j = 0; j < NH; ++j)
        gcar[j] = dA[j] = 0.0f;
    float dDa = 0.0f, dba = 0.0f;  // kept by the channel's first thread
    float dW[4] = {0.f, 0.f, 0.f, 0.f}, dcb = 0.0f;  // conv taps, bias (first thread)
    float dp1 = 0.f, dp2 = 0.f, dp3 = 0.f;            // dpre of tokens t+1, t+2, t+3
    for (int k = a.nck - 1; k >= 0; --k) {
        const int t0 = k * T, t1 = min(a.L, t0 + T);
        float hc[NH];
#pragma unroll
        for (int j = 0; j < NH; ++j)
            hc[j] = live ? *slot(a.ck, k, j) : 0.0f;
        walk(t0, t1, hc, true);
        float ht[NH];  // h_t; the state after the chunk's last token is still in hc
#pragma unroll
        for (int j = 0; j < NH; ++j)
            ht[j] = live ? hc[j] : 0.0f;
        // h_{t-1} of token t: the chunk buffer's previous row, or the checkpoint
        auto load_prev = [&](int t, float (&hp)[NH]) {
#pragma unroll
            for (int j = 0; j < NH; ++j)
                hp[j] = live ? (t > t0 ? *slot(a.hb, t - t0 - 1, j) : *slot(a.ck, k, j)) : 0.0f;
        };
        Tok cur, nxt;
        float hpc[NH], hpn[NH];
        if (PF) {
            load_tok(t1 - 1, cur, true);
            load_prev(t1 - 1, hpc);
        }
        for (int t = t1 - 1; t >= t0; --t) {
            if (!PF) {
                load_tok(t, cur, true);
                load_prev(t, hpc);
            } else if (t - 1 >= t0) {
                load_tok(t - 1, nxt, true);
                load_prev(t - 1, hpn);
            }
            float hp[NH];  // h_{t-1}
#pragma unroll
            for (int j = 0; j < NH; ++j)
                hp[j] = hpc[j];
            const float v = cur.dt + bias;
            const float delta = softplus_f(v);
            float pre = 0.0f, uu;
            if (CONV) {
                pre = pre_of(cur);
                uu = pre / (1.0f + expf(-pre));
            } else {
                uu = cur.x[3];
            }
            const float dyv = cur.dy;
            float sp = 0.0f;
#pragma unroll
            for (int j = 0; j < NH; ++j)
                sp = fmaf(ht[j], cur.C[j], sp);
            const float s = fmaf(Dd, uu, chan_sum(sp));
            float gate = 1.0f;
            const size_t o = (static_cast<size_t>(b) * a.L + t) * a.d + c;
            if (a.has_z) {
                const float zv = cur.z;
                const float sg = 1.0f / (1.0f + expf(-zv));
                gate = zv * sg;
                if (live && q == 0)
                    a.dz[o] = dyv * s * sg * (1.0f + zv * (1.0f - sg));
            }
            const float ds = dyv * gate;
            float dup = 0.0f, ddp = 0.0f;  // this thread's shares of du and dDelta
            float dBn[NH], dCn[NH];
#pragma unroll
            for (int j = 0; j < NH; ++j) {
                const float ab = ex2_approx(delta * A2[j]);
                const float Bn = cur.B[j], Cn = cur.C[j];
                const bool inN = n0 + j < a.N;
                const float gain = ZOH ? (inN ? zoh_gain(delta * A[j], A[j]) : 0.0f) : delta;
                dCn[j] = ds * ht[j];
                const float dh = fmaf(ds, Cn, gcar[j]);
                const float da = dh * hp[j];
                const float dgain = dh * Bn * uu;
                dBn[j] = dh * gain * uu;
                dup = fmaf(dh * gain, Bn, dup);
                ddp = fmaf(da * ab, A[j], ddp);
                float dAn = da * ab * delta;
                if (ZOH) {
                    ddp = fmaf(dgain, ab, ddp);
                    if (inN)
                        dAn += dgain * zoh_dgain_dA(delta * A[j], delta, A[j]);
                } else if (inN) {
                    ddp += dgain;
                }
                dA[j] += dAn;
                gcar[j] = dh * ab;
            }
            const float dut = fmaf(ds, Dd, chan_sum(dup));
            const float dv = chan_sum(ddp) / (1.0f + expf(-v));  // softplus'(v) = sigmoid(v)
            if (q == 0) {
                dDa = fmaf(ds, uu, dDa);
                dba += dv;
                float dxo = dut;
                if (CONV) {
                    const float sg = 1.0f / (1.0f + expf(-pre));
                    const float dpre = dut * sg * (1.0f + pre * (1.0f - sg));  // SiLU'(pre)
                    dxo = fmaf(w[3], dpre, fmaf(w[2], dp1, fmaf(w[1], dp2, w[0] * dp3)));
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dW[i] = fmaf(dpre, cur.x[i], dW[i]);
                    dcb += dpre;
                    dp3 = dp2;
                    dp2 = dp1;
                    dp1 = dpre;
                }
                if (live) {
                    a.du[o] = dxo;
                    a.ddt[o] = dv;
                }
            }
            // dB, dC rows of (b, t): sum over the warp's 8 channels
            float *dBr = a.dB + (static_cast<size_t>(b) * a.L + t) * a.N + n0;
            float *dCr = a.dC + (static_cast<size_t>(b) * a.L + t) * a.N + n0;
            if (one_seq) {
#pragma unroll
                for (int j = 0; j < NH; ++j) {
                    float vb = dBn[j], vc = dCn[j];
#pragma unroll
                    for (int off = TPC; off < 32; off <<= 1) {
                        vb += __shfl_xor_sync(full, vb, off);
                        vc += __shfl_xor_sync(full, vc, off);
                    }
                    if ((threadIdx.x & 31) < TPC && n0 + j < a.N) {
                        atomicAdd(dBr + j, vb);
                        atomicAdd(dCr + j, vc);
                    }
                }
            } else if (live) {
#pragma unroll
                for (int j = 0; j < NH; ++j)
                    if (n0 + j < a.N) {
                        atomicAdd(dBr + j, dBn[j]);
                        atomicAdd(dCr + j, dCn[j]);
                    }
            }
#pragma unroll
            for (int j = 0; j < NH; ++j)
                ht[j] = hp[j];
            if (PF) {
#pragma unroll
                for (int j = 0; j < NH; ++j)
                    hpc[j] = hpn[j];
                cur = nxt;
            }
        }
    }
    if (!live)
        return;
#pragma unroll
    for (int j = 0; j < NH; ++j)
        if (n0 + j < a.N) {
            if (a.dh_init)
                a.dh_init[gc * a.N + n0 + j] = gcar[j];
            atomicAdd(a.dA_log + static_cast<size_t>(c) * a.N + n0 + j, dA[j] * A[j]);  // dA/dA_log = A
        }
    if (q == 0) {
        atomicAdd(a.dD + c, dDa);
        if (a.ddt_bias)
            atomicAdd(a.ddt_bias + c, dba);
        if (CONV) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int src = k - (4 - a.K);
                if (src >= 0)
                    atomicAdd(a.dconv_w + static_cast<size_t>(c) * a.K + src, dW[k]);
            }
            if (a.dconv_b)
                atomicAdd(a.dconv_b + c, dcb);
        }
    }
}

}  // namespace s6
