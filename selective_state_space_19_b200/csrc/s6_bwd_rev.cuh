// s6_bwd_rev.cuh -- backward of the selective scan at N = 16 (sm_100a): the
// reverse walk of the gradient recurrence over state checkpoints.
//
// Gradients of the loss sum_t dy[t] * y[t] ("Carry context through a selective
// state": the recurrence is what makes training slow, every timestep touching
// N states).  Per (sequence b, channel c), with Delta_t = softplus(v_t),
// v_t = dt_t + dt_bias, a_t = 2^(Delta_t A log2 e), gain_t = Delta_t
// (simplified write) or (a_t - 1)/A (exact ZOH):
//
//     s_t   = <h_t, C_t> + D u_t,  y_t = s_t * SiLU(z_t)
//     ds_t  = dy_t SiLU(z_t);  dz_t = dy_t s_t SiLU'(z_t)
//     dh_t  = ds_t C_t + a_{t+1} dh_{t+1}               (the reverse recurrence)
//     dC_t += ds_t h_t;  dB_t += dh_t gain_t u_t;  du_t = ds_t D + <dh_t, gain_t B_t>
//     dDelta_t = <dh_t h_{t-1} a_t, A> + <dh_t B_t u_t, dgain/dDelta>
//     dA      += dh_t h_{t-1} a_t Delta_t (+ exact ZOH: dh_t B_t u_t dgain/dA)
//     ddt_t = dDelta_t sigmoid(v_t);  dA_log = dA * A;  dD += ds_t u_t
//
// The forward kernel (s6_scan.cuh, checkpoint mode) first stores the state
// before every kRevChunk-th token.  This kernel then walks each (sequence,
// 64-channel tile) chain backwards one sub-chunk of kRevChunk tokens at a
// time: a producer warp brings the sub-chunk's rows of x (with the conv's
// halo), dt, z, dy and its B / C rows into a shared-memory ring by TMA; the
// four consumer warps recompute the sub-chunk forward from its checkpoint,
// keeping every state in shared memory, and walk it back token by token.  Two
// threads share a channel (8 states each, packed f32x2 arithmetic).  dB and dC
// are sums over the channels of a sequence: each warp reduce-scatters its 16
// channels' 32 values per token across its lanes (15 shuffles a thread), the
// four warps add theirs in shared memory, and one row per (tile, token) is
// written to a partial buffer that s6_bwd_bc_reduce_kernel sums over the
// tiles -- no global atomics (the order of the four warps' shared-memory adds
// is not fixed, so runs agree to float32 rounding).  A chain is cut
// into segments pulled last-first from a global counter; a segment's unit
// starts from dLoss/dh (and the conv's dpre window) published by the unit of
// the segment after it, which was pulled earlier, so every (bounded) wait ends.
#pragma once

#include <type_traits>

#include "s6_common.cuh"
#include "s6_scan.cuh"

namespace s6 {

constexpr int kRevChunk = kCkptEvery;  // tokens per sub-chunk = checkpoint spacing
constexpr int kRevStages = 2;
constexpr int kRevCarry = 20;  // floats published per channel: dLoss/dh (16) + dpre window (3) + pad

struct RevArgs {
    int Bt, L, d, K, has_z;
    int tiles, nseg, seg_len, units, dynamic, nck;
    const float *A_log, *D, *dt_bias, *conv_w, *conv_b;
    const float *ckpt;  // [Bt][nck][d][16] state before token k * kRevChunk
    float *du, *ddt, *dz;  // [Bt, L, d]; du is dx in the fused form
    float *part;           // [tiles][Bt][L][32]: dB (n) and dC (16 + n) summed over a tile's channels
    float *dA_log, *dD, *ddt_bias, *dconv_w, *dconv_b, *dh_init;
    unsigned int *counter;  // dynamic: next unit to hand out (zeroed before launch)
    unsigned int *flags;    // dynamic: [chains][consumer warps] segments finished, counted from the end
    float *carry;           // dynamic: [chains][64][kRevCarry]
    unsigned int carry_polls;
};

template <typename IO, bool CONV>
struct RevSmem {
    static constexpr int XR = kRevChunk + (CONV ? kHalo : 0);
    Tile<IO, XR, 64> x[kRevStages];  // row r: token t0 - (CONV ? 3 : 0) + r
    Tile<IO, kRevChunk, 64> dt[kRevStages];
    Tile<IO, kRevChunk, 64> z[kRevStages];
    Tile<IO, kRevChunk, 64> dy[kRevStages];
    Tile<IO, 1, kRevChunk * 16> braw[kRevStages];
    Tile<IO, 1, kRevChunk * 16> craw[kRevStages];
    float bc[kRevStages][kRevChunk][2][16];         // B | C rows in float32
    float4 hbuf[kConsumerWarps][kRevChunk + 1][2][32];  // per warp: each lane's 8 states before token j (slot j)
    float4 tab[kConsumerWarps][kRevChunk][16];      // per warp: (Delta, u, ds, dy SiLU'(z)) of its channels
    float acc[2][kRevChunk][32];                    // dB | dC of the tile's channels, per sub-chunk parity
    int4 meta[kRevStages];                          // {unit, t0, tcount, flags}
    uint64_t full[kRevStages], ready[kRevStages], empty[kRevStages];
    uint64_t csync;  // the consumer warps meet once per sub-chunk (dB / dC sums complete)
};

struct RevPos {
    int b, tile, seg, chain;
};

// Units in reverse segment-major order: every chain's last segment first.
__device__ __forceinline__ RevPos rev_pos(int u, const RevArgs &a) {
    const int per = a.Bt * a.tiles;
    RevPos p;
    const int r = u / per;
    p.seg = a.nseg - 1 - r;
    p.chain = u - r * per;
    p.b = p.chain / a.tiles;
    p.tile = p.chain - p.b * a.tiles;
    return p;
}

// Sum of 16 values per lane over the 16 lanes of a warp that share lane & 1
// (the warp's 16 channels), scattered so that each lane keeps one sum: lane l
// ends with output o = 16 * bit4(l) + 8 * (l & 1) + 4 * bit3(l) + 2 * bit2(l) +
// bit1(l) of v = (vB[0..7], vC[0..7]) indexed as (which, n0 + i).
__device__ __forceinline__ float reduce_scatter16(const float (&vB)[8], const float (&vC)[8], int lane) {
    const unsigned full = 0xffffffffu;
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
    float r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float keep = b4 ? vC[i] : vB[i];
        const float send = b4 ? vB[i] : vC[i];
        r[i] = keep + __shfl_xor_sync(full, send, 16);
    }
    float r2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float keep = b3 ? r[i + 4] : r[i];
        const float send = b3 ? r[i] : r[i + 4];
        r2[i] = keep + __shfl_xor_sync(full, send, 8);
    }
    float r3[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float keep = b2 ? r2[i + 2] : r2[i];
        const float send = b2 ? r2[i] : r2[i + 2];
        r3[i] = keep + __shfl_xor_sync(full, send, 4);
    }
    const float keep = b1 ? r3[1] : r3[0];
    const float send = b1 ? r3[0] : r3[1];
    return keep + __shfl_xor_sync(full, send, 2);
}

__device__ __forceinline__ int reduce_scatter16_index(int lane) {
    return 16 * ((lane >> 4) & 1) + 8 * (lane & 1) + 4 * ((lane >> 3) & 1) + 2 * ((lane >> 2) & 1) + ((lane >> 1) & 1);
}

// d gain / dA at fixed Delta for the exact ZOH write, gain = (e^x - 1)/A with
// x = Delta A: (x e^x - (e^x - 1))/A^2 = Delta^2 (1/2 + x/3 + x^2/8 + x^3/30 +
// ...).  The closed form cancels in float32 as x -> 0: its two terms carry
// errors of about 2^-22 |x| against a difference of about x^2/2, i.e. about
// 1e-6/|x| relative; the series to x^2 is used for |x| < 1/16, where its
// truncation (x^3/30 against 1/2) is below 2e-5 relative and the closed form's
// error above 1.5e-5.  e^x is the decay a; 1/A^2 is taken as nrA^2 with
// nrA = -1/A, which the walk holds per state, instead of a division per state
// and token.
__device__ __forceinline__ float zoh_dgain_dA_rev(float x, float a, float delta, float nrA) {
    const float p = fmaf(fmaf(x, 0.125f, 1.0f / 3.0f), x, 0.5f);
    const float series = delta * delta * p;
    const float closed = (x * a - (a - 1.0f)) * (nrA * nrA);
    return fabsf(x) < 0.0625f ? series : closed;
}


// Registers: the register file is allotted per SM sub-partition (16,384
// each), and two CTAs of five warps put two warps of a CTA on one of them, so
// 168 a thread is the most that keeps two CTAs per SM (the exact-ZOH fused
// instantiation would otherwise take 181 and run one CTA per SM).
template <typename IO, bool ZOH, bool CONV>
__global__ void __maxnreg__(168)
    s6_scan_bwd_rev_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_dt,
                           const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_dy,
                           const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_C,
                           const RevArgs a) {
    using Smem = RevSmem<IO, CONV>;
    using tr = io_traits<IO>;
    constexpr int KC = kRevChunk;
    constexpr int XR = Smem::XR;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const unsigned full = 0xffffffffu;

    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < kRevStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.ready[s], 1);
            mbar_init(&sm.empty[s], kConsumerWarps);
        }
        mbar_init(&sm.csync, kConsumerWarps);
        fence_mbarrier_init();
    }
    for (int i = tid; i < 2 * KC * 32; i += blockDim.x)
        (&sm.acc[0][0][0])[i] = 0.0f;
    __syncthreads();

    if (warp == kConsumerWarps) {
        // =========================================================== producer
        // (its waits sleep between polls, leaving the issue slots to the consumers)
        if (lane == 0) {
            prefetch_tensormap(&tm_x);
            prefetch_tensormap(&tm_dt);
            prefetch_tensormap(&tm_dy);
            prefetch_tensormap(&tm_B);
            prefetch_tensormap(&tm_C);
            if (a.has_z)
                prefetch_tensormap(&tm_z);
        }
        int unit = -1, k = -1, ta = 0, tb = 0;
        bool first_pull = true;
        for (int c = 0;; ++c) {
            const int s = c % kRevStages;
            bool ok = true;
            if (c >= kRevStages) {
                bool got = true;
                if (lane == 0)
                    got = mbar_wait_sleep_bounded(&sm.empty[s], ((c / kRevStages) - 1) & 1, kSleepPolls, kSleepNs);
                ok = __shfl_sync(full, got ? 1 : 0, 0) != 0;
                if (!ok && lane == 0)
                    raise_device_error(1u);
            }
            bool start = false;
            if (ok && k < 0) {
                int u = 0;
                if (lane == 0)
                    u = a.dynamic ? static_cast<int>(atomicAdd(a.counter, 1u))
                                  : (first_pull ? static_cast<int>(blockIdx.x) : a.units);
                u = __shfl_sync(full, u, 0);
                first_pull = false;
                if (u < a.units) {
                    const RevPos rp = rev_pos(u, a);
                    unit = u;
                    ta = rp.seg * a.seg_len;
                    tb = min(a.L, ta + a.seg_len);
                    k = (tb - ta + KC - 1) / KC - 1;
                    start = true;
                } else {
                    unit = -1;
                }
            }
            if (!ok || unit < 0) {
                if (lane == 0) {
                    sm.meta[s] = make_int4(-1, 0, 0, kMetaEnd);
                    mbar_arrive(&sm.ready[s]);
                }
                break;
            }
            const RevPos rp = rev_pos(unit, a);
            const int t0 = ta + k * KC;
            const int fl = (start ? kMetaFirst : 0) | (k == 0 ? kMetaLast : 0);
            if (start && a.dynamic && rp.seg + 1 < a.nseg) {
                // dLoss/dh entering the segment from the right: one flag per consumer warp
                bool got = true;
                if (lane < kConsumerWarps) {
                    got = false;
                    const unsigned int *f = &a.flags[static_cast<size_t>(rp.chain) * kConsumerWarps + lane];
                    const unsigned int need = static_cast<unsigned int>(a.nseg - 1 - rp.seg);
                    for (uint32_t i = 0; i < a.carry_polls; ++i) {
                        if (ld_acquire_gpu(f) >= need) {
                            got = true;
                            break;
                        }
                        __nanosleep(64);
                    }
                }
                if (!__all_sync(full, got) && lane == 0)
                    raise_device_error(2u);
            }
            if (lane == 0) {
                sm.meta[s] = make_int4(unit, t0, min(KC, tb - t0), fl);
                const int c0 = rp.tile * 64;
                constexpr uint32_t kX = XR * 64 * sizeof(IO);
                constexpr uint32_t kR = KC * 64 * sizeof(IO);
                constexpr uint32_t kBC = 2u * KC * 16 * sizeof(IO);
                mbar_arrive_expect_tx(&sm.full[s], kX + 2 * kR + (a.has_z ? kR : 0u) + kBC);
                tma_load_3d(&sm.x[s].v[0][0], &tm_x, &sm.full[s], c0, t0 - (CONV ? kHalo : 0), rp.b);
                tma_load_3d(&sm.dt[s].v[0][0], &tm_dt, &sm.full[s], c0, t0, rp.b);
                tma_load_3d(&sm.dy[s].v[0][0], &tm_dy, &sm.full[s], c0, t0, rp.b);
                if (a.has_z)
                    tma_load_3d(&sm.z[s].v[0][0], &tm_z, &sm.full[s], c0, t0, rp.b);
                tma_load_3d(&sm.braw[s].v[0][0], &tm_B, &sm.full[s], 0, t0, rp.b);
                tma_load_3d(&sm.craw[s].v[0][0], &tm_C, &sm.full[s], 0, t0, rp.b);
            }
            // B / C rows to float32 once the tile has landed, then the stage is ready
            bool got = true;
            if (lane == 0)
                got = mbar_wait_sleep_bounded(&sm.full[s], (c / kRevStages) & 1, kSleepPolls, kSleepNs);
            got = __shfl_sync(full, got ? 1 : 0, 0) != 0;
            if (!got && lane == 0)
                raise_device_error(1u);
            {
                // each step fills one 512-byte group of bc (4 tokens x B|C x 16
                // states), lane l its bytes [16 l, 16 l + 16): token l / 8 of the
                // group, B or C by bit 2, states 4 (l & 3) .. +3
                const int which = (lane >> 2) & 1;
                const int n4 = (lane & 3) * 4;
                const int tl = lane >> 3;
                const IO *src = (which ? &sm.craw[s].v[0][0] : &sm.braw[s].v[0][0]) + tl * 16 + n4;
                float *dst = &sm.bc[s][tl][which][n4];
#pragma unroll
                for (int i = 0; i < KC / 4; ++i) {
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (got) {
                        if constexpr (sizeof(IO) == 2) {
                            const uint2 r = *reinterpret_cast<const uint2 *>(src + i * 64);
                            v = make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xffff0000u),
                                            __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xffff0000u));
                        } else {
                            v = *reinterpret_cast<const float4 *>(src + i * 64);
                        }
                    }
                    *reinterpret_cast<float4 *>(dst + i * 128) = v;
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.ready[s]);
            --k;
        }
        return;
    }

    // ============================================================== consumers
    const int cw = lane >> 1;        // channel within the warp
    const int sub = lane & 1;        // which 8 states of the channel
    const int cl = warp * 16 + cw;   // channel within the tile
    const int n0 = sub * 8;
    const int o_lane = reduce_scatter16_index(lane);
    const f2_t zero2 = f2_pack(0.f, 0.f);

    f2_t A2p[4], Ap[4], nrAp[4], gcar[4], dAacc[4];
    float Dd = 0.f, bias = 0.f, w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, cbv = 0.f;
    float dDa = 0.f, dba = 0.f, dW0 = 0.f, dW1 = 0.f, dW2 = 0.f, dW3 = 0.f, dcb = 0.f;
    float dp1 = 0.f, dp2 = 0.f, dp3 = 0.f;  // dpre of the next three tokens
    int b = 0, tile = 0, seg = 0, chain = 0, ch = 0;
    bool live = false;
#pragma unroll
    for (int q = 0; q < 4; ++q)
        A2p[q] = Ap[q] = nrAp[q] = gcar[q] = dAacc[q] = zero2;

    // the unit's parameter gradients: the two threads of a channel hold the same
    // per-channel sums (the first adds them), each its own states' dA
    auto flush_params = [&]() {
        if (!live)
            return;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float v0, v1, A0, A1;
            f2_unpack(dAacc[q], v0, v1);
            f2_unpack(Ap[q], A0, A1);
            atomicAdd(a.dA_log + static_cast<size_t>(ch) * 16 + n0 + 2 * q, v0 * A0);  // dA/dA_log = A
            atomicAdd(a.dA_log + static_cast<size_t>(ch) * 16 + n0 + 2 * q + 1, v1 * A1);
        }
        if (sub == 0) {
            atomicAdd(a.dD + ch, dDa);
            if (a.ddt_bias)
                atomicAdd(a.ddt_bias + ch, dba);
            if (CONV) {
                const float dWv[4] = {dW0, dW1, dW2, dW3};
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int src = kk - (4 - a.K);
                    if (src >= 0)
                        atomicAdd(a.dconv_w + static_cast<size_t>(ch) * a.K + src, dWv[kk]);
                }
                if (a.dconv_b)
                    atomicAdd(a.dconv_b + ch, dcb);
            }
        }
    };

    for (int c = 0;; ++c) {
        const int s = c % kRevStages;
        const bool got = mbar_wait_bounded(&sm.ready[s], (c / kRevStages) & 1, kWaitPolls);
        if (!__all_sync(full, got)) {
            if (lane == 0)
                raise_device_error(1u);
            break;
        }
        const int4 m = sm.meta[s];
        if (m.w & kMetaEnd)
            break;
        const int t0 = m.y, tcount = m.z;

        if (m.w & kMetaFirst) {
            // ---- a new unit: channel parameters and the carry from the right
            const RevPos rp = rev_pos(m.x, a);
            b = rp.b;
            tile = rp.tile;
            seg = rp.seg;
            chain = rp.chain;
            ch = tile * 64 + cl;
            live = ch < a.d;
            const int chc = live ? ch : 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float al[2], nr[2], av[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float A = -expf(a.A_log[static_cast<size_t>(chc) * 16 + n0 + 2 * q + e]);  // A = -exp(A_log)
                    av[e] = A;
                    al[e] = A * kLog2e;
                    nr[e] = -1.0f / A;
                }
                A2p[q] = f2_pack(al[0], al[1]);
                Ap[q] = f2_pack(av[0], av[1]);
                nrAp[q] = f2_pack(nr[0], nr[1]);
                dAacc[q] = zero2;
            }
            Dd = a.D[chc];
            bias = a.dt_bias ? a.dt_bias[chc] : 0.0f;
            if (CONV) {
                float wv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int src = kk - (4 - a.K);
                    wv[kk] = src >= 0 ? a.conv_w[static_cast<size_t>(chc) * a.K + src] : 0.0f;
                }
                w0 = wv[0];
                w1 = wv[1];
                w2 = wv[2];
                w3 = wv[3];
                cbv = a.conv_b ? a.conv_b[chc] : 0.0f;
            }
            dDa = dba = dW0 = dW1 = dW2 = dW3 = dcb = 0.f;
            if (a.dynamic && seg + 1 < a.nseg) {
                const float *cp = a.carry + (static_cast<size_t>(chain) * 64 + cl) * kRevCarry;
                const float4 g0 = __ldcg(reinterpret_cast<const float4 *>(cp + n0));
                const float4 g1 = __ldcg(reinterpret_cast<const float4 *>(cp + n0 + 4));
                gcar[0] = f2_pack(g0.x, g0.y);
                gcar[1] = f2_pack(g0.z, g0.w);
                gcar[2] = f2_pack(g1.x, g1.y);
                gcar[3] = f2_pack(g1.z, g1.w);
                const float4 wdp = __ldcg(reinterpret_cast<const float4 *>(cp + 16));
                dp1 = wdp.x;
                dp2 = wdp.y;
                dp3 = wdp.z;
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    gcar[q] = zero2;
                dp1 = dp2 = dp3 = 0.f;
            }
        }

        // ---- the checkpoint: the state before token t0 (read now, used after the scalars)
        float4 ck0 = make_float4(0.f, 0.f, 0.f, 0.f), ck1 = ck0;
        if (live) {
            const float *cp = a.ckpt + ((static_cast<size_t>(b) * a.nck + t0 / KC) * a.d + ch) * 16 + n0;
            ck0 = __ldcg(reinterpret_cast<const float4 *>(cp));
            ck1 = __ldcg(reinterpret_cast<const float4 *>(cp + 4));
        }
        const IO(*xs)[64] = sm.x[s].v;
        const IO(*dts)[64] = sm.dt[s].v;
        const IO(*zs)[64] = sm.z[s].v;
        const IO(*dys)[64] = sm.dy[s].v;
        const float(*bc)[2][16] = sm.bc[s];
        float4(*hb)[2][32] = sm.hbuf[warp];
        float4(*tb)[16] = sm.tab[warp];
        auto ld = [&](const IO(*t)[64], int row) { return tr::to_f(t[row][cl]); };
        auto pre_at = [&](int j) {  // conv pre-activation of token t0 + j (x rows j .. j+3)
            return fmaf(w3, ld(xs, j + 3), fmaf(w2, ld(xs, j + 2), fmaf(w1, ld(xs, j + 1), fmaf(w0, ld(xs, j), cbv))));
        };

        // ---- 1. the per-token scalars of the sub-chunk, once per (token, channel):
        // each thread of a pair takes half of the tokens, two at a time (j and
        // j + 2) in packed arithmetic -- the forward's own softplus and SiLU
        for (int j = sub; j < tcount; j += 4) {
            const int j2 = min(j + 2, KC - 1);  // a partial sub-chunk's spare lane reads a row it does not store
            const f2_t v2 = f2_add(f2_pack(ld(dts, j), ld(dts, j2)), f2_pack(bias, bias));
            const f2_t d2 = f2_softplus_fast(v2);
            const f2_t u2 = CONV ? f2_silu_fast(f2_pack(pre_at(j), pre_at(j2))) : f2_pack(ld(xs, j), ld(xs, j2));
            const f2_t dy2 = f2_pack(ld(dys, j), ld(dys, j2));
            f2_t g2 = f2_pack(1.0f, 1.0f), gp2 = f2_pack(0.0f, 0.0f);
            if (a.has_z) {
                const float za = ld(zs, j), zb = ld(zs, j2);
                // sigmoid(z), SiLU(z) = z sigmoid(z), SiLU'(z) = sigmoid(z) (1 + z (1 - sigmoid(z)))
                const f2_t sz = f2_pack(rcp_approx(1.0f + ex2_approx(fminf(-za * kLog2e, 120.0f))),
                                        rcp_approx(1.0f + ex2_approx(fminf(-zb * kLog2e, 120.0f))));
                const f2_t z2 = f2_pack(za, zb);
                g2 = f2_mul(z2, sz);
                gp2 = f2_mul(sz, f2_fma(z2, f2_sub(f2_pack(1.0f, 1.0f), sz), f2_pack(1.0f, 1.0f)));
            }
            float da, db, ua, ub, ga, gb, pa, pb;
            f2_unpack(d2, da, db);
            f2_unpack(u2, ua, ub);
            f2_unpack(f2_mul(dy2, g2), ga, gb);
            f2_unpack(f2_mul(dy2, gp2), pa, pb);
            tb[j][cw] = make_float4(da, ua, ga, pa);
            if (j + 2 < tcount)
                tb[j + 2][cw] = make_float4(db, ub, gb, pb);
        }
        __syncwarp();

        float *accp = &sm.acc[c & 1][0][0];  // this sub-chunk's dB / dC sums
        // phases 2 and 3 over the sub-chunk's tokens; a full sub-chunk takes a
        // compile-time trip count
        auto phases = [&](auto full_tag) {
            constexpr bool FULL = decltype(full_tag)::value;
            const int tc = FULL ? KC : tcount;
            // ---- 2. recompute the sub-chunk forward from the checkpoint; keep every state
            {
                hb[0][0][lane] = ck0;
                hb[0][1][lane] = ck1;
                f2_t h[4] = {f2_pack(ck0.x, ck0.y), f2_pack(ck0.z, ck0.w), f2_pack(ck1.x, ck1.y), f2_pack(ck1.z, ck1.w)};
#pragma unroll 2
                for (int j = 0; j < tc; ++j) {
                    const float4 du = tb[j][cw];
                    const f2_t dd = f2_pack(du.x, du.x);
                    const f2_t uu = f2_pack(du.y, du.y);
                    const f2_t wdu = f2_mul(dd, uu);
                    const ulonglong2 B01 = *reinterpret_cast<const ulonglong2 *>(&bc[j][0][n0]);
                    const ulonglong2 B23 = *reinterpret_cast<const ulonglong2 *>(&bc[j][0][n0 + 4]);
                    const f2_t Bq[4] = {B01.x, B01.y, B23.x, B23.y};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float x0, x1;
                        f2_unpack(f2_mul(dd, A2p[q]), x0, x1);
                        const f2_t ab = f2_pack(ex2_approx(x0), ex2_approx(x1));
                        if (ZOH) {
                            const f2_t nk = f2_mul(nrAp[q], f2_mul(uu, Bq[q]));
                            h[q] = f2_fma(ab, f2_sub(h[q], nk), nk);
                        } else {
                            h[q] = f2_fma(ab, h[q], f2_mul(wdu, Bq[q]));
                        }
                    }
                    float a0, a1, a2, a3, a4, a5, a6, a7;
                    f2_unpack(h[0], a0, a1);
                    f2_unpack(h[1], a2, a3);
                    f2_unpack(h[2], a4, a5);
                    f2_unpack(h[3], a6, a7);
                    hb[j + 1][0][lane] = make_float4(a0, a1, a2, a3);
                    hb[j + 1][1][lane] = make_float4(a4, a5, a6, a7);
                }
            }
            __syncwarp();

            // ---- 3. walk the sub-chunk back
            // h_t of the token being walked back; h_{t-1} becomes the next token's h_t
            float4 h0 = hb[tc][0][lane], h1 = hb[tc][1][lane];
            // the conv window: x rows j+1 .. j+3 of token j kept from the token
            // after it, so that each token reads one new row (row j)
            float xr1 = 0.f, xr2 = 0.f, xr3 = 0.f;
            if (CONV) {
                xr1 = ld(xs, tc);
                xr2 = ld(xs, tc + 1);
                xr3 = ld(xs, tc + 2);
            }
#pragma unroll 2
            for (int j = tc - 1; j >= 0; --j) {
                const float4 du = tb[j][cw];
                const float delta = du.x, u = du.y, ds = du.z, dygp = du.w;
                // softplus'(v) = sigmoid(v) = 1 - e^-Delta (Delta = softplus(v))
                const float sig_v = 1.0f - ex2_approx(-delta * kLog2e);
                const float4 p0 = hb[j][0][lane], p1 = hb[j][1][lane];  // h_{t-1}
                const f2_t ht[4] = {f2_pack(h0.x, h0.y), f2_pack(h0.z, h0.w), f2_pack(h1.x, h1.y), f2_pack(h1.z, h1.w)};
                const f2_t hp[4] = {f2_pack(p0.x, p0.y), f2_pack(p0.z, p0.w), f2_pack(p1.x, p1.y), f2_pack(p1.z, p1.w)};
                const ulonglong2 B01 = *reinterpret_cast<const ulonglong2 *>(&bc[j][0][n0]);
                const ulonglong2 B23 = *reinterpret_cast<const ulonglong2 *>(&bc[j][0][n0 + 4]);
                const ulonglong2 C01 = *reinterpret_cast<const ulonglong2 *>(&bc[j][1][n0]);
                const ulonglong2 C23 = *reinterpret_cast<const ulonglong2 *>(&bc[j][1][n0 + 4]);
                const f2_t Bq[4] = {B01.x, B01.y, B23.x, B23.y};
                const f2_t Cq[4] = {C01.x, C01.y, C23.x, C23.y};
                const f2_t dsv = f2_pack(ds, ds);
                const f2_t dd = f2_pack(delta, delta);
                const f2_t uu = f2_pack(u, u);
                const f2_t wdu = f2_mul(dd, uu);
                f2_t acc_s = zero2, acc_b = zero2, acc_q = zero2, acc_z = zero2;
                float vB[8], vC[8];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float x0, x1;
                    f2_unpack(f2_mul(dd, A2p[q]), x0, x1);
                    const f2_t ab = f2_pack(ex2_approx(x0), ex2_approx(x1));
                    const f2_t dh = f2_fma(dsv, Cq[q], gcar[q]);
                    acc_s = f2_fma(ht[q], Cq[q], acc_s);
                    const f2_t dC2 = f2_mul(dsv, ht[q]);
                    f2_t dB2;
                    if (ZOH) {
                        const f2_t gain = f2_mul(f2_sub(f2_pack(1.f, 1.f), ab), nrAp[q]);  // (a - 1)/A
                        const f2_t dhB = f2_mul(dh, Bq[q]);
                        dB2 = f2_mul(f2_mul(dh, gain), uu);
                        acc_b = f2_fma(dhB, gain, acc_b);
                        acc_z = f2_fma(dhB, ab, acc_z);  // dgain/dDelta = a
                    } else {
                        dB2 = f2_mul(dh, wdu);
                        acc_b = f2_fma(dh, Bq[q], acc_b);
                    }
                    const f2_t qv = f2_mul(f2_mul(dh, hp[q]), ab);  // dh h_{t-1} a
                    acc_q = f2_fma(qv, Ap[q], acc_q);
                    dAacc[q] = f2_fma(qv, dd, dAacc[q]);
                    if (ZOH) {
                        float g0, g1, A0, A1, nr0, nr1, ab0, ab1, dhb0, dhb1;
                        f2_unpack(Ap[q], A0, A1);
                        f2_unpack(nrAp[q], nr0, nr1);
                        f2_unpack(ab, ab0, ab1);
                        f2_unpack(f2_mul(f2_mul(dh, Bq[q]), uu), dhb0, dhb1);
                        g0 = dhb0 * zoh_dgain_dA_rev(delta * A0, ab0, delta, nr0);
                        g1 = dhb1 * zoh_dgain_dA_rev(delta * A1, ab1, delta, nr1);
                        dAacc[q] = f2_add(dAacc[q], f2_pack(g0, g1));
                    }
                    gcar[q] = f2_mul(dh, ab);
                    f2_unpack(dB2, vB[2 * q], vB[2 * q + 1]);
                    f2_unpack(dC2, vC[2 * q], vC[2 * q + 1]);
                }
                // sums over the channel's 16 states: this thread's 8, then the partner's
                float s0, s1, b0, b1, q0, q1, z0, z1;
                f2_unpack(acc_s, s0, s1);
                f2_unpack(acc_b, b0, b1);
                f2_unpack(acc_q, q0, q1);
                f2_unpack(acc_z, z0, z1);
                float sp = s0 + s1, bp = b0 + b1, qp = q0 + q1;
                sp += __shfl_xor_sync(full, sp, 1);
                bp += __shfl_xor_sync(full, bp, 1);
                qp += __shfl_xor_sync(full, qp, 1);
                float zp = 0.f;
                if (ZOH) {
                    zp = z0 + z1;
                    zp += __shfl_xor_sync(full, zp, 1);
                }
                const float s_tot = fmaf(Dd, u, sp);
                const float dut = ZOH ? fmaf(ds, Dd, bp) : fmaf(ds, Dd, delta * bp);
                const float ddel = ZOH ? fmaf(u, zp, qp) : fmaf(u, bp, qp);
                const float dv = ddel * sig_v;
                float dxo = dut;
                if (CONV) {
                    const float xr0 = ld(xs, j);
                    const float pre = fmaf(w3, xr3, fmaf(w2, xr2, fmaf(w1, xr1, fmaf(w0, xr0, cbv))));
                    const float sp_ = rcp_approx(1.0f + ex2_approx(fminf(-pre * kLog2e, 120.0f)));
                    const float dpre = dut * sp_ * fmaf(pre, 1.0f - sp_, 1.0f);  // SiLU'(pre)
                    dxo = fmaf(w3, dpre, fmaf(w2, dp1, fmaf(w1, dp2, w0 * dp3)));
                    dW0 = fmaf(dpre, xr0, dW0);
                    dW1 = fmaf(dpre, xr1, dW1);
                    dW2 = fmaf(dpre, xr2, dW2);
                    dW3 = fmaf(dpre, xr3, dW3);
                    xr3 = xr2;
                    xr2 = xr1;
                    xr1 = xr0;
                    dcb += dpre;
                    dp3 = dp2;
                    dp2 = dp1;
                    dp1 = dpre;
                }
                dDa = fmaf(ds, u, dDa);
                dba += dv;
                // the token's outputs, written out by the warp after the walk (this
                // tab row is not read again)
                if (sub == 0)
                    tb[j][cw] = make_float4(dxo, dv, dygp * s_tot, 0.f);
                // dB, dC of token t0 + j summed over the warp's channels, then the CTA's
                const float r = reduce_scatter16(vB, vC, lane);
                atomicAdd(accp + j * 32 + o_lane, r);
                h0 = p0;
                h1 = p1;
            }
        };
        if (tcount == KC)
            phases(std::true_type{});
        else
            phases(std::false_type{});

        // du, ddt, dz of the sub-chunk from the tab rows: lanes 0-15 one token,
        // 16-31 the next, each a channel -- 64-byte runs per token and output
        __syncwarp();
        {
            const int wc = tile * 64 + warp * 16 + (lane & 15);
            if (wc < a.d) {
                for (int j = lane >> 4; j < tcount; j += 2) {
                    const float4 v = tb[j][lane & 15];
                    const size_t o = (static_cast<size_t>(b) * a.L + t0 + j) * a.d + wc;
                    a.du[o] = v.x;
                    a.ddt[o] = v.y;
                    if (a.has_z)
                        a.dz[o] = v.z;
                }
            }
        }

        // release the stage (its tiles are no longer read)
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sm.empty[s]);

        // ---- 4. the tile's dB / dC rows of this sub-chunk to the partial buffer, once
        // every consumer warp has added its share (a bounded wait on an mbarrier)
        if (lane == 0)
            mbar_arrive(&sm.csync);
        if (!__all_sync(full, mbar_wait_bounded(&sm.csync, c & 1, kWaitPolls))) {
            if (lane == 0)
                raise_device_error(1u);
            break;
        }
        {
            float *dst = a.part + ((static_cast<size_t>(tile) * a.Bt + b) * a.L + t0) * 32;
            for (int i = tid; i < KC * 32; i += kScanThreads) {
                if (i < tcount * 32)
                    dst[i] = accp[i];
                accp[i] = 0.0f;
            }
        }

        if (m.w & kMetaLast) {
            // ---- the unit's first token is done: hand dLoss/dh (and the dpre window) to the left
            if (a.dynamic && seg > 0) {
                float *cp = a.carry + (static_cast<size_t>(chain) * 64 + cl) * kRevCarry;
                float g[8];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    f2_unpack(gcar[q], g[2 * q], g[2 * q + 1]);
                __stcg(reinterpret_cast<float4 *>(cp + n0), make_float4(g[0], g[1], g[2], g[3]));
                __stcg(reinterpret_cast<float4 *>(cp + n0 + 4), make_float4(g[4], g[5], g[6], g[7]));
                if (sub == 0)
                    __stcg(reinterpret_cast<float4 *>(cp + 16), make_float4(dp1, dp2, dp3, 0.f));
                __syncwarp();
                if (lane == 0) {
                    __threadfence();
                    st_release_gpu(&a.flags[static_cast<size_t>(chain) * kConsumerWarps + warp],
                                   static_cast<unsigned int>(a.nseg - seg));
                }
            } else if (seg == 0 && a.dh_init && live) {
                float g[8];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    f2_unpack(gcar[q], g[2 * q], g[2 * q + 1]);
                float *hp = a.dh_init + (static_cast<size_t>(b) * a.d + ch) * 16 + n0;
                *reinterpret_cast<float4 *>(hp) = make_float4(g[0], g[1], g[2], g[3]);
                *reinterpret_cast<float4 *>(hp + 4) = make_float4(g[4], g[5], g[6], g[7]);
            }
            flush_params();
        }
    }
}

// dB, dC = sums over the channel tiles of the partial rows.
__global__ void s6_bwd_bc_reduce_kernel(const float *part, int tiles, long long rows, float *dB, float *dC) {
    const long long total = rows * 32;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        float sum = 0.f;
        for (int t = 0; t < tiles; ++t)
            sum += __ldcs(part + static_cast<long long>(t) * total + i);
        const long long r = i >> 5;
        const int o = static_cast<int>(i & 31);
        if (o < 16)
            dB[r * 16 + o] = sum;
        else
            dC[r * 16 + o - 16] = sum;
    }
}

}  // namespace s6
