// s6_scan.cuh -- full-sequence selective scan (optionally fused with the
// causal depthwise conv + SiLU in front of it), sm_100a.
//
// The recurrence ("mamba, live", what is actually running; "the s6 cell", the
// recurrence), per batch b, channel d, token t, state coordinate n:
//     u      = SiLU(conv_b + sum_k w[k] x[t-3+k])     (fused form) or u = u_t
//     Delta  = softplus(dt_t + dt_bias)
//     A_bar  = 2^(Delta * A[n] * log2 e),  A = -exp(A_log)
//     write  = Delta * B_t[n] * u                      (zoh_mode 0)
//            = (A_bar - 1) / A[n] * B_t[n] * u         (zoh_mode 1, exact ZOH of
//              "Carry context through a selective state")
//     h[n]   = A_bar * h[n] + write
//     y      = (sum_n h[n] C_t[n] + D u) * SiLU(z_t)   (C reads the updated state)
//
// Work decomposition.  TPC threads share one channel (TPC = 2 at N = 16:
// each keeps NH = N/TPC float32 states in registers), so a CTA of 128
// threads owns CPB = 128/TPC consecutive channels of one sequence.  A
// sequence's channel tile is a chain of segments of seg_len tokens; a
// (segment, tile) pair is a unit of work.  In the dynamic mode persistent
// CTAs pull units, segment-major, from a global counter; a unit whose segment
// is not the first waits (bounded) for the state its predecessor publishes in
// a carry buffer -- the predecessor was pulled earlier by a running CTA, so
// the wait always ends.  This spreads B*d/CPB chains evenly over every SM
// whatever their count, without recomputing a single decay.  In the static
// mode (plenty of chains) each CTA runs one whole chain.
//
// Data movement.  Per chunk of T tokens one elected thread issues TMA tile
// loads of the [T(+3 halo) x CPB] slices of x, dt and z and the [T x N] rows
// of B and C into a STAGES-deep shared-memory ring (mbarrier completion; the
// chunk's unit, first token and flags travel with it in shared memory).  The
// 3 halo rows give the conv its K-1 earlier inputs; rows before token 0 are
// zero-filled by the TMA unit (the conv's zero left padding).  B/C rows are
// converted once per chunk to float32 (shared by all channels); each thread
// reads its channel column and the broadcast B/C rows and writes y into a
// triple-buffered tile that the elected thread stores with a TMA bulk store.
//
// Arithmetic.  The 16 decays per element are the binding work (one live
// exponential per state per token, "the s6 cell").  They go to the MUFU ex2
// pipe; SiLU and softplus use one MUFU op each, with their reciprocal and
// log1p on the FMA pipe; with TPC = 2 the two threads of a channel split the
// two SiLUs (conv output, gate) and exchange them with one shuffle.  State
// arithmetic runs on packed float32 pairs (f32x2).  Scalars of token j+1 are
// computed before the state update of token j to give the scheduler
// independent work.
//
// No tensor cores: the recurrence is diagonal (an elementwise product with a
// data-dependent decay), not a contraction.
#pragma once

#include "s6_common.cuh"

namespace s6 {

constexpr int kScanThreads = 128;
constexpr int kHalo = 3;  // conv history rows (taps padded to 4)

constexpr int kMetaFirst = 1;  // first chunk of its unit
constexpr int kMetaLast = 2;   // last chunk of its unit
constexpr int kMetaEnd = 4;    // no more work

struct ScanArgs {
    int Bt, L, d, N, K;
    int has_z;
    int tiles;    // channel tiles per sequence
    int nseg;     // segments per sequence
    int seg_len;  // tokens per segment (a multiple of the chunk length)
    int units;    // Bt * tiles * nseg
    int dynamic;  // 1: persistent CTAs pull units from *counter
    int bc_tma;   // 1: B/C rows arrive by TMA with the stage
    const void *B;  // [Bt, L, N] io (read directly when bc_tma == 0)
    const void *C;
    const float *A_log;    // [d, N]
    const float *D;        // [d]
    const float *dt_bias;  // [d] or null
    const float *conv_w;   // [d, K] taps, oldest first (fused form), else null
    const float *conv_b;   // [d] or null
    float *h_final;        // [Bt, d, N] or null
    unsigned int *counter;  // dynamic: next unit to hand out (zeroed before launch)
    unsigned int *flags;    // dynamic: [Bt*tiles] segments whose end state is published
    float *carry;           // dynamic: [Bt*tiles][CPB][NS] published end states
};

template <int NS, int TPC, int T, bool CONV>
struct ScanShape {
    static constexpr int NH = NS / TPC;             // states per thread
    static constexpr int CPB = kScanThreads / TPC;  // channels per CTA
    static constexpr int XR = T + (CONV ? kHalo : 0);
    static_assert(NH % 4 == 0, "states per thread must be a multiple of 4");
};

template <typename IO, int NS, int TPC, int T, int STAGES, bool CONV>
struct ScanSmem {
    using Sh = ScanShape<NS, TPC, T, CONV>;
    IO x[STAGES][Sh::XR][Sh::CPB];
    IO dt[STAGES][T][Sh::CPB];
    IO z[STAGES][T][Sh::CPB];
    IO y[3][T][Sh::CPB];
    IO braw[STAGES][T * NS];
    IO craw[STAGES][T * NS];
    float bc[2][T][2][NS];  // [buffer][token][B|C][n], float32, zero-padded to NS
    int4 meta[STAGES];      // {unit, t0, tcount, flags}
    uint64_t full[STAGES];
};

struct UnitPos {
    int b, tile, seg, chain;
};

__device__ __forceinline__ UnitPos unit_pos(int u, const ScanArgs &a) {
    const int per = a.Bt * a.tiles;
    UnitPos p;
    p.seg = u / per;
    p.chain = u - p.seg * per;
    p.b = p.chain / a.tiles;
    p.tile = p.chain - p.b * a.tiles;
    return p;
}

// Per-token scalars of one channel.
struct TokScalars {
    float u, delta, g;
};

template <typename IO, int NS, int TPC, int T, int STAGES, bool CONV, bool ZOH>
__global__ void __launch_bounds__(kScanThreads, 2)
    s6_scan_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_dt,
                   const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_y,
                   const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_C,
                   const ScanArgs a) {
    using Sh = ScanShape<NS, TPC, T, CONV>;
    using Smem = ScanSmem<IO, NS, TPC, T, STAGES, CONV>;
    using tr = io_traits<IO>;
    constexpr int NH = Sh::NH;
    constexpr int NP = NH / 2;  // state pairs per thread
    constexpr int CPB = Sh::CPB;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);

    const int tid = threadIdx.x;
    const int cl = tid / TPC;                    // channel within the tile
    const int half = (TPC == 2) ? (tid & 1) : 0;  // which NH states of the channel
    const int n0 = half * NH;

    // ------------------------------------------------ producer (thread 0 only)
    int p_unit = -1, p_k = 0, p_nk = 0, p_tlo = 0, p_thi = 0, p_count = 0;
    bool p_done = false, p_first_pull = true;
    auto pull_unit = [&]() {
        int u;
        if (a.dynamic) {
            u = static_cast<int>(atomicAdd(a.counter, 1u));
        } else {
            u = p_first_pull ? static_cast<int>(blockIdx.x) : a.units;
        }
        p_first_pull = false;
        if (u >= a.units) {
            p_done = true;
            return;
        }
        const UnitPos up = unit_pos(u, a);
        p_unit = u;
        p_k = 0;
        p_tlo = up.seg * a.seg_len;
        p_thi = min(a.L, p_tlo + a.seg_len);
        p_nk = (p_thi - p_tlo + T - 1) / T;
    };
    auto produce = [&](int s) {
        ++p_count;
        if (!p_done && p_k == p_nk)
            pull_unit();
        if (p_done) {
            sm.meta[s] = make_int4(-1, 0, 0, kMetaEnd);
            mbar_arrive(&sm.full[s]);
            return;
        }
        const UnitPos up = unit_pos(p_unit, a);
        const int t0 = p_tlo + p_k * T;
        const int fl = (p_k == 0 ? kMetaFirst : 0) | (p_k == p_nk - 1 ? kMetaLast : 0);
        sm.meta[s] = make_int4(p_unit, t0, min(T, p_thi - t0), fl);
        const int c0 = up.tile * CPB;
        constexpr uint32_t kX = Sh::XR * CPB * sizeof(IO);
        constexpr uint32_t kR = T * CPB * sizeof(IO);
        const uint32_t kBC = a.bc_tma ? 2u * T * a.N * static_cast<uint32_t>(sizeof(IO)) : 0u;
        mbar_arrive_expect_tx(&sm.full[s], kX + kR + (a.has_z ? kR : 0u) + kBC);
        tma_load_3d(&sm.x[s][0][0], &tm_x, &sm.full[s], c0, t0 - (CONV ? kHalo : 0), up.b);
        tma_load_3d(&sm.dt[s][0][0], &tm_dt, &sm.full[s], c0, t0, up.b);
        if (a.has_z)
            tma_load_3d(&sm.z[s][0][0], &tm_z, &sm.full[s], c0, t0, up.b);
        if (a.bc_tma) {
            tma_load_3d(&sm.braw[s][0], &tm_B, &sm.full[s], 0, t0, up.b);
            tma_load_3d(&sm.craw[s][0], &tm_C, &sm.full[s], 0, t0, up.b);
        }
        ++p_k;
    };

    // B/C rows of a chunk -> float32 buffer (all threads; zero beyond N and L)
    auto stage_bc = [&](int s, int buf) {
        constexpr int kSlots = 2 * T * NS;
        const int4 m = sm.meta[s];
        if (m.w & kMetaEnd)
            return;
        const UnitPos up = unit_pos(m.x, a);
#pragma unroll
        for (int k = 0; k < (kSlots + kScanThreads - 1) / kScanThreads; ++k) {
            const int j = tid + k * kScanThreads;
            if (j < kSlots) {
                const int which = j / (T * NS);
                const int rem = j - which * (T * NS);
                const int tt = rem / NS;
                const int n = rem - tt * NS;
                float v = 0.0f;
                if (n < a.N && tt < m.z) {
                    if (a.bc_tma) {
                        v = tr::to_f(which ? sm.craw[s][tt * a.N + n] : sm.braw[s][tt * a.N + n]);
                    } else {
                        const size_t off = (static_cast<size_t>(up.b) * a.L + m.y + tt) * a.N + n;
                        v = tr::to_f(which ? static_cast<const IO *>(a.C)[off] : static_cast<const IO *>(a.B)[off]);
                    }
                }
                sm.bc[buf][tt][which][n] = v;
            }
        }
    };

    if (tid == 0) {
        prefetch_tensormap(&tm_x);
        prefetch_tensormap(&tm_dt);
        prefetch_tensormap(&tm_y);
        if (a.has_z)
            prefetch_tensormap(&tm_z);
        if (a.bc_tma) {
            prefetch_tensormap(&tm_B);
            prefetch_tensormap(&tm_C);
        }
#pragma unroll
        for (int s = 0; s < STAGES; ++s)
            mbar_init(&sm.full[s], 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s)
            produce(s);
    }

    // ------------------------------------------------ per-channel state
    f2_t hp[NP], A2p[NP], nrAp[NP];
    float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, cb = 0.f, Dd = 0.f, bias = 0.f;
    bool live = false;
    int chain = 0, seg = 0, bseq = 0, c0 = 0;
#pragma unroll
    for (int q = 0; q < NP; ++q)
        hp[q] = A2p[q] = nrAp[q] = f2_pack(0.f, 0.f);

    bool ok = mbar_wait_bounded(&sm.full[0], 0, 1u << 24);
    if (ok)
        stage_bc(0, 0);
    ok = !__syncthreads_or(!ok);
    if (!ok && tid == 0)
        raise_device_error(1u);

    int ci = 0;
    while (ok) {
        const int s = ci % STAGES;
        const int4 m = sm.meta[s];
        if (m.w & kMetaEnd)
            break;
        const UnitPos up = unit_pos(m.x, a);

        if (m.w & kMetaFirst) {
            // ---- a new unit: this thread's channel parameters and start state
            chain = up.chain;
            seg = up.seg;
            bseq = up.b;
            c0 = up.tile * CPB;
            const int ch = c0 + cl;
            live = ch < a.d;
            float wv[4] = {0.f, 0.f, 0.f, 0.f};
            if (CONV && live) {
                // taps right-aligned into 4 slots: width K is the width-4 conv
                // with its 4-K oldest taps zero, so the halo is always 3 rows
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int src = k - (4 - a.K);
                    wv[k] = (src >= 0) ? a.conv_w[static_cast<size_t>(ch) * a.K + src] : 0.0f;
                }
            }
            w0 = wv[0];
            w1 = wv[1];
            w2 = wv[2];
            w3 = wv[3];
            cb = (CONV && live && a.conv_b) ? a.conv_b[ch] : 0.0f;
            Dd = live ? a.D[ch] : 0.0f;
            bias = (live && a.dt_bias) ? a.dt_bias[ch] : 0.0f;
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                float al[2] = {0.f, 0.f}, nr[2] = {0.f, 0.f};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int n = n0 + 2 * q + e;
                    if (live && n < a.N) {
                        const float A = -expf(a.A_log[static_cast<size_t>(ch) * a.N + n]);  // A = -exp(A_log)
                        al[e] = A * kLog2e;
                        nr[e] = -1.0f / A;
                    }
                }
                A2p[q] = f2_pack(al[0], al[1]);
                nrAp[q] = f2_pack(nr[0], nr[1]);
                hp[q] = f2_pack(0.f, 0.f);
            }
            if (a.dynamic && seg > 0) {
                // wait for the end state of the previous segment of this chain
                bool got = true;
                if (tid == 0) {
                    got = false;
                    for (uint32_t i = 0; i < (1u << 22); ++i) {
                        if (ld_acquire_gpu(&a.flags[chain]) >= static_cast<unsigned int>(seg)) {
                            got = true;
                            break;
                        }
                        __nanosleep(64);
                    }
                    if (!got)
                        raise_device_error(2u);
                }
                __syncthreads();
                const float *cp = a.carry + (static_cast<size_t>(chain) * CPB + cl) * NS + n0;
#pragma unroll
                for (int q = 0; q < NP; q += 2) {
                    const float4 v = __ldcg(reinterpret_cast<const float4 *>(cp + 2 * q));
                    hp[q] = f2_pack(v.x, v.y);
                    hp[q + 1] = f2_pack(v.z, v.w);
                }
            }
        }

        // ---------------------------------------------- the chunk's tokens
        const int tcount = m.z;
        const IO(*xs)[CPB] = sm.x[s];
        const IO(*dts)[CPB] = sm.dt[s];
        const IO(*zs)[CPB] = sm.z[s];
        IO(*ys)[CPB] = sm.y[ci % 3];
        const float(*bc)[2][NS] = sm.bc[ci & 1];

        float xm3 = 0.f, xm2 = 0.f, xm1 = 0.f;
        if (CONV) {
            xm3 = tr::to_f(xs[0][cl]);
            xm2 = tr::to_f(xs[1][cl]);
            xm1 = tr::to_f(xs[2][cl]);
        }
        // scalars of token j (advances the conv history by one token)
        auto scalars = [&](int j) {
            TokScalars r;
            const float zv = a.has_z ? tr::to_f(zs[j][cl]) : 0.0f;
            float pre;
            if (CONV) {
                const float x0 = tr::to_f(xs[j + kHalo][cl]);
                pre = fmaf(w0, xm3, cb);
                pre = fmaf(w1, xm2, pre);
                pre = fmaf(w2, xm1, pre);
                pre = fmaf(w3, x0, pre);
                xm3 = xm2;
                xm2 = xm1;
                xm1 = x0;
            } else {
                pre = tr::to_f(xs[j][cl]);
            }
            if (TPC == 2) {
                // the two threads of a channel take one SiLU each and swap
                const float v = (CONV && half == 0) ? pre : zv;
                const float sv = silu_fast(v);
                const float other = __shfl_xor_sync(0xffffffffu, sv, 1);
                r.u = CONV ? (half == 0 ? sv : other) : pre;
                r.g = a.has_z ? (CONV ? (half == 0 ? other : sv) : sv) : 1.0f;
            } else {
                r.u = CONV ? silu_fast(pre) : pre;
                r.g = a.has_z ? silu_fast(zv) : 1.0f;
            }
            r.delta = softplus_fast(tr::to_f(dts[j][cl]) + bias);
            return r;
        };

        TokScalars cur = scalars(0);
#pragma unroll 2
        for (int j = 0; j < tcount; ++j) {
            const TokScalars nxt = scalars(j + 1 < tcount ? j + 1 : j);
            const f2_t dd = f2_pack(cur.delta, cur.delta);
            const f2_t uu = f2_pack(cur.u, cur.u);
            const f2_t du = f2_mul(dd, uu);
            f2_t acc = f2_pack(0.f, 0.f);
            const ulonglong2 *Bq = reinterpret_cast<const ulonglong2 *>(&bc[j][0][n0]);
            const ulonglong2 *Cq = reinterpret_cast<const ulonglong2 *>(&bc[j][1][n0]);
#pragma unroll
            for (int q2 = 0; q2 < NP / 2; ++q2) {
                const ulonglong2 Bv = Bq[q2];
                const ulonglong2 Cv = Cq[q2];
                const f2_t Bp[2] = {Bv.x, Bv.y};
                const f2_t Cp[2] = {Cv.x, Cv.y};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int q = 2 * q2 + e;
                    const f2_t dA = f2_mul(dd, A2p[q]);
                    float d0, d1;
                    f2_unpack(dA, d0, d1);
                    const f2_t ab = f2_pack(ex2_approx(d0), ex2_approx(d1));
                    if (ZOH) {
                        // h' = abar*h + (abar-1)*k, k = B u / A; with nk = -k:
                        // h' = abar*(h - nk) + nk
                        const f2_t nk = f2_mul(nrAp[q], f2_mul(uu, Bp[e]));
                        hp[q] = f2_fma(ab, f2_sub(hp[q], nk), nk);
                    } else {
                        hp[q] = f2_fma(ab, hp[q], f2_mul(du, Bp[e]));
                    }
                    acc = f2_fma(hp[q], Cp[e], acc);
                }
            }
            float a0, a1;
            f2_unpack(acc, a0, a1);
            float yv = a0 + a1;
            if (TPC == 2)
                yv += __shfl_xor_sync(0xffffffffu, yv, 1);
            yv = fmaf(Dd, cur.u, yv) * cur.g;
            if (half == 0)
                ys[j][cl] = tr::from_f(yv);
            cur = nxt;
        }

        if (m.w & kMetaLast) {
            const int ch = c0 + cl;
            if (a.dynamic && seg + 1 < a.nseg) {
                float *cp = a.carry + (static_cast<size_t>(chain) * CPB + cl) * NS + n0;
#pragma unroll
                for (int q = 0; q < NP; q += 2) {
                    float v0, v1, v2, v3;
                    f2_unpack(hp[q], v0, v1);
                    f2_unpack(hp[q + 1], v2, v3);
                    __stcg(reinterpret_cast<float4 *>(cp + 2 * q), make_float4(v0, v1, v2, v3));
                }
            } else if (live && a.h_final) {
                float *hf = a.h_final + (static_cast<size_t>(bseq) * a.d + ch) * a.N;
#pragma unroll
                for (int q = 0; q < NP; ++q) {
                    float v0, v1;
                    f2_unpack(hp[q], v0, v1);
                    if (n0 + 2 * q < a.N)
                        hf[n0 + 2 * q] = v0;
                    if (n0 + 2 * q + 1 < a.N)
                        hf[n0 + 2 * q + 1] = v1;
                }
            }
        }

        // ---- the next chunk: wait for its stage and stage its B/C rows
        const int s1 = (ci + 1) % STAGES;
        const bool got = mbar_wait_bounded(&sm.full[s1], ((ci + 1) / STAGES) & 1, 1u << 24);
        if (got)
            stage_bc(s1, (ci + 1) & 1);
        fence_proxy_async_smem();
        if (__syncthreads_or(!got)) {
            if (tid == 0)
                raise_device_error(1u);
            ok = false;
        }
        if (tid == 0) {
            if ((m.w & kMetaLast) && a.dynamic && seg + 1 < a.nseg) {
                __threadfence();
                st_release_gpu(&a.flags[chain], static_cast<unsigned int>(seg + 1));
            }
            tma_store_3d(&tm_y, &sm.y[ci % 3][0][0], c0, m.y, bseq);
            bulk_commit_group();
            if (ok)
                produce(s);
            // the y buffer written next-but-one chunk must be free again
            bulk_wait_group_read<1>();
        }
        ++ci;
    }
    if (tid == 0) {
        if (!ok) {
            // after a failed wait, give the loads still in flight a bounded
            // chance to land before the shared memory they target is released
            for (int c = ci + 1; c < p_count; ++c)
                (void)mbar_wait_bounded(&sm.full[c % STAGES], (c / STAGES) & 1, 1u << 20);
        }
        bulk_wait_group<0>();
    }
}

}  // namespace s6
