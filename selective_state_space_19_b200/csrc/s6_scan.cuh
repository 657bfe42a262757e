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
// Work decomposition.  TPC threads share one channel (TPC = 2 at N = 16,
// each keeping NH = N/TPC float32 states in registers); the 4 consumer warps
// of a CTA own CPB = 128/TPC consecutive channels of one sequence.  A
// sequence's channel tile is a chain of segments of seg_len tokens; a
// (segment, tile) pair is a unit of work.  In the dynamic mode persistent
// CTAs pull units, segment-major, from a global counter, and a unit whose
// segment is not the first starts from the state its predecessor published in
// a carry buffer.  The predecessor was pulled earlier by a running CTA, so the
// (bounded) wait for it always ends.  This spreads B*d/CPB chains evenly over
// every SM whatever their count, without recomputing a single decay.  In the
// static mode (plenty of chains) each CTA runs one whole chain.
//
// Warp roles.  Warp 4 is the producer: it pulls units, issues per chunk of T
// tokens the TMA tile loads of the [T(+3 halo) x CPB] slices of x, dt, z and
// the [T x N] rows of B and C into a STAGES-deep shared-memory ring, fetches a
// unit's start state from the carry buffer once its flags are published, and
// converts each chunk's B/C rows to float32 before marking the stage ready.
// It shares an SM sub-partition with consumer warps, so it keeps its own
// instruction count low: the B/C copy moves whole 512-byte groups with
// constant per-lane addresses, and its waits sleep between polls.  It is the
// CTA's fifth warp, so that the four consumer warps (warps 0-3) fall on the
// SM's four sub-partitions: moving the producer to another warp index put two
// consumers on one sub-partition and cost a quarter of the throughput.
// The 3 halo rows give the conv its K-1 earlier inputs; rows before token 0
// are zero-filled by the TMA unit (the conv's zero left padding).  Warps 0-3
// are consumers: each waits for a ready stage, runs its 32/TPC channels over
// the chunk, releases the stage, and stores its own y tile with a TMA bulk
// store -- no CTA-wide barrier in the steady state.
//
// Arithmetic.  The 16 decays per element are the binding work (one live
// exponential per state per token, "the s6 cell") and go to the MUFU ex2
// pipe.  SiLU and softplus take one MUFU op each (SiLU by tanh for bfloat16
// I/O); the reciprocal and log1p run on the FMA pipe.  With TPC = 2 the two
// threads of a channel walk the tokens in quads: each computes the per-token
// scalars (conv, both SiLUs, softplus) of two of the four tokens in packed
// form, and the pair swaps (u, Delta) through per-lane shared-memory slots, so
// no scalar is computed twice; each thread then updates its NH states token
// by token, issuing the next token's decays among the current token's FMAs,
// and the partial readouts are swapped with one shuffle so that each thread
// finishes and writes its own tokens.  The next quad's scalars are computed
// at the start of a quad, its (u, Delta) exchanged after the updates, and the
// rows they read (conv window, z, dt) fetched one quad ahead.  State
// arithmetic runs on packed float32 pairs (f32x2).
//
// The extended instantiations (EXT = 1) also start a chain from a given state
// (h_init, and for the fused form the conv history before token 0) and take
// the associative split of few long chains; the checkpoint instantiation
// (EXT = 2) stores the backward's state checkpoints and computes no output.
// They are separate so that the plain scan's code is untouched by that support.
//
// No tensor cores: the recurrence is diagonal (an elementwise product with a
// data-dependent decay), not a contraction.
#pragma once

#include <type_traits>

#include "s6_common.cuh"

namespace s6 {

constexpr int kConsumerWarps = 4;
constexpr int kScanThreads = 32 * kConsumerWarps;  // consumer threads
constexpr int kScanBlock = kScanThreads + 32;      // + one producer warp
constexpr int kHalo = 3;                           // conv history rows (taps padded to 4)
#ifndef S6_SCAN_YBUF
#define S6_SCAN_YBUF 2
#endif
constexpr int kYBuf = S6_SCAN_YBUF;  // y tiles per consumer warp

constexpr int kMetaFirst = 1;  // first chunk of its unit
constexpr int kMetaLast = 2;   // last chunk of its unit
constexpr int kMetaEnd = 4;    // no more work
constexpr int kMetaCarry = 8;  // the unit starts from a published carry or the given start state
constexpr int kMetaNoY = 16;   // associative split: a state-only unit (no outputs)

constexpr int kCkptEvery = 16;  // tokens between the backward's state checkpoints

// Write and decay forms (the MODE template argument).
constexpr int kModeSimplified = 0;  // decay 2^(Delta A log2 e), write Delta B u
constexpr int kModeZOH = 1;         // decay as above, write (A_bar - 1)/A B u
constexpr int kModeConst = 2;       // constant decay 2^w per (channel, state), write B u:
                                    // the constant-decay cell of "the s6 cell",
                                    // "one cell, two architectures"; A_log carries w

struct ScanArgs {
    int Bt, L, d, N, K;
    int has_z;
    int tiles;    // channel tiles per sequence
    int nseg;     // segments per sequence
    int seg_len;  // tokens per segment (a multiple of the chunk length)
    int units;    // Bt * tiles * nseg (serial), Bt * tiles * (2 nseg - 1) (associative)
    int dynamic;  // 1: persistent CTAs pull units from *counter
    int assoc;    // 1: associative split (extended instantiation only)
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
    unsigned int *flags;    // dynamic: [Bt*tiles][consumer warps] last published segment + 1
    float *carry;           // serial: [Bt*tiles][CPB][NS] published end states;
                            // associative: [Bt*tiles][nseg][CPB][NS] end state of segment 0 (slot 0)
                            // and the state-only units' states from zero (slots 1..nseg-1)
    float *carry_sum;       // associative: [Bt*tiles][nseg][CPB] sum of Delta over each state-only unit
    const float *h_init;    // [Bt, d, N] start state, or null (zeros)
    const void *conv_hist;  // [Bt, d, K-1] io conv history before token 0 (oldest first), or null (zeros)
    float *ckpt;               // extended instantiation, N = 16: the state before every
                               // kCkptEvery-th token, [Bt][ceil(L / kCkptEvery)][d][16]
                               // (the backward's checkpoints); y is then not written.  Or null.
    unsigned int carry_polls;  // polls of a predecessor's flag before the wait gives up
    int skip_publish;          // fault injection for tests: this unit publishes no carry (-1: none)
};

template <int NS, int TPC, int T, bool CONV>
struct ScanShape {
    static constexpr int NH = NS / TPC;             // states per thread
    static constexpr int CPB = kScanThreads / TPC;  // channels per CTA
    static constexpr int CPW = 32 / TPC;            // channels per consumer warp
    static constexpr int XR = T + (CONV ? kHalo : 0);
    static constexpr int XPAD = 4;  // rows after the x tile read only for tokens past the chunk
    static_assert(NH % 4 == 0, "states per thread must be a multiple of 4");
    static_assert(TPC == 1 || TPC == 2, "one or two threads per channel");
    static_assert(T % (2 * TPC) == 0, "chunks hold whole token groups");
};

// A tile moved by TMA: every buffer starts on a 128-byte boundary.
template <typename E, int R, int C>
struct alignas(128) Tile {
    E v[R][C];
};

template <typename IO, int NS, int TPC, int T, int STAGES, bool CONV>
struct ScanSmem {
    using Sh = ScanShape<NS, TPC, T, CONV>;
    Tile<IO, Sh::XR + Sh::XPAD, Sh::CPB> x[STAGES];
    Tile<IO, T + Sh::XPAD, Sh::CPB> dt[STAGES];
    Tile<IO, T + Sh::XPAD, Sh::CPB> z[STAGES];
    Tile<IO, T, Sh::CPW> y[kConsumerWarps][kYBuf];  // per consumer warp, rotating
    Tile<IO, 1, T * NS> braw[STAGES];
    Tile<IO, 1, T * NS> craw[STAGES];
    float bc[STAGES][T][2][NS];        // [stage][token][B|C][n], float32, zero-padded
    float hinit[STAGES][Sh::CPB][NS];  // start state of a unit that begins in the stage
    float4 xch[2][kConsumerWarps][32];  // per-lane (u, Delta) of its own tokens, by quad parity
    int4 meta[STAGES];                 // {unit, t0, tcount, flags}
    uint64_t full[STAGES];             // TMA bytes landed (producer waits)
    uint64_t ready[STAGES];            // stage complete and converted (consumers wait)
    uint64_t empty[STAGES];            // all consumer warps done with the stage
};

struct UnitPos {
    int b, tile, seg, chain;
    bool state_only;  // associative split: scan from zero, outputs not written
};

// Unit order.  Serial split: segment-major, unit u = seg * chains + chain.
// Associative split: first every chain's segment 0 (a full unit), then the
// state-only units of segments 1..nseg-1, then the full units of segments
// 1..nseg-1 -- each in segment-major order.  A unit only ever waits for units
// handed out before it.
__device__ __forceinline__ UnitPos unit_pos(int u, const ScanArgs &a) {
    const int per = a.Bt * a.tiles;
    UnitPos p;
    p.state_only = false;
    if (a.assoc) {
        const int ns = a.nseg;
        if (u >= per * ns) {
            u -= per * ns;
            p.seg = u / per + 1;
        } else {
            p.seg = u / per;
            p.state_only = p.seg > 0;
        }
        p.chain = u - (u / per) * per;
    } else {
        p.seg = u / per;
        p.chain = u - p.seg * per;
    }
    p.b = p.chain / a.tiles;
    p.tile = p.chain - p.b * a.tiles;
    return p;
}

constexpr uint32_t kWaitPolls = 1u << 24;
// sleeping waits: at most kSleepPolls polls of at most kSleepNs each (about 2 s)
constexpr uint32_t kSleepPolls = 1u << 21;
constexpr uint32_t kSleepNs = 1000u;

// EXT: 0 the plain scan; 1 the extended scan, which may start from a given
// state (h_init, conv_hist) and may take the associative split; 2 the
// extended scan in checkpoint mode for the backward (N = 16 only, no
// outputs); 3 the same with its outputs, a training forward whose checkpoints
// the backward then reuses.  Separate instantiations, so that each one carries
// only its own code.
//
// Registers: two CTAs of kScanBlock threads per SM allow 200 per thread; a
// cap of 168 measured 0.8 % faster on the long-sequence workload than the
// allocator's own choice under that bound (165), and leaves the same two CTAs.
template <typename IO, int NS, int TPC, int T, int STAGES, bool CONV, int MODE, int EXT>
__global__ void __maxnreg__(168)
    s6_scan_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_dt,
                   const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_y,
                   const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_C,
                   const ScanArgs a) {
    using Sh = ScanShape<NS, TPC, T, CONV>;
    using Smem = ScanSmem<IO, NS, TPC, T, STAGES, CONV>;
    using tr = io_traits<IO>;
    constexpr bool ZOH = MODE == kModeZOH;
    constexpr bool CONSTD = MODE == kModeConst;  // decay from a constant, no step size
    constexpr bool INIT = EXT >= 1;  // given start state, associative split
    constexpr bool CKPT = EXT >= 2;   // the state before every kCkptEvery-th token
    constexpr bool NOOUT = EXT == 2;  // the backward's own forward: no y, no readout
    static_assert(!CKPT || (NS == 16 && TPC == 2), "checkpoints are kept at N = 16 only");
    constexpr int NH = Sh::NH;
    constexpr int NP = NH / 2;  // state pairs per thread
    constexpr int CPB = Sh::CPB;
    constexpr int CPW = Sh::CPW;
    constexpr int XR = Sh::XR;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.ready[s], 1);
            mbar_init(&sm.empty[s], kConsumerWarps);
        }
        fence_mbarrier_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // =========================================================== producer
        // Its waits sleep between polls (kSleepNs): this warp shares an SM
        // sub-partition with consumer warps, and a spinning wait would take
        // their issue slots.
        if (lane == 0) {
            prefetch_tensormap(&tm_x);
            if (!CONSTD)
                prefetch_tensormap(&tm_dt);
            if (a.has_z)
                prefetch_tensormap(&tm_z);
            if (a.bc_tma) {
                prefetch_tensormap(&tm_B);
                prefetch_tensormap(&tm_C);
            }
        }
        int unit = -1, k = 0, nk = 0, tlo = 0, thi = 0;
        bool done = false, first_pull = true, ok = true;

        // B/C rows of chunk cc -> float32 (all 32 lanes), then the stage is ready
        auto finish = [&](int cc) {
            const int sp = cc % STAGES;
            __syncwarp();  // lane 0's metadata write is visible to the warp
            bool got = true;
            if (lane == 0)
                got = mbar_wait_sleep_bounded(&sm.full[sp], (cc / STAGES) & 1, kSleepPolls, kSleepNs);
            got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
            if (!got) {
                if (lane == 0)
                    raise_device_error(1u);
                ok = false;
            }
            const int4 m = sm.meta[sp];
            const UnitPos up = unit_pos(m.x, a);
            if (INIT && CONV && got && a.conv_hist && m.y == 0) {
                // the sequence's first chunk: its halo rows before token 0 (zeros
                // from the tensor copy) take the given conv history instead
                const int K1 = a.K - 1;
                const IO *hsrc = static_cast<const IO *>(a.conv_hist) + static_cast<size_t>(up.b) * a.d * K1;
                const int c0 = up.tile * CPB;
                for (int i = lane; i < CPB * K1; i += 32) {
                    const int ch = i / K1;
                    const int kk = i - ch * K1;
                    if (c0 + ch < a.d)
                        sm.x[sp].v[kHalo - K1 + kk][ch] = hsrc[static_cast<size_t>(c0 + ch) * K1 + kk];
                }
                fence_proxy_async_smem();  // before the stage is refilled by the tensor unit
            }
            constexpr int kSlots = 2 * T * NS;
            if constexpr (NS == 16 && T % 4 == 0) {
                if (got && a.bc_tma && a.N == NS) {
                    // Whole rows.  This warp shares an SM sub-partition with
                    // consumer warps, so the copy is kept to a few instructions a
                    // value: each step fills one 512-byte group of bc (4 tokens x
                    // B|C x 16 states), lane l its bytes [16 l, 16 l + 16) -- token
                    // l / 8 of the group, B or C by bit 2, states 4 (l & 3) .. +3 --
                    // with every address a per-lane base plus a constant.
                    const int which = (lane >> 2) & 1;
                    const int n4 = (lane & 3) * 4;
                    const int tl = lane >> 3;
                    const IO *src = (which ? &sm.craw[sp].v[0][0] : &sm.braw[sp].v[0][0]) + tl * NS + n4;
                    float *dst = &sm.bc[sp][tl][which][n4];
                    auto row4 = [&](int i) {
                        if constexpr (sizeof(IO) == 2) {
                            const uint2 r = *reinterpret_cast<const uint2 *>(src + i * 4 * NS);
                            return make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xffff0000u),
                                               __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xffff0000u));
                        } else {
                            return *reinterpret_cast<const float4 *>(src + i * 4 * NS);
                        }
                    };
                    if (m.z == T) {
#pragma unroll
                        for (int i = 0; i < T / 4; ++i)
                            *reinterpret_cast<float4 *>(dst + i * 4 * 2 * NS) = row4(i);
                    } else {
                        // a partial chunk: rows past its tokens are zeroed
                        for (int i = 0; i < T / 4; ++i)
                            *reinterpret_cast<float4 *>(dst + i * 4 * 2 * NS) =
                                (4 * i + tl < m.z) ? row4(i) : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&sm.ready[sp]);
                    return;
                }
            }
            if (got && a.bc_tma && a.N == NS) {
                // whole rows: four values per lane step
                for (int j = lane; j < kSlots / 4; j += 32) {
                    const int which = j / (T * NS / 4);
                    const int rem = j - which * (T * NS / 4);
                    const int tt = rem / (NS / 4);
                    const int n = (rem - tt * (NS / 4)) * 4;
                    const IO *src = which ? &sm.craw[sp].v[0][tt * NS + n] : &sm.braw[sp].v[0][tt * NS + n];
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (tt < m.z) {
                        if constexpr (sizeof(IO) == 2) {
                            const uint2 r = *reinterpret_cast<const uint2 *>(src);
                            v = make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xffff0000u),
                                            __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xffff0000u));
                        } else {
                            v = *reinterpret_cast<const float4 *>(src);
                        }
                    }
                    *reinterpret_cast<float4 *>(&sm.bc[sp][tt][which][n]) = v;
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&sm.ready[sp]);
                return;
            }
            for (int j = lane; j < kSlots; j += 32) {
                const int which = j / (T * NS);
                const int rem = j - which * (T * NS);
                const int tt = rem / NS;
                const int n = rem - tt * NS;
                float v = 0.0f;
                if (got && n < a.N && tt < m.z) {
                    if (a.bc_tma) {
                        v = tr::to_f(which ? sm.craw[sp].v[0][tt * a.N + n] : sm.braw[sp].v[0][tt * a.N + n]);
                    } else {
                        const size_t off = (static_cast<size_t>(up.b) * a.L + m.y + tt) * a.N + n;
                        v = tr::to_f(which ? static_cast<const IO *>(a.C)[off] : static_cast<const IO *>(a.B)[off]);
                    }
                }
                sm.bc[sp][tt][which][n] = v;
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.ready[sp]);
        };

        int c = 0;
        for (;; ++c) {
            const int s = c % STAGES;
            // Make the previous chunk ready first: the consumers can start on it
            // while this warp waits for a free stage or for a carry -- which may
            // be published by this CTA's own previous unit.
            if (c >= 1)
                finish(c - 1);
            if (c >= STAGES) {
                bool got = true;
                if (lane == 0)
                    got = mbar_wait_sleep_bounded(&sm.empty[s], ((c / STAGES) - 1) & 1, kSleepPolls, kSleepNs);
                got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
                if (!got) {
                    if (lane == 0)
                        raise_device_error(1u);
                    ok = false;
                }
            }
            if (ok && !done && k == nk) {
                int u = 0;
                if (lane == 0) {
                    if (a.dynamic)
                        u = static_cast<int>(atomicAdd(a.counter, 1u));
                    else
                        u = first_pull ? static_cast<int>(blockIdx.x) : a.units;
                }
                u = __shfl_sync(0xffffffffu, u, 0);
                first_pull = false;
                if (u >= a.units) {
                    done = true;
                } else {
                    const UnitPos up = unit_pos(u, a);
                    unit = u;
                    k = 0;
                    tlo = up.seg * a.seg_len;
                    thi = min(a.L, tlo + a.seg_len);
                    nk = (thi - tlo + T - 1) / T;
                }
            }
            if (done || !ok) {
                if (lane == 0)
                    sm.meta[s] = make_int4(-1, 0, 0, kMetaEnd);
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&sm.ready[s]);
                break;
            }
            const UnitPos up = unit_pos(unit, a);
            const int t0 = tlo + k * T;
            const bool carry_in = a.dynamic && k == 0 && up.seg > 0 && !up.state_only;
            const bool given_in = INIT && a.h_init && k == 0 && up.seg == 0;  // a chain's start state is given
            const int fl = (k == 0 ? kMetaFirst : 0) | (k == nk - 1 ? kMetaLast : 0) |
                           (carry_in || given_in ? kMetaCarry : 0) | (up.state_only ? kMetaNoY : 0);
            if (lane == 0) {
                sm.meta[s] = make_int4(unit, t0, min(T, thi - t0), fl);
                const int c0 = up.tile * CPB;
                constexpr uint32_t kX = XR * CPB * sizeof(IO);
                constexpr uint32_t kR = T * CPB * sizeof(IO);
                const uint32_t kBC = a.bc_tma ? 2u * T * a.N * static_cast<uint32_t>(sizeof(IO)) : 0u;
                mbar_arrive_expect_tx(&sm.full[s], kX + (CONSTD ? 0u : kR) + (a.has_z ? kR : 0u) + kBC);
                tma_load_3d(&sm.x[s].v[0][0], &tm_x, &sm.full[s], c0, t0 - (CONV ? kHalo : 0), up.b);
                if (!CONSTD)
                    tma_load_3d(&sm.dt[s].v[0][0], &tm_dt, &sm.full[s], c0, t0, up.b);
                if (a.has_z)
                    tma_load_3d(&sm.z[s].v[0][0], &tm_z, &sm.full[s], c0, t0, up.b);
                if (a.bc_tma) {
                    tma_load_3d(&sm.braw[s].v[0][0], &tm_B, &sm.full[s], 0, t0, up.b);
                    tma_load_3d(&sm.craw[s].v[0][0], &tm_C, &sm.full[s], 0, t0, up.b);
                }
            }
            if (given_in) {
                // rows of h_init for this tile's channels, zero past d and N
                const float *src = a.h_init + static_cast<size_t>(up.b) * a.d * a.N;
                const int c0 = up.tile * CPB;
                for (int i = lane; i < CPB * NS; i += 32) {
                    const int ch = i / NS;
                    const int n = i - ch * NS;
                    const int cc = c0 + ch;
                    sm.hinit[s][ch][n] = (cc < a.d && n < a.N) ? __ldg(src + static_cast<size_t>(cc) * a.N + n) : 0.0f;
                }
            }
            if (carry_in) {
                if (INIT && a.assoc) {
                    // Associative split.  The start state of segment `seg` is
                    // E_{seg-1}, folded from segment 0's end state E_0 and the
                    // state-only units' (P_j, s_j) for j = 1 .. seg-1:
                    //     E_j = P_j * E_{j-1} + s_j,   P_j = prod of the segment's
                    //     decays = 2^(A log2 e * sum of its Delta)
                    // -- the pair combine (a1, b1) o (a2, b2) = (a1 a2, a2 b1 + b2)
                    // applied left to right.  Every unit folded here was handed
                    // out before this one, so the (bounded) waits end.
                    const size_t base = static_cast<size_t>(up.chain) * a.nseg;
                    bool got = true;
                    if (lane < kConsumerWarps) {
                        for (int j = 0; j < up.seg && got; ++j) {
                            got = false;
                            const unsigned int *f = &a.flags[(base + j) * kConsumerWarps + lane];
                            for (uint32_t i = 0; i < a.carry_polls; ++i) {
                                if (ld_acquire_gpu(f) >= 1u) {
                                    got = true;
                                    break;
                                }
                                __nanosleep(64);
                            }
                        }
                    }
                    if (!__all_sync(0xffffffffu, got)) {
                        if (lane == 0)
                            raise_device_error(2u);
                    }
                    const int c0 = up.tile * CPB;
                    for (int i = lane; i < CPB * NS; i += 32) {
                        const int ch = i / NS;
                        const int n = i - ch * NS;
                        const int cc = c0 + ch;
                        // A log2 e with A = -exp(A_log) (the constant cell: w, the log2
                        // of its decay, with a unit step per token); zero for padding
                        float A2 = 0.0f;
                        if (cc < a.d && n < a.N) {
                            const float al = a.A_log[static_cast<size_t>(cc) * a.N + n];
                            A2 = CONSTD ? al : -expf(al) * kLog2e;
                        }
                        float h = __ldcg(a.carry + base * CPB * NS + i);
                        for (int j = 1; j < up.seg; ++j) {
                            const float sj = __ldcg(a.carry_sum + (base + j) * CPB + ch);
                            h = fmaf(ex2_approx(A2 * sj), h, __ldcg(a.carry + (base + j) * CPB * NS + i));
                        }
                        sm.hinit[s][ch][n] = h;
                    }
                } else {
                    // the predecessor segment publishes one flag per consumer warp
                    bool got = true;
                    if (lane < kConsumerWarps) {
                        got = false;
                        const unsigned int *f = &a.flags[static_cast<size_t>(up.chain) * kConsumerWarps + lane];
                        for (uint32_t i = 0; i < a.carry_polls; ++i) {
                            if (ld_acquire_gpu(f) >= static_cast<unsigned int>(up.seg)) {
                                got = true;
                                break;
                            }
                            __nanosleep(64);
                        }
                    }
                    if (!__all_sync(0xffffffffu, got)) {
                        if (lane == 0)
                            raise_device_error(2u);
                    }
                    const float4 *src =
                        reinterpret_cast<const float4 *>(a.carry + static_cast<size_t>(up.chain) * CPB * NS);
                    float4 *dst = reinterpret_cast<float4 *>(&sm.hinit[s][0][0]);
                    for (int i = lane; i < CPB * NS / 4; i += 32)
                        dst[i] = __ldcg(src + i);
                }
            }
            ++k;
        }
        return;
    }

    // ============================================================== consumers
    const int cw = lane / TPC;       // channel within the warp
    const int cl = warp * CPW + cw;  // channel within the CTA tile
    const int sub = lane % TPC;  // which NH states of the channel this thread holds
    const int half = (TPC == 2) ? sub : 0;
    const int n0 = sub * NH;

    f2_t hp[NP], A2p[NP], nrAp[NP];
    float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, cb = 0.f, Dd = 0.f, bias = 0.f;
    float sdel = 0.f;  // extended instantiation: sum of the unit's Delta (associative split)
    bool live = false;
    int chain = 0, seg = 0, bseq = 0, c0 = 0;
#pragma unroll
    for (int q = 0; q < NP; ++q)
        hp[q] = A2p[q] = nrAp[q] = f2_pack(0.f, 0.f);

    // Software-pipelined form: ab[] holds this token's decays; the next
    // token's decays are issued pair by pair among this token's FMAs, so the
    // MUFU pipe is fed while the state arithmetic proceeds.
    f2_t ab[NP];
    auto decays = [&](float delta) {
        if constexpr (!CONSTD) {  // the constant cell's decays are the constants in A2p
            const f2_t dd = f2_pack(delta, delta);
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                float d0, d1;
                f2_unpack(f2_mul(dd, A2p[q]), d0, d1);
                ab[q] = f2_pack(ex2_approx(d0), ex2_approx(d1));
            }
        }
    };
    auto update_pipe = [&](const float(*bcrow)[NS], float u, float delta, float delta_next, auto next_tag) -> float {
        constexpr bool NEXT = decltype(next_tag)::value;
        const f2_t uu = f2_pack(u, u);
        const f2_t du = f2_mul(f2_pack(delta, delta), uu);
        const f2_t ddn = f2_pack(delta_next, delta_next);
        f2_t acc = f2_pack(0.f, 0.f), acc_b = f2_pack(0.f, 0.f);
        const ulonglong2 *Bq = reinterpret_cast<const ulonglong2 *>(&bcrow[0][n0]);
        const ulonglong2 *Cq = reinterpret_cast<const ulonglong2 *>(&bcrow[1][n0]);
#pragma unroll
        for (int q2 = 0; q2 < NP / 2; ++q2) {
            const ulonglong2 Bv = Bq[q2];
            const ulonglong2 Cv = Cq[q2];
            const f2_t Bp[2] = {Bv.x, Bv.y};
            const f2_t Cp[2] = {Cv.x, Cv.y};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int q = 2 * q2 + e;
                const f2_t abq = CONSTD ? A2p[q] : ab[q];
                if (NEXT && !CONSTD) {
                    float d0, d1;
                    f2_unpack(f2_mul(ddn, A2p[q]), d0, d1);
                    ab[q] = f2_pack(ex2_approx(d0), ex2_approx(d1));
                }
                if (CONSTD) {
                    hp[q] = f2_fma(abq, hp[q], f2_mul(uu, Bp[e]));
                } else if (ZOH) {
                    const f2_t nk = f2_mul(nrAp[q], f2_mul(uu, Bp[e]));
                    hp[q] = f2_fma(abq, f2_sub(hp[q], nk), nk);
                } else {
                    hp[q] = f2_fma(abq, hp[q], f2_mul(du, Bp[e]));
                }
                if (e == 0)
                    acc = f2_fma(hp[q], Cp[e], acc);
                else
                    acc_b = f2_fma(hp[q], Cp[e], acc_b);
            }
        }
        float a0, a1;
        f2_unpack(f2_add(acc, acc_b), a0, a1);
        return a0 + a1;
    };

    for (int c = 0;; ++c) {
        const int s = c % STAGES;
        const bool got = mbar_wait_bounded(&sm.ready[s], (c / STAGES) & 1, kWaitPolls);
        if (!__all_sync(0xffffffffu, got)) {
            if (lane == 0)
                raise_device_error(1u);
            break;
        }
        const int4 m = sm.meta[s];
        if (m.w & kMetaEnd)
            break;

        if (m.w & kMetaFirst) {
            // ---- a new unit: this thread's channel parameters and start state
            const UnitPos up = unit_pos(m.x, a);
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
                for (int kk = 0; kk < 4; ++kk) {
                    const int src = kk - (4 - a.K);
                    wv[kk] = (src >= 0) ? a.conv_w[static_cast<size_t>(ch) * a.K + src] : 0.0f;
                }
            }
            w0 = wv[0];
            w1 = wv[1];
            w2 = wv[2];
            w3 = wv[3];
            cb = (CONV && live && a.conv_b) ? a.conv_b[ch] : 0.0f;
            Dd = live ? a.D[ch] : 0.0f;
            bias = (live && a.dt_bias) ? a.dt_bias[ch] : 0.0f;
            const bool carry_in = (m.w & kMetaCarry) != 0;
            sdel = 0.f;
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                float al[2] = {0.f, 0.f}, nr[2] = {0.f, 0.f};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int n = n0 + 2 * q + e;
                    if (live && n < a.N) {
                        if (CONSTD) {
                            // the constant cell: its decay 2^w, computed once per unit in
                            // double precision and rounded once -- a decay near 1 keeps
                            // about 1/(1 - a) tokens, and its rounding error is
                            // multiplied by that memory length
                            al[e] = static_cast<float>(exp2(static_cast<double>(a.A_log[static_cast<size_t>(ch) * a.N + n])));
                        } else {
                            const float A = -expf(a.A_log[static_cast<size_t>(ch) * a.N + n]);  // A = -exp(A_log)
                            al[e] = A * kLog2e;
                            nr[e] = -1.0f / A;
                        }
                    }
                }
                A2p[q] = f2_pack(al[0], al[1]);
                nrAp[q] = f2_pack(nr[0], nr[1]);
                hp[q] = carry_in ? f2_pack(sm.hinit[s][cl][n0 + 2 * q], sm.hinit[s][cl][n0 + 2 * q + 1])
                                 : f2_pack(0.f, 0.f);
            }
        }

        // ---------------------------------------------- the chunk's tokens
        const int tcount = m.z;
        const IO(*xs)[CPB] = sm.x[s].v;
        const IO(*dts)[CPB] = sm.dt[s].v;
        const IO(*zs)[CPB] = sm.z[s].v;
        IO(*yw)[CPW] = sm.y[warp][c % kYBuf].v;
        const float(*bc)[2][NS] = sm.bc[s];

        if constexpr (TPC == 2) {
            // Tokens in quads (p .. p+3).  This thread owns tokens ja = p + half
            // and jb = ja + 2: it computes their scalars (packed, one pair of
            // values per instruction), publishes (u, Delta) of both in a per-lane
            // shared slot, reads the channel's four tokens back in order from
            // its own and its partner's slot, updates its NH states token by
            // token -- each update also issuing the next token's decays -- and
            // after swapping partial readouts writes its two outputs.  Rows past
            // the chunk lie in the tiles' padding and feed only unwritten tokens.
            const IO *xq = &xs[half][cl];  // row r: token half + r - 3
            const IO *dq = &dts[half][cl];
            const IO *zq = &zs[half][cl];
            auto ld = [&](const IO *q, int row) { return tr::to_f(q[row * CPB]); };
            float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f, r4 = 0.f, r5 = 0.f;  // rows p+half .. p+half+5
            if (CONV) {
                r0 = ld(xq, 0);
                r1 = ld(xq, 1);
                r2 = ld(xq, 2);
                r3 = ld(xq, 3);
                r4 = ld(xq, 4);
                r5 = ld(xq, 5);
            }
            const f2_t BIAS = f2_pack(bias, bias);
            auto silu2 = [&](f2_t v) {
                // bfloat16 outputs take the tanh form; float32 outputs, and any
                // scan that keeps checkpoints (the backward recomputes from them
                // with this form), the exponential one
                if constexpr (sizeof(IO) == 2) {
                    if constexpr (CKPT)
                        return f2_silu_fast(v);
                    else
                        return f2_silu_tanh(v);
                } else {
                    return f2_silu_fast(v);
                }
            };
            float za = ld(zq, 0), zb = ld(zq, 2), da = 0.f, db = 0.f;
            if (!CONSTD) {
                da = ld(dq, 0);
                db = ld(dq, 2);
            }
            float xa = CONV ? 0.f : ld(xq, 0), xb = CONV ? 0.f : ld(xq, 2);
            auto quad_scalars = [&](int p, f2_t &u2, f2_t &d2, f2_t &g2) {
                if (CONV) {
                    // the two tokens' taps as scalar FMAs (packing the window
                    // rows into pairs would cost register moves)
                    const float pa = fmaf(w3, r3, fmaf(w2, r2, fmaf(w1, r1, fmaf(w0, r0, cb))));
                    const float pb = fmaf(w3, r5, fmaf(w2, r4, fmaf(w1, r3, fmaf(w0, r2, cb))));
                    const f2_t pre = f2_pack(pa, pb);
                    r0 = r4;
                    r1 = r5;
                    r2 = ld(xq, p + 6);
                    r3 = ld(xq, p + 7);
                    r4 = ld(xq, p + 8);
                    r5 = ld(xq, p + 9);
                    u2 = silu2(pre);
                } else {
                    u2 = f2_pack(xa, xb);
                    xa = ld(xq, p + 4);
                    xb = ld(xq, p + 6);
                }
                const f2_t gz = silu2(f2_pack(za, zb));
                g2 = a.has_z ? gz : f2_pack(1.0f, 1.0f);
                if constexpr (CONSTD)
                    d2 = f2_pack(1.0f, 1.0f);  // a unit step: the segment sums count tokens
                else
                    d2 = f2_softplus_fast(f2_add(f2_pack(da, db), BIAS));
                // this thread's z and dt rows of the next quad, read one quad
                // ahead like the conv window (rows past the chunk lie in the
                // tiles' padding)
                za = ld(zq, p + 4);
                zb = ld(zq, p + 6);
                if (!CONSTD) {
                    da = ld(dq, p + 4);
                    db = ld(dq, p + 6);
                }
            };
            const int base = lane & ~1;
            // publish this thread's (u, Delta) of its two tokens; read the quad's
            // four tokens in order: p = slot[base].xy, p+1 = slot[base+1].xy,
            // p+2 = slot[base].zw, p+3 = slot[base+1].zw
            auto exchange = [&](int buf, f2_t u2, f2_t d2, float4 &s0, float4 &s1) {
                float ua, ub, da, db;
                f2_unpack(u2, ua, ub);
                f2_unpack(d2, da, db);
                sm.xch[buf][warp][lane] = make_float4(ua, da, ub, db);
                __syncwarp();
                s0 = sm.xch[buf][warp][base];
                s1 = sm.xch[buf][warp][base + 1];
            };
            auto run = [&](auto full_tag) {
                constexpr bool FULL = decltype(full_tag)::value;
                const int tc = FULL ? T : tcount;
                f2_t u2c, d2c, g2c;
                float4 c0s, c1s;
                quad_scalars(0, u2c, d2c, g2c);
                exchange(0, u2c, d2c, c0s, c1s);
                decays(c0s.y);  // the chunk's first token
                auto quad = [&](int p, int q, auto last_tag) {
                    constexpr bool LAST = decltype(last_tag)::value;
                    // the next quad's scalars (none after a chunk's last quad: its
                    // last token issues no further decays)
                    f2_t u2n = u2c, d2n = d2c, g2n = g2c;
                    float dnext = 0.f;
                    if (!LAST) {
                        quad_scalars(p + 4, u2n, d2n, g2n);
                        // Delta of the next quad's first token (thread `base` owns
                        // it) for this quad's last update; the full exchange of the
                        // next quad waits until after the updates, so that no warp
                        // barrier separates the scalar work from the state updates
                        float dlo, dhi;
                        f2_unpack(d2n, dlo, dhi);
                        dnext = __shfl_sync(0xffffffffu, dlo, base);
                    }
                    if constexpr (CKPT) {
                        // checkpoint mode: the state before every kCkptEvery-th token
                        // (chunks start on multiples of it); state-only units hold
                        // no true state
                        if ((p % kCkptEvery) == 0 && !(m.w & kMetaNoY) && live) {
                            const int tk = m.y + p;
                            const int nck = (a.L + kCkptEvery - 1) / kCkptEvery;
                            float *cp = a.ckpt + ((static_cast<size_t>(bseq) * nck + tk / kCkptEvery) * a.d +
                                                  (c0 + cl)) * 16 + n0;
#pragma unroll
                            for (int qq = 0; qq < NP; qq += 2) {
                                float v0, v1, v2, v3;
                                f2_unpack(hp[qq], v0, v1);
                                f2_unpack(hp[qq + 1], v2, v3);
                                *reinterpret_cast<float4 *>(cp + 2 * qq) = make_float4(v0, v1, v2, v3);
                            }
                        }
                    }
                    const float acc0 = update_pipe(bc[p], c0s.x, c0s.y, c1s.y, std::true_type{});
                    float acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
                    if (FULL || p + 1 < tc)
                        acc1 = update_pipe(bc[p + 1], c1s.x, c1s.y, c0s.w, std::true_type{});
                    if (FULL || p + 2 < tc)
                        acc2 = update_pipe(bc[p + 2], c0s.z, c0s.w, c1s.w, std::true_type{});
                    if (FULL || p + 3 < tc)
                        acc3 = update_pipe(bc[p + 3], c1s.z, c1s.w, dnext, std::integral_constant<bool, !LAST>{});
                    if constexpr (INIT) {
                        sdel += c0s.y;
                        if (FULL || p + 1 < tc)
                            sdel += c1s.y;
                        if (FULL || p + 2 < tc)
                            sdel += c0s.w;
                        if (FULL || p + 3 < tc)
                            sdel += c1s.w;
                    }
                    // each thread finishes its own tokens: own partial + the partner's
                    // (the backward's own forward writes no y, so the readout, the
                    // gate and z are not computed at all there)
                    if constexpr (!NOOUT) {
                        const float ra = __shfl_xor_sync(0xffffffffu, half ? acc0 : acc1, 1);
                        const float rb = __shfl_xor_sync(0xffffffffu, half ? acc2 : acc3, 1);
                        float ua, ub, ga, gb;
                        f2_unpack(u2c, ua, ub);
                        f2_unpack(g2c, ga, gb);
                        const float ya = fmaf(Dd, ua, (half ? acc1 : acc0) + ra) * ga;
                        const float yb = fmaf(Dd, ub, (half ? acc3 : acc2) + rb) * gb;
                        if (FULL || p + half < tc)
                            yw[p + half][cw] = tr::from_f(ya);
                        if (FULL || p + 2 + half < tc)
                            yw[p + 2 + half][cw] = tr::from_f(yb);
                    }
                    if (!LAST)
                        exchange((q + 1) & 1, u2n, d2n, c0s, c1s);
                    u2c = u2n;
                    g2c = g2n;
                };
                if (FULL) {
#pragma unroll 2
                    for (int p = 0; p < T - 4; p += 4)
                        quad(p, p >> 2, std::false_type{});
                    quad(T - 4, (T - 4) >> 2, std::true_type{});
                } else {
#pragma unroll 1
                    for (int p = 0; p < tc; p += 4) {
                        if (p + 4 < tc)
                            quad(p, p >> 2, std::false_type{});
                        else
                            quad(p, p >> 2, std::true_type{});
                    }
                }
            };
            if (tcount == T)
                run(std::true_type{});
            else
                run(std::false_type{});
        } else {
            // One thread per channel.  Tokens in pairs (p, p+1): the scalars of
            // the next pair are computed in packed form (one pair of values per
            // instruction) while the state advances through the current pair.
            // Rows past the chunk (read only for the pair after the last) lie in
            // the tile's padding, so no index needs clamping.
            const IO *xp = &xs[0][cl];
            const IO *dp = &dts[0][cl];
            const IO *zp = &zs[0][cl];
            auto ld = [&](const IO *q, int row) { return tr::to_f(q[row * CPB]); };
            const f2_t W0 = f2_pack(w0, w0), W1 = f2_pack(w1, w1), W2 = f2_pack(w2, w2), W3 = f2_pack(w3, w3);
            const f2_t CB = f2_pack(cb, cb), BIAS = f2_pack(bias, bias);
            // conv window: rows p .. p+4 hold tokens p-3 .. p+1
            float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f, r4 = 0.f;
            if (CONV) {
                r0 = ld(xp, 0);
                r1 = ld(xp, 1);
                r2 = ld(xp, 2);
                r3 = ld(xp, 3);
                r4 = ld(xp, 4);
            }
            auto pair_scalars = [&](int p, int pr, f2_t &u2, f2_t &d2, f2_t &g2) {
                // p: first token of the pair; pr: row index used for dt / z
                if (CONV) {
                    f2_t pre = f2_fma(W0, f2_pack(r0, r1), CB);
                    pre = f2_fma(W1, f2_pack(r1, r2), pre);
                    pre = f2_fma(W2, f2_pack(r2, r3), pre);
                    pre = f2_fma(W3, f2_pack(r3, r4), pre);
                    r0 = r2;
                    r1 = r3;
                    r2 = r4;
                    r3 = ld(xp, p + 5);
                    r4 = ld(xp, p + 6);
                    u2 = f2_silu_fast(pre);
                } else {
                    u2 = f2_pack(ld(xp, pr), ld(xp, pr + 1));
                }
                const f2_t gz = f2_silu_fast(f2_pack(ld(zp, pr), ld(zp, pr + 1)));
                g2 = a.has_z ? gz : f2_pack(1.0f, 1.0f);
                if constexpr (CONSTD)
                    d2 = f2_pack(1.0f, 1.0f);
                else
                    d2 = f2_softplus_fast(f2_add(f2_pack(ld(dp, pr), ld(dp, pr + 1)), BIAS));
            };
            auto run = [&](auto full_tag) {
                constexpr bool FULL = decltype(full_tag)::value;
                const int tc = FULL ? T : tcount;
                // pairs start at even p < tc <= T (T even), so rows p and p+1 of the
                // dt / z tiles always exist; past tcount they only feed tokens
                // that are not written
                f2_t u2c, d2c, g2c;
                pair_scalars(0, 0, u2c, d2c, g2c);
                {
                    float d0, d1;
                    f2_unpack(d2c, d0, d1);
                    decays(d0);  // the chunk's first token
                }
                // one pair: token p issues token p+1's decays; token p+1 issues
                // the next pair's first decays when LAST is false
                auto pair = [&](int p, auto last_tag) {
                    constexpr bool LAST = decltype(last_tag)::value;
                    f2_t u2n = u2c, d2n = d2c, g2n = g2c;
                    if (!LAST)  // no next pair after a chunk's last
                        pair_scalars(p + 2, p + 2, u2n, d2n, g2n);
                    float u0, u1, d0, d1, g0, g1, dn0, dn1;
                    f2_unpack(u2c, u0, u1);
                    f2_unpack(d2c, d0, d1);
                    f2_unpack(g2c, g0, g1);
                    f2_unpack(d2n, dn0, dn1);
                    const float acc0 = update_pipe(bc[p], u0, d0, d1, std::true_type{});
                    yw[p][cw] = tr::from_f(fmaf(Dd, u0, acc0) * g0);
                    if constexpr (INIT)
                        sdel += d0;
                    if (FULL || p + 1 < tc) {
                        const float acc1 = update_pipe(bc[p + 1], u1, d1, dn0, std::integral_constant<bool, !LAST>{});
                        yw[p + 1][cw] = tr::from_f(fmaf(Dd, u1, acc1) * g1);
                        if constexpr (INIT)
                            sdel += d1;
                    }
                    u2c = u2n;
                    d2c = d2n;
                    g2c = g2n;
                };
                if (FULL) {
#pragma unroll 1
                    for (int p = 0; p < T - 2; p += 2)
                        pair(p, std::false_type{});
                    pair(T - 2, std::true_type{});
                } else {
#pragma unroll 1
                    for (int p = 0; p < tc; p += 2) {
                        if (p + 2 < tc)
                            pair(p, std::false_type{});
                        else
                            pair(p, std::true_type{});
                    }
                }
            };
            if (tcount == T)
                run(std::true_type{});
            else
                run(std::false_type{});
        }

        if (m.w & kMetaLast) {
            const int ch = c0 + cl;
            if (INIT && a.assoc) {
                // associative split: a state-only unit publishes (h from zero,
                // sum of Delta); the first segment publishes its end state
                if ((m.w & kMetaNoY) || (seg == 0 && a.nseg > 1)) {
                    if (m.x != a.skip_publish) {
                        const size_t slot = static_cast<size_t>(chain) * a.nseg + seg;
                        float *cp = a.carry + (slot * CPB + cl) * NS + n0;
#pragma unroll
                        for (int q = 0; q < NP; q += 2) {
                            float v0, v1, v2, v3;
                            f2_unpack(hp[q], v0, v1);
                            f2_unpack(hp[q + 1], v2, v3);
                            __stcg(reinterpret_cast<float4 *>(cp + 2 * q), make_float4(v0, v1, v2, v3));
                        }
                        if (sub == 0)
                            __stcg(a.carry_sum + slot * CPB + cl, sdel);
                        __syncwarp();
                        if (lane == 0) {
                            __threadfence();
                            st_release_gpu(&a.flags[slot * kConsumerWarps + warp], 1u);
                        }
                    }
                } else if (seg == a.nseg - 1 && live && a.h_final) {
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
            } else if (a.dynamic && seg + 1 < a.nseg) {
                if (m.x != a.skip_publish) {
                    float *cp = a.carry + (static_cast<size_t>(chain) * CPB + cl) * NS + n0;
#pragma unroll
                    for (int q = 0; q < NP; q += 2) {
                        float v0, v1, v2, v3;
                        f2_unpack(hp[q], v0, v1);
                        f2_unpack(hp[q + 1], v2, v3);
                        __stcg(reinterpret_cast<float4 *>(cp + 2 * q), make_float4(v0, v1, v2, v3));
                    }
                    __syncwarp();
                    if (lane == 0) {
                        __threadfence();
                        st_release_gpu(&a.flags[static_cast<size_t>(chain) * kConsumerWarps + warp],
                                       static_cast<unsigned int>(seg + 1));
                    }
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

        // release the stage, then store this warp's y tile
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&sm.empty[s]);
            if (!NOOUT && !(INIT && (m.w & kMetaNoY))) {
                if (c0 + warp * CPW < a.d) {  // a tile's last warps may lie past d
                    tma_store_3d(&tm_y, &sm.y[warp][c % kYBuf].v[0][0], c0 + warp * CPW, m.y, bseq);
                    bulk_commit_group();
                }
                // the buffer this warp writes next chunk (stored kYBuf-1 chunks
                // ago) must have been read by its store
                bulk_wait_group_read<kYBuf - 1>();
            } else {
                // no store from this chunk: drain all, so that the rotation's
                // next buffer is free whatever the earlier chunks stored
                bulk_wait_group_read<0>();
            }
        }
        __syncwarp();
    }
    if (lane == 0)
        bulk_wait_group<0>();
}

}  // namespace s6
