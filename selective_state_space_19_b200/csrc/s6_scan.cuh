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
// Mapping.  One thread owns one channel of one sequence and keeps its NS
// float32 states in registers for the whole sequence; a CTA owns 128
// consecutive channels of one sequence.  The sequence is walked in chunks of T
// tokens.  Per chunk, one elected thread issues TMA tile loads of the
// [T(+3 halo) x 128] slices of x, dt and z into a STAGES-deep shared-memory
// ring (completion on an mbarrier), while all threads stage the chunk's B_t and
// C_t rows (T x N each, shared by all 128 channels) through registers into
// shared memory as float32, one chunk ahead.  Each thread then reads its
// column (conflict-free: consecutive threads, consecutive addresses) and the
// broadcast B/C rows (one address per warp), and writes y into a
// triple-buffered [T x 128] tile that the elected thread stores with a TMA
// bulk tensor store.  The conv's K-1 earlier inputs come from the 3 halo rows
// of the x tile (a TMA load at token t0-3; rows before token 0 are zero-filled
// by the TMA unit, which is the conv's zero left padding).
//
// No tensor cores: the recurrence is diagonal (an elementwise product with a
// data-dependent decay), not a contraction.
#pragma once

#include "s6_common.cuh"

namespace s6 {

constexpr int kScanThreads = 128;  // channels per CTA
constexpr int kHalo = 3;           // conv history rows (taps padded to 4)

struct ScanArgs {
    int Bt, L, d, N;
    int has_z;
    const void *B;  // [Bt, L, N] io
    const void *C;
    const float *A_log;    // [d, N]
    const float *D;        // [d]
    const float *dt_bias;  // [d] or null
    const float *conv_w;   // [d, K] taps, oldest first (fused form), else null
    const float *conv_b;   // [d] or null
    int K;                 // conv width 2..4 (fused form)
    float *h_final;        // [Bt, d, N] or null
};

template <typename IO, int NS, int T, int STAGES, bool CONV>
struct ScanSmem {
    static constexpr int XR = T + (CONV ? kHalo : 0);  // rows of the x tile
    IO x[STAGES][XR][kScanThreads];
    IO dt[STAGES][T][kScanThreads];
    IO z[STAGES][T][kScanThreads];
    IO y[3][T][kScanThreads];
    float bc[2][T][2][NS];  // [buffer][token][B|C][n]
    uint64_t full[STAGES];
};

template <typename IO, int NS, int T>
struct BCPrefetch {
    // 2*T*NS slots spread over the CTA's threads.
    static constexpr int kSlots = 2 * T * NS;
    static constexpr int kPer = (kSlots + kScanThreads - 1) / kScanThreads;
    float v[kPer];

    __device__ __forceinline__ void load(const ScanArgs &a, int b, int t0, int tid) {
        const IO *Bp = static_cast<const IO *>(a.B);
        const IO *Cp = static_cast<const IO *>(a.C);
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int j = tid + k * kScanThreads;
            const int which = j / (T * NS);
            const int rem = j - which * (T * NS);
            const int tt = rem / NS;
            const int n = rem - tt * NS;
            const int t = t0 + tt;
            float val = 0.0f;
            if (j < kSlots && t < a.L && n < a.N) {
                const size_t off = (static_cast<size_t>(b) * a.L + t) * a.N + n;
                val = io_traits<IO>::to_f(which ? Cp[off] : Bp[off]);
            }
            v[k] = val;
        }
    }

    __device__ __forceinline__ void store(float (*bc)[2][NS], int tid) const {
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int j = tid + k * kScanThreads;
            if (j < kSlots) {
                const int which = j / (T * NS);
                const int rem = j - which * (T * NS);
                const int tt = rem / NS;
                const int n = rem - tt * NS;
                bc[tt][which][n] = v[k];
            }
        }
    }
};

template <typename IO, int NS, int T, int STAGES, bool CONV, bool ZOH>
__global__ void __launch_bounds__(kScanThreads)
    s6_scan_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_dt,
                   const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_y,
                   const ScanArgs a) {
    using Smem = ScanSmem<IO, NS, T, STAGES, CONV>;
    using tr = io_traits<IO>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);

    const int tid = threadIdx.x;
    const int c0 = blockIdx.x * kScanThreads;
    const int b = blockIdx.y;
    const int ch = c0 + tid;
    const bool live = ch < a.d;
    const int nchunks = (a.L + T - 1) / T;

    constexpr uint32_t kXBytes = Smem::XR * kScanThreads * sizeof(IO);
    constexpr uint32_t kTBytes = T * kScanThreads * sizeof(IO);
    const uint32_t stage_bytes = kXBytes + kTBytes + (a.has_z ? kTBytes : 0u);

    // ---- per-channel constants
    float A2[NS], rA[NS], h[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) {
        A2[n] = 0.0f;
        rA[n] = 0.0f;
        h[n] = 0.0f;
        if (live && n < a.N) {
            const float A = -expf(a.A_log[static_cast<size_t>(ch) * a.N + n]);  // A = -exp(A_log)
            A2[n] = A * kLog2e;
            rA[n] = 1.0f / A;
        }
    }
    const float Dd = live ? a.D[ch] : 0.0f;
    const float bias = (live && a.dt_bias) ? a.dt_bias[ch] : 0.0f;
    // Taps right-aligned into 4 slots: a width-K conv is the width-4 conv
    // whose 4-K oldest taps are zero, so the halo is always 3 rows.
    float w[4] = {0.f, 0.f, 0.f, 0.f};
    float cb = 0.f;
    if (CONV && live) {
        for (int k = 0; k < a.K; ++k)
            w[4 - a.K + k] = a.conv_w[static_cast<size_t>(ch) * a.K + k];
        cb = a.conv_b ? a.conv_b[ch] : 0.0f;
    }
    const float w0 = w[0], w1 = w[1], w2 = w[2], w3 = w[3];

    auto issue_loads = [&](int ci, int s) {
        const int t0 = ci * T;
        mbar_arrive_expect_tx(&sm.full[s], stage_bytes);
        tma_load_3d(&sm.x[s][0][0], &tm_x, &sm.full[s], c0, t0 - (CONV ? kHalo : 0), b);
        tma_load_3d(&sm.dt[s][0][0], &tm_dt, &sm.full[s], c0, t0, b);
        if (a.has_z)
            tma_load_3d(&sm.z[s][0][0], &tm_z, &sm.full[s], c0, t0, b);
    };

    if (tid == 0) {
        prefetch_tensormap(&tm_x);
        prefetch_tensormap(&tm_dt);
        prefetch_tensormap(&tm_y);
        if (a.has_z)
            prefetch_tensormap(&tm_z);
#pragma unroll
        for (int s = 0; s < STAGES; ++s)
            mbar_init(&sm.full[s], 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s)
            if (s < nchunks)
                issue_loads(s, s);
    }

    BCPrefetch<IO, NS, T> pf;
    pf.load(a, b, 0, tid);
    pf.store(sm.bc[0], tid);
    if (nchunks > 1)
        pf.load(a, b, T, tid);
    __syncthreads();

    bool ok = true;
    int fail_ci = nchunks;
    for (int ci = 0; ci < nchunks; ++ci) {
        const int s = ci % STAGES;
        const int t0 = ci * T;
        const int tcount = min(T, a.L - t0);
        const bool got = mbar_wait_bounded(&sm.full[s], (ci / STAGES) & 1, 1u << 24);
        // uniform decision: every thread leaves the loop together, or none does
        if (__syncthreads_or(!got)) {
            if (tid == 0)
                raise_device_error(1u);
            ok = false;
            fail_ci = ci;
            break;
        }

        const IO(*xs)[kScanThreads] = sm.x[s];
        const IO(*dts)[kScanThreads] = sm.dt[s];
        const IO(*zs)[kScanThreads] = sm.z[s];
        IO(*ys)[kScanThreads] = sm.y[ci % 3];
        const float(*bc)[2][NS] = sm.bc[ci & 1];

        float xm3 = 0.f, xm2 = 0.f, xm1 = 0.f;
        if (CONV) {
            xm3 = tr::to_f(xs[0][tid]);
            xm2 = tr::to_f(xs[1][tid]);
            xm1 = tr::to_f(xs[2][tid]);
        }
#pragma unroll 2
        for (int tt = 0; tt < tcount; ++tt) {
            float u;
            if (CONV) {
                const float x0 = tr::to_f(xs[tt + kHalo][tid]);
                float pre = fmaf(w0, xm3, cb);
                pre = fmaf(w1, xm2, pre);
                pre = fmaf(w2, xm1, pre);
                pre = fmaf(w3, x0, pre);
                xm3 = xm2;
                xm2 = xm1;
                xm1 = x0;
                u = silu_f(pre);
            } else {
                u = tr::to_f(xs[tt][tid]);
            }
            const float delta = softplus_f(tr::to_f(dts[tt][tid]) + bias);
            const float du = delta * u;
            const float4 *Bq = reinterpret_cast<const float4 *>(&bc[tt][0][0]);
            const float4 *Cq = reinterpret_cast<const float4 *>(&bc[tt][1][0]);
            float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
            for (int q = 0; q < NS / 4; ++q) {
                const float4 Bv = Bq[q];
                const float4 Cv = Cq[q];
                const float Bn[4] = {Bv.x, Bv.y, Bv.z, Bv.w};
                const float Cn[4] = {Cv.x, Cv.y, Cv.z, Cv.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int n = 4 * q + j;
                    const float abar = ex2_approx(delta * A2[n]);
                    if (ZOH) {
                        // h' = abar*h + (abar-1)*k with k = B u / A, written as abar*(h+k) - k
                        const float k = rA[n] * (Bn[j] * u);
                        h[n] = fmaf(abar, h[n] + k, -k);
                    } else {
                        h[n] = fmaf(abar, h[n], du * Bn[j]);
                    }
                    if (j & 1)
                        acc1 = fmaf(h[n], Cn[j], acc1);
                    else
                        acc0 = fmaf(h[n], Cn[j], acc0);
                }
            }
            float yv = fmaf(Dd, u, acc0 + acc1);
            if (a.has_z)
                yv *= silu_f(tr::to_f(zs[tt][tid]));
            ys[tt][tid] = tr::from_f(yv);
        }

        // Stage the next chunk's B/C (prefetched into registers one chunk ago)
        // and start fetching the one after it.
        if (ci + 1 < nchunks)
            pf.store(sm.bc[(ci + 1) & 1], tid);
        if (ci + 2 < nchunks)
            pf.load(a, b, (ci + 2) * T, tid);
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tma_store_3d(&tm_y, &sm.y[ci % 3][0][0], c0, t0, b);
            bulk_commit_group();
            if (ci + STAGES < nchunks)
                issue_loads(ci + STAGES, s);
            // the y buffer written next-but-one iteration must be free again
            bulk_wait_group_read<1>();
        }
    }

    if (ok && live && a.h_final) {
        float *hf = a.h_final + (static_cast<size_t>(b) * a.d + ch) * a.N;
#pragma unroll
        for (int n = 0; n < NS; ++n)
            if (n < a.N)
                hf[n] = h[n];
    }
    if (tid == 0) {
        // after a failed wait, give the loads still in flight a bounded chance
        // to land before the shared memory they target is released
        for (int ci = fail_ci + 1; ci < nchunks && ci < fail_ci + STAGES; ++ci)
            (void)mbar_wait_bounded(&sm.full[ci % STAGES], (ci / STAGES) & 1, 1u << 20);
        bulk_wait_group<0>();
    }
}

}  // namespace s6
