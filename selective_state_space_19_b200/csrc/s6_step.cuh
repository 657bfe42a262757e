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


// ------------------------------------------------------------------------
// Pipelined form for N in {4, 8, 16}.  Per (sequence, channel) the step reads
// and writes N float32 states and touches only a few other bytes, so it runs
// at the speed the SMs can stream h.  One thread owns one channel and all of
// its N states, so the per-channel scalar work (conv, SiLU, softplus, gate) is
// done once.  Tiles are (kStepThreads consecutive channels, one sequence),
// ordered channel tile first, sequence fastest; each persistent CTA walks one
// contiguous range of them, so the per-channel parameters (conv taps, biases,
// D, the rates A log2 e from A_log) stay in registers and are reloaded only
// when the channel tile changes.  A tile's states are one contiguous run of h:
// a bulk copy brings it into a ring of kStepStages shared-memory stages
// (issued kStepStages - 1 tiles ahead), the CTA updates it in place, and a bulk
// store writes it back.  With BIO (every per-token row 16-byte aligned) the
// tile's u, Delta, z and conv-history runs travel the same way, in and out,
// and y leaves by a bulk store; otherwise they are read with plain loads one
// tile ahead and written directly.  The tile's B and C rows are staged once in
// shared memory.
constexpr int kStepStages = 4;
constexpr uint32_t kStepWaitPolls = 1u << 22;

template <typename IO, int NS>
struct StepStage {
    static constexpr int CT = kStepThreads;
    float h[CT * NS];
    IO u[CT], dt[CT], z[CT], y[CT];
    IO hist[CT * 3];  // [channel][K-1] as in memory
};

template <typename IO, int NS, bool ZOH, bool BIO>
__global__ void __launch_bounds__(kStepThreads) s6_step_bulk_kernel(const StepArgs a, const int ctiles, const int per_cta) {
    using tr = io_traits<IO>;
    using Stage = StepStage<IO, NS>;
    constexpr int CT = kStepThreads;  // channels per tile
    __shared__ alignas(128) Stage st[kStepStages];
    __shared__ alignas(16) float bcs[2][2 * NS];  // B row, C row of the tile's sequence, by tile parity
    __shared__ alignas(8) uint64_t full[kStepStages];
    static_assert(sizeof(Stage) % 16 == 0, "stages keep 16-byte alignment");
    static_assert((CT * NS * 4) % 16 == 0 && (CT * sizeof(IO)) % 16 == 0, "runs start 16-byte aligned");

    const int tid = threadIdx.x;
    // A thread's N states are NS/4 16-byte chunks of its channel's row in the
    // stage; rows of neighbouring threads are NS*4 bytes apart, so walking the
    // chunks in the same order on every thread would put several threads of a
    // warp on the same banks.  Register chunk j of this thread holds row chunk
    // j ^ rot, with rot chosen so that the 8 threads sharing a 128-byte span
    // use 8 different 16-byte bank groups; the thread's A rates and its reads
    // of B and C use the same order.
    constexpr int kChunks = NS / 4;
    const int rot = (tid / (8 / kChunks)) & (kChunks - 1);
    const long long ntiles = static_cast<long long>(ctiles) * a.Bt;
    const long long t_begin = static_cast<long long>(blockIdx.x) * per_cta;
    const long long t_end = t_begin + per_cta < ntiles ? t_begin + per_cta : ntiles;
    const int count = t_begin < t_end ? static_cast<int>(t_end - t_begin) : 0;
    const int ct_begin = static_cast<int>(t_begin / a.Bt);  // the only divisions
    const int b_begin = static_cast<int>(t_begin - static_cast<long long>(ct_begin) * a.Bt);
    const int K1 = a.K - 1;  // history length, 0..3

    if (tid == 0) {
        for (int s = 0; s < kStepStages; ++s)
            mbar_init(&full[s], 1);
        fence_mbarrier_init();
    }
    __syncthreads();

    const IO *u_p = static_cast<const IO *>(a.u);
    const IO *dt_p = static_cast<const IO *>(a.dt);
    const IO *z_p = static_cast<const IO *>(a.z);
    const IO *B_p = static_cast<const IO *>(a.B);
    const IO *C_p = static_cast<const IO *>(a.C);
    IO *cs_p = static_cast<IO *>(a.conv_state);
    IO *y_p = static_cast<IO *>(a.y);

    // tile (ct, b): first channel element g0 = b*d + c0 and channel count
    auto tile_g0 = [&](int ct, int b, size_t &g0, int &cnt) {
        const int c0 = ct * CT;
        cnt = a.d - c0 < CT ? a.d - c0 : CT;
        g0 = static_cast<size_t>(b) * a.d + c0;
    };
    // (ct, b) of the tile that the producer thread loads next
    int ld_ct = ct_begin, ld_b = b_begin, ld_i = 0;
    auto issue_next = [&]() {
        size_t g0;
        int cnt;
        tile_g0(ld_ct, ld_b, g0, cnt);
        const int s = ld_i % kStepStages;
        const uint32_t hb = static_cast<uint32_t>(cnt) * NS * 4u;  // multiples of 16 (checked on the host)
        const uint32_t ib = static_cast<uint32_t>(cnt) * sizeof(IO);
        const uint32_t cb_ = ib * static_cast<uint32_t>(K1);
        uint32_t tx = hb;
        if (BIO)
            tx += 2u * ib + (a.has_z ? ib : 0u) + cb_;
        mbar_arrive_expect_tx(&full[s], tx);
        bulk_load(st[s].h, a.h + g0 * NS, hb, &full[s]);
        if (BIO) {
            bulk_load(st[s].u, u_p + g0, ib, &full[s]);
            bulk_load(st[s].dt, dt_p + g0, ib, &full[s]);
            if (a.has_z)
                bulk_load(st[s].z, z_p + g0, ib, &full[s]);
            if (cb_)
                bulk_load(st[s].hist, cs_p + g0 * K1, cb_, &full[s]);
        }
        ++ld_i;
        if (++ld_b == a.Bt) {
            ld_b = 0;
            ++ld_ct;
        }
    };
    if (tid == 0)
        while (ld_i < count && ld_i < kStepStages - 1)
            issue_next();

    // inputs of a tile read with plain loads, one tile ahead
    float nx = 0.f, ndt = 0.f, nz = 0.f, nh0 = 0.f, nh1 = 0.f, nh2 = 0.f, nbc = 0.f;
    auto load_inputs = [&](int ct, int b) {
        const int c = ct * CT + tid;
        if (!BIO && c < a.d) {
            const size_t g = static_cast<size_t>(b) * a.d + c;
            nx = tr::to_f(u_p[g]);
            ndt = tr::to_f(dt_p[g]);
            nz = a.has_z ? tr::to_f(z_p[g]) : 0.f;
            const IO *hc = cs_p + g * K1;
            nh0 = K1 > 0 ? tr::to_f(hc[0]) : 0.f;
            nh1 = K1 > 1 ? tr::to_f(hc[1]) : 0.f;
            nh2 = K1 > 2 ? tr::to_f(hc[2]) : 0.f;
        }
        if (tid < 2 * NS)
            nbc = tr::to_f(tid < NS ? B_p[static_cast<size_t>(b) * NS + tid] : C_p[static_cast<size_t>(b) * NS + tid - NS]);
    };
    if (count > 0)
        load_inputs(ct_begin, b_begin);

    // per-channel parameters of the current channel tile
    int cur_ct = -1;
    float wh[3] = {0.f, 0.f, 0.f}, wx = 0.f, cb = 0.f, bias = 0.f, Dd = 0.f;  // taps: history, new token
    f2_t A2p[NS / 2], nrAp[NS / 2];  // pairs of states
#pragma unroll
    for (int n = 0; n < NS / 2; ++n)
        A2p[n] = nrAp[n] = f2_pack(0.f, 0.f);

    int ct = ct_begin, b = b_begin;
    for (int i = 0; i < count; ++i) {
        const int c = ct * CT + tid;
        const bool live = c < a.d;
        if (ct != cur_ct) {
            cur_ct = ct;
            if (live) {
                // tap k (oldest first) meets history element k; the last tap the new token
                const float *wc = a.conv_w + static_cast<size_t>(c) * a.K;
#pragma unroll
                for (int k = 0; k < 3; ++k)
                    wh[k] = k < K1 ? wc[k] : 0.f;
                wx = wc[K1];
                cb = a.conv_b ? a.conv_b[c] : 0.f;
                bias = a.dt_bias ? a.dt_bias[c] : 0.f;
                Dd = a.D[c];
                const float4 *al4 = reinterpret_cast<const float4 *>(a.A_log + static_cast<size_t>(c) * NS);
#pragma unroll
                for (int v = 0; v < NS / 4; ++v) {
                    const float4 al = __ldg(al4 + (v ^ rot));
                    const float alv[4] = {al.x, al.y, al.z, al.w};
                    float A2v[4], nrv[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float A = -ex2_approx(alv[j] * kLog2e);  // A = -exp(A_log)
                        A2v[j] = A * kLog2e;
                        nrv[j] = -1.0f / A;
                    }
                    A2p[2 * v] = f2_pack(A2v[0], A2v[1]);
                    A2p[2 * v + 1] = f2_pack(A2v[2], A2v[3]);
                    nrAp[2 * v] = f2_pack(nrv[0], nrv[1]);
                    nrAp[2 * v + 1] = f2_pack(nrv[2], nrv[3]);
                }
            }
        }
        float xt = nx, dtr = ndt, zr = nz, h0 = nh0, h1 = nh1, h2 = nh2;
        if (tid < 2 * NS)
            bcs[i & 1][tid] = nbc;
        int nct = ct, nb = b + 1;
        if (nb == a.Bt) {
            nb = 0;
            ++nct;
        }
        if (i + 1 < count)
            load_inputs(nct, nb);

        const int s = i % kStepStages;
        Stage &sg = st[s];
        const bool ok = mbar_wait_bounded(&full[s], static_cast<uint32_t>(i / kStepStages) & 1u, kStepWaitPolls);
        // the stage has landed everywhere (or the CTA gives up); the B/C rows are visible
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                raise_device_error(4u);
                // let the copies still in flight land before the CTA exits
                for (int j = i + 1; j < ld_i; ++j)
                    mbar_wait_bounded(&full[j % kStepStages], static_cast<uint32_t>(j / kStepStages) & 1u,
                                      kStepWaitPolls);
                bulk_wait_group<0>();
            }
            return;
        }
        if (BIO && live) {
            xt = tr::to_f(sg.u[tid]);
            dtr = tr::to_f(sg.dt[tid]);
            zr = a.has_z ? tr::to_f(sg.z[tid]) : 0.f;
            h0 = K1 > 0 ? tr::to_f(sg.hist[tid * K1]) : 0.f;
            h1 = K1 > 1 ? tr::to_f(sg.hist[tid * K1 + 1]) : 0.f;
            h2 = K1 > 2 ? tr::to_f(sg.hist[tid * K1 + 2]) : 0.f;
        }

        // this channel's scalars: conv over (history, new token), SiLU, softplus, gate
        const float hist[3] = {h0, h1, h2};
        float pre = cb;
#pragma unroll
        for (int k = 0; k < 3; ++k)
            if (k < K1)
                pre = fmaf(wh[k], hist[k], pre);
        pre = fmaf(wx, xt, pre);
        const float u = silu_f(pre);
        const float delta = softplus_f(dtr + bias);
        const float zg = a.has_z ? silu_f(zr) : 1.0f;
        const float du = delta * u;

        if (live) {
            // the N states in pairs (packed float32 arithmetic); the readout
            // sums into two accumulator pairs
            float4 *hrow = reinterpret_cast<float4 *>(&sg.h[tid * NS]);
            const float4 *B4 = reinterpret_cast<const float4 *>(&bcs[i & 1][0]);
            const float4 *C4 = reinterpret_cast<const float4 *>(&bcs[i & 1][NS]);
            const f2_t dd = f2_pack(delta, delta), duu = f2_pack(du, du), uu = f2_pack(u, u);
            f2_t acc2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
            for (int v = 0; v < NS / 4; ++v) {
                const int vr = v ^ rot;  // the row chunk in register chunk v
                const float4 h4 = hrow[vr], B = B4[vr], C = C4[vr];
                f2_t hp[2] = {f2_pack(h4.x, h4.y), f2_pack(h4.z, h4.w)};
                const f2_t Bp[2] = {f2_pack(B.x, B.y), f2_pack(B.z, B.w)};
                const f2_t Cp[2] = {f2_pack(C.x, C.y), f2_pack(C.z, C.w)};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int q = 2 * v + e;
                    float d0, d1;
                    f2_unpack(f2_mul(dd, A2p[q]), d0, d1);
                    const f2_t ab = f2_pack(ex2_approx(d0), ex2_approx(d1));  // A_bar of the pair
                    if (ZOH) {
                        const f2_t nk = f2_mul(nrAp[q], f2_mul(uu, Bp[e]));  // (B u) / (-A)
                        hp[e] = f2_fma(ab, f2_sub(hp[e], nk), nk);
                    } else {
                        hp[e] = f2_fma(ab, hp[e], f2_mul(duu, Bp[e]));
                    }
                    acc2[e] = f2_fma(hp[e], Cp[e], acc2[e]);
                }
                float h0v, h1v, h2v, h3v;
                f2_unpack(hp[0], h0v, h1v);
                f2_unpack(hp[1], h2v, h3v);
                hrow[vr] = make_float4(h0v, h1v, h2v, h3v);
            }
            float a0, a1, a2, a3;
            f2_unpack(acc2[0], a0, a1);
            f2_unpack(acc2[1], a2, a3);
            const float acc = (a0 + a1) + (a2 + a3);
            const IO yv = tr::from_f(fmaf(Dd, u, acc) * zg);
            // history shifts one place; the new token enters last
            IO *hc = BIO ? &sg.hist[tid * K1] : cs_p + (static_cast<size_t>(b) * a.d + c) * K1;
#pragma unroll
            for (int k = 0; k < 2; ++k)
                if (k + 1 < K1)
                    hc[k] = tr::from_f(hist[k + 1]);
            if (K1 > 0)
                hc[K1 - 1] = tr::from_f(xt);
            if (BIO)
                sg.y[tid] = yv;
            else
                y_p[static_cast<size_t>(b) * a.d + c] = yv;
        }
        // the updated stage goes back by bulk stores
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            size_t g0;
            int cnt;
            tile_g0(ct, b, g0, cnt);
            bulk_store(a.h + g0 * NS, sg.h, static_cast<uint32_t>(cnt) * NS * 4u);
            if (BIO) {
                const uint32_t ib = static_cast<uint32_t>(cnt) * sizeof(IO);
                bulk_store(y_p + g0, sg.y, ib);
                if (K1 > 0)
                    bulk_store(cs_p + g0 * K1, sg.hist, ib * static_cast<uint32_t>(K1));
            }
            bulk_commit_group();
            // the stage of the previous tile is free once its stores have read it
            bulk_wait_group_read<1>();
            if (ld_i < count)
                issue_next();
        }
        ct = nct;
        b = nb;
    }
    if (tid == 0)
        bulk_wait_group<0>();
}

}  // namespace s6
