// s6_conv.cuh -- standalone causal depthwise conv + SiLU, sm_100a.
//
// "mamba, live" (what is actually running): xc = SiLU(depthwise_conv4(xin)),
// 4-tap causal, per channel.  "Carry context through a selective state"
// (manifest step "local"): the conv is left-padded, reading the current and
// the K-1 earlier inputs.
//
//     out[b,t,c] = SiLU(conv_b[c] + sum_{k<K} conv_w[c,k] * x[b, t-K+1+k, c]),  x[b,<0,c] = 0
//
// HBM-bound: every input element is read once (plus 3 halo rows per tile of
// tokens) and every output written once.  Persistent CTAs walk contiguous
// ranges of tiles (ConvShape::CC channels x kConvT tokens of one sequence,
// ordered channel tile first, then sequence, then tokens); each tile and its
// 3 halo rows arrive by one TMA copy into a ring of kConvStages shared-memory
// stages issued kConvStages tiles ahead (halo rows before the sequence
// start read as zeros), which keeps tens of KB of reads in flight per SM.  A
// lane owns VEC = 16/sizeof(io) consecutive channels (one 16-byte vector per
// token row, a warp covers one 512-byte row segment) and a warp a run of
// kConvT/4 tokens, so the conv taps of the lane's channels stay in registers
// and change only with the channel tile.  Outputs go straight to global
// memory, one 16-byte store per token.  SiLU costs one special-function op
// per element: v/2 (1 + tanh(v/2)) for bfloat16 output, 2^x with a Newton
// reciprocal on the FMA pipe for float32.
#pragma once

#include "s6_common.cuh"

namespace s6 {

constexpr int kConvWarps = 4;
constexpr int kConvT = 48;      // tokens per tile
constexpr int kConvStages = 4;
constexpr uint32_t kConvWaitPolls = 1u << 22;

template <typename IO>
struct ConvShape {
    static constexpr int VEC = 16 / sizeof(IO);  // channels per lane
    static constexpr int CC = 32 * VEC;          // channels per tile (512 bytes)
    static constexpr int TW = kConvT / kConvWarps;  // tokens per warp
    union U {
        uint4 raw;
        IO v[VEC];
    };
};

struct ConvArgs {
    int Bt, L, d, K;
    int ctiles, ttiles, per_cta;  // tiles: channel tiles, token tiles per sequence, tiles per CTA
    const void *x;
    const float *conv_w;  // [d, K]
    const float *conv_b;  // [d] or null
    void *out;
};

template <typename IO>
struct ConvSmem {
    IO x[kConvStages][kConvT + 3][ConvShape<IO>::CC];  // tile rows, 3 halo rows first
    uint64_t full[kConvStages];
};

template <typename IO>
__device__ __forceinline__ float conv_silu(float v) {
    if constexpr (sizeof(IO) == 2) {
        const float hv = 0.5f * v;
        return fmaf(hv, tanh_approx(hv), hv);
    } else {
        return silu_fast(v);
    }
}

template <typename IO>
__global__ void __launch_bounds__(32 * kConvWarps) s6_conv_silu_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                                       const ConvArgs a) {
    using Sh = ConvShape<IO>;
    using tr = io_traits<IO>;
    constexpr int VEC = Sh::VEC, CC = Sh::CC, TW = Sh::TW, XR = kConvT + 3;
    extern __shared__ __align__(128) unsigned char s6_conv_smem[];
    auto &sm = *reinterpret_cast<ConvSmem<IO> *>(s6_conv_smem);
    auto &xs = sm.x;
    uint64_t *full = sm.full;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long per_seq = static_cast<long long>(a.ttiles);
    const long long ntiles = static_cast<long long>(a.ctiles) * a.Bt * per_seq;
    const long long t_begin = static_cast<long long>(blockIdx.x) * a.per_cta;
    const long long t_end = t_begin + a.per_cta < ntiles ? t_begin + a.per_cta : ntiles;
    const int count = t_begin < t_end ? static_cast<int>(t_end - t_begin) : 0;
    // tile index -> (channel tile, sequence, token tile), stepped without division
    int ct = 0, b = 0, tt = 0;
    if (count > 0) {
        const long long per_ct = a.Bt * per_seq;
        ct = static_cast<int>(t_begin / per_ct);
        const long long r = t_begin - ct * per_ct;
        b = static_cast<int>(r / per_seq);
        tt = static_cast<int>(r - b * per_seq);
    }

    if (tid == 0) {
        prefetch_tensormap(&tm_x);
        for (int s = 0; s < kConvStages; ++s)
            mbar_init(&full[s], 1);
        fence_mbarrier_init();
    }
    __syncthreads();

    int ld_ct = ct, ld_b = b, ld_tt = tt, ld_i = 0;
    auto issue_next = [&]() {
        const int s = ld_i % kConvStages;
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(XR * CC * sizeof(IO)));
        tma_load_3d(&xs[s][0][0], &tm_x, &full[s], ld_ct * CC, ld_tt * kConvT - 3, ld_b);
        ++ld_i;
        if (++ld_tt == a.ttiles) {
            ld_tt = 0;
            if (++ld_b == a.Bt) {
                ld_b = 0;
                ++ld_ct;
            }
        }
    };
    if (tid == 0)
        while (ld_i < count && ld_i < kConvStages)
            issue_next();

    float w[VEC][4], cb[VEC];
    int cur_ct = -1;
    for (int i = 0; i < count; ++i) {
        const int c_base = ct * CC + lane * VEC;
        const bool live = c_base < a.d;  // d is a multiple of VEC
        if (ct != cur_ct) {
            cur_ct = ct;
            // taps right-aligned into 4 slots (missing oldest taps are zero)
#pragma unroll
            for (int j = 0; j < VEC; ++j) {
                const int c = live ? c_base + j : 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int src = k - (4 - a.K);
                    w[j][k] = (src >= 0) ? a.conv_w[static_cast<size_t>(c) * a.K + src] : 0.0f;
                }
                cb[j] = a.conv_b ? a.conv_b[c] : 0.0f;
            }
        }
        const int s = i % kConvStages;
        const bool ok = mbar_wait_bounded(&full[s], static_cast<uint32_t>(i / kConvStages) & 1u, kConvWaitPolls);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                raise_device_error(8u);
                for (int j = i + 1; j < ld_i; ++j)
                    mbar_wait_bounded(&full[j % kConvStages], static_cast<uint32_t>(j / kConvStages) & 1u,
                                      kConvWaitPolls);
            }
            return;
        }
        // this warp's tokens: rows warp*TW + 3 .. + TW of the stage; halo the 3 rows before
        const int t0 = tt * kConvT + warp * TW;  // first token of the run
        const IO(*xr)[CC] = xs[s];
        const int r0 = warp * TW;  // stage row of token t0 - 3
        auto row = [&](int r, float (&dst)[VEC]) {
            typename Sh::U u;
            u.raw = *reinterpret_cast<const uint4 *>(&xr[r][lane * VEC]);
#pragma unroll
            for (int j = 0; j < VEC; ++j)
                dst[j] = tr::to_f(u.v[j]);
        };
        float h3[VEC], h2[VEC], h1[VEC], xt[VEC];  // x[t-3], x[t-2], x[t-1], x[t]
        row(r0, h3);
        row(r0 + 1, h2);
        row(r0 + 2, h1);
        IO *op = static_cast<IO *>(a.out) + (static_cast<size_t>(b) * a.L + t0) * a.d + c_base;
        const int tn = a.L - t0 < TW ? a.L - t0 : TW;  // tokens of the run inside the sequence
#pragma unroll 4
        for (int k = 0; k < TW; ++k) {
            row(r0 + 3 + k, xt);
            typename Sh::U o;
#pragma unroll
            for (int j = 0; j < VEC; ++j) {
                float pre = fmaf(w[j][0], h3[j], cb[j]);
                pre = fmaf(w[j][1], h2[j], pre);
                pre = fmaf(w[j][2], h1[j], pre);
                pre = fmaf(w[j][3], xt[j], pre);
                o.v[j] = tr::from_f(conv_silu<IO>(pre));
                h3[j] = h2[j];
                h2[j] = h1[j];
                h1[j] = xt[j];
            }
            if (live && k < tn)
                *reinterpret_cast<uint4 *>(op + static_cast<size_t>(k) * a.d) = o.raw;
        }
        // every thread is done with stage s: refill it with the tile kConvStages ahead
        __syncthreads();
        if (tid == 0 && ld_i < count)
            issue_next();
        if (++tt == a.ttiles) {
            tt = 0;
            if (++b == a.Bt) {
                b = 0;
                ++ct;
            }
        }
    }
}

}  // namespace s6
