// s6_block.cuh -- one token through a Mamba-mini decode block for a batch of
// sequences, sm_100a ("mamba, live", what is actually running: the per-block
// listing; its Weights paragraph: per-row symmetric int8, w = int8_row x
// scale_row, A_log in float32).
//
//     hn      = LayerNorm(x)                     x: the residual stream [Bt, dm]
//     [xin,z] = in_proj(hn)                      dm -> 2 di
//     xc      = SiLU(conv_K(xin))                (K-1)-token history per channel
//     [dt,B,C]= x_proj(xc)                       di -> R + 2N
//     Delta   = softplus(dt_proj(dt) + dt_bias)  R -> di
//     h       = 2^(Delta A log2 e) h + (Delta B) xc,   y = <h, C> + D xc
//     x      += out_proj(y SiLU(z))              di -> dm
//
// Four kernels: (1) LayerNorm fused into the in_proj product, (2) the conv +
// SiLU fused into the x_proj product (K split across blocks, partial sums
// added atomically), (3) dt_proj fused with the recurrence, one thread per
// (sequence, channel) with its N states, and (4) out_proj with the residual
// add (K split, atomic adds into x).  The products are float32 on the CUDA
// cores: the int8 weights are converted exactly when a tile is staged in
// shared memory and the row scale is applied to the finished sum.
#pragma once

#include "s6_common.cuh"

namespace s6 {

constexpr int kGemmBM = 64;  // rows (sequences) per block tile
constexpr int kGemmBN = 64;  // outputs per block tile
constexpr int kGemmBK = 32;  // reduction slice staged per step
constexpr int kGemmThreads = 256;
constexpr int kProPlain = 0;  // X read as is
constexpr int kProLN = 1;     // X = LayerNorm of the rows
constexpr int kProConv = 2;   // X = SiLU(conv(history, xin)) per (row, channel)

struct Q8GemmArgs {
    int M, N, K;
    const float *x;  // [M][ldx]: the rows (the pre-conv xin rows for kProConv)
    int ldx;
    const int8_t *wq;  // [N][K] int8 rows
    const float *ws;   // [N] row scales
    float *y;          // [M][ldy]
    int ldy;
    int accumulate;  // 1: y += (atomic adds, for split K), 0: y =
    int k_split;     // reduction length per blockIdx.z
    const float *ln_w, *ln_b;  // kProLN: [K]
    float eps;
    const float *hist;    // kProConv: [M][K][Kc-1] conv history, oldest first
    const float *conv_w;  // kProConv: [K][Kc]
    const float *conv_b;  // kProConv: [K] or null
    int Kc;
};

__device__ __forceinline__ float silu_exact(float v) { return v / (1.0f + __expf(-v)); }

// Y[m][n] (+)= ws[n] * sum_k wq[n][k] X[m][k].  A 64 x 64 output tile per
// block, 4 x 4 outputs per thread, 32-wide slices of K staged in shared memory
// (X transposed to [k][m], the int8 weights converted to float [k][n]).
template <int PRO>
__global__ void __launch_bounds__(kGemmThreads) q8_gemm_kernel(const Q8GemmArgs a) {
    constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK;
    __shared__ __align__(16) float Xs[BK][BM + 4];
    __shared__ __align__(16) float Ws[BK][BN + 4];
    __shared__ float2 stats[BM];  // kProLN: (mean, 1/sqrt(var + eps)) of each row
    const int tid = threadIdx.x;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int kb = blockIdx.z * a.k_split;
    const int ke = min(a.K, kb + a.k_split);
    const int tm = tid >> 4, tn = tid & 15;

    if (PRO == kProLN) {
        // row statistics over the whole row (this kernel is launched unsplit)
        const int warp = tid >> 5, lane = tid & 31;
        for (int r = warp; r < BM; r += kGemmThreads / 32) {
            const int m = m0 + r;
            float s = 0.f;
            if (m < a.M)
                for (int k = lane; k < a.K; k += 32)
                    s += a.x[static_cast<size_t>(m) * a.ldx + k];
#pragma unroll
            for (int o = 16; o; o >>= 1)
                s += __shfl_xor_sync(0xffffffffu, s, o);
            const float mean = s / a.K;
            float v = 0.f;
            if (m < a.M)
                for (int k = lane; k < a.K; k += 32) {
                    const float dlt = a.x[static_cast<size_t>(m) * a.ldx + k] - mean;
                    v = fmaf(dlt, dlt, v);
                }
#pragma unroll
            for (int o = 16; o; o >>= 1)
                v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0)
                stats[r] = make_float2(mean, rsqrtf(v / a.K + a.eps));
        }
        __syncthreads();
    }

    f2_t acc[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        acc[i][0] = acc[i][1] = f2_pack(0.f, 0.f);

    for (int k0 = kb; k0 < ke; k0 += BK) {
#pragma unroll
        for (int i = 0; i < (BM * BK) / kGemmThreads; ++i) {
            const int e = tid + i * kGemmThreads;
            const int r = e / BK, kk = e % BK;
            const int m = m0 + r, k = k0 + kk;
            float v = 0.f;
            if (m < a.M && k < ke) {
                if (PRO == kProConv) {
                    const float *hs = a.hist + (static_cast<size_t>(m) * a.K + k) * (a.Kc - 1);
                    const float *w = a.conv_w + static_cast<size_t>(k) * a.Kc;
                    float pre = a.conv_b ? a.conv_b[k] : 0.f;
                    for (int j = 0; j < a.Kc - 1; ++j)
                        pre = fmaf(w[j], hs[j], pre);
                    pre = fmaf(w[a.Kc - 1], a.x[static_cast<size_t>(m) * a.ldx + k], pre);
                    v = silu_exact(pre);
                } else {
                    v = a.x[static_cast<size_t>(m) * a.ldx + k];
                    if (PRO == kProLN) {
                        const float2 st = stats[r];
                        v = fmaf((v - st.x) * st.y, a.ln_w[k], a.ln_b[k]);
                    }
                }
            }
            Xs[kk][r] = v;
        }
#pragma unroll
        for (int i = 0; i < (BN * BK) / kGemmThreads; ++i) {
            const int e = tid + i * kGemmThreads;
            const int r = e / BK, kk = e % BK;
            const int n = n0 + r, k = k0 + kk;
            Ws[kk][r] = (n < a.N && k < ke) ? static_cast<float>(a.wq[static_cast<size_t>(n) * a.K + k]) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < BK; ++kk) {
            const float4 xv = *reinterpret_cast<const float4 *>(&Xs[kk][tm * 4]);
            const float4 wv = *reinterpret_cast<const float4 *>(&Ws[kk][tn * 4]);
            const f2_t w01 = f2_pack(wv.x, wv.y), w23 = f2_pack(wv.z, wv.w);
            const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const f2_t xx = f2_pack(xs[i], xs[i]);
                acc[i][0] = f2_fma(xx, w01, acc[i][0]);
                acc[i][1] = f2_fma(xx, w23, acc[i][1]);
            }
        }
        __syncthreads();
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + tm * 4 + i;
        if (m >= a.M)
            continue;
        float v[4];
        f2_unpack(acc[i][0], v[0], v[1]);
        f2_unpack(acc[i][1], v[2], v[3]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tn * 4 + j;
            if (n >= a.N)
                continue;
            const float out = v[j] * a.ws[n];
            float *dst = a.y + static_cast<size_t>(m) * a.ldy + n;
            if (a.accumulate)
                atomicAdd(dst, out);
            else
                *dst = out;
        }
    }
}

struct BlockSsmArgs {
    int Bt, di, N, R, Kc;
    const float *xz;   // [Bt][2 di]: xin | z
    const float *dbc;  // [Bt][dbc_ld]: dt | B | C (the x_proj rows, R + 2N used)
    int dbc_ld;
    const int8_t *dt_q;
    const float *dt_s, *dt_bias;  // [di][R], [di], [di]
    const float *A_log, *D;       // [di][N], [di]
    const float *conv_w, *conv_b;  // [di][Kc], [di] or null
    float *hist;  // [Bt][di][Kc-1] conv history, updated in place
    float *h;     // [Bt][di][N] state, updated in place
    float *g;     // [Bt][di] gated readout y * SiLU(z)
};

constexpr int kSsmThreads = 256;

// One thread per (sequence, channel): the conv + SiLU (history shifted in
// place), dt_proj from the sequence's R dt values, softplus, the N state
// updates and the readout, gated.  HBM-bound on h (read and written once).
template <int NS>
__global__ void __launch_bounds__(kSsmThreads) block_ssm_kernel(const BlockSsmArgs a) {
    extern __shared__ float srow[];  // this sequence's x_proj row (R + 2N floats)
    const int rowlen = a.R + 2 * a.N;
    const int m = blockIdx.y;  // the sequence
    const int c = blockIdx.x * kSsmThreads + threadIdx.x;
    for (int i = threadIdx.x; i < rowlen; i += kSsmThreads)
        srow[i] = a.dbc[static_cast<size_t>(m) * a.dbc_ld + i];
    __syncthreads();
    if (c >= a.di)
        return;
    const float xin = a.xz[static_cast<size_t>(m) * 2 * a.di + c];
    const float zv = a.xz[static_cast<size_t>(m) * 2 * a.di + a.di + c];
    // conv + SiLU, history shifted
    float *hs = a.hist + (static_cast<size_t>(m) * a.di + c) * (a.Kc - 1);
    const float *w = a.conv_w + static_cast<size_t>(c) * a.Kc;
    float pre = a.conv_b ? a.conv_b[c] : 0.f;
    float hv[3] = {0.f, 0.f, 0.f};
    for (int j = 0; j < a.Kc - 1; ++j) {
        hv[j] = hs[j];
        pre = fmaf(w[j], hv[j], pre);
    }
    pre = fmaf(w[a.Kc - 1], xin, pre);
    for (int j = 0; j + 1 < a.Kc - 1; ++j)
        hs[j] = hv[j + 1];
    hs[a.Kc - 2] = xin;
    const float xc = silu_exact(pre);
    // dt_proj + softplus
    float dtv = 0.f;
    const int8_t *q = a.dt_q + static_cast<size_t>(c) * a.R;
    for (int r = 0; r < a.R; ++r)
        dtv = fmaf(static_cast<float>(q[r]), srow[r], dtv);
    const float v = fmaf(dtv, a.dt_s[c], a.dt_bias[c]);
    const float delta = fmaxf(v, 0.f) + log1pf(__expf(-fabsf(v)));
    // the recurrence and the readout
    const float *Bm = srow + a.R, *Cm = srow + a.R + a.N;
    const float *al = a.A_log + static_cast<size_t>(c) * a.N;
    float *hp = a.h + (static_cast<size_t>(m) * a.di + c) * a.N;
    float acc = 0.f;
    const float du = delta * xc;
    if (NS == 16 && a.N == 16) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            float4 h4 = reinterpret_cast<const float4 *>(hp)[q4];
            const float4 a4 = reinterpret_cast<const float4 *>(al)[q4];
            float hh[4] = {h4.x, h4.y, h4.z, h4.w};
            const float aa[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int n = 4 * q4 + e;
                const float ab = ex2_approx(delta * (-__expf(aa[e])) * kLog2e);  // exp(Delta A), A = -exp(A_log)
                hh[e] = fmaf(ab, hh[e], du * Bm[n]);
                acc = fmaf(hh[e], Cm[n], acc);
            }
            reinterpret_cast<float4 *>(hp)[q4] = make_float4(hh[0], hh[1], hh[2], hh[3]);
        }
    } else {
        for (int n = 0; n < a.N; ++n) {
            const float ab = ex2_approx(delta * (-__expf(al[n])) * kLog2e);
            const float hn = fmaf(ab, hp[n], du * Bm[n]);
            hp[n] = hn;
            acc = fmaf(hn, Cm[n], acc);
        }
    }
    const float y = fmaf(a.D[c], xc, acc);
    a.g[static_cast<size_t>(m) * a.di + c] = y * silu_exact(zv);
}

}  // namespace s6
