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
// Kernels: LayerNorm (a warp per row); the in_proj product; the conv + SiLU
// with the history shifted in place, and the x_proj product (a block per
// sequence); dt_proj fused with the recurrence and the gate (a thread per
// (sequence, channel)); the out_proj product added into x.  The in_proj and
// out_proj products run on the tensor cores (q8_tc_gemm_kernel: TF32 with the
// activations split into two terms, float32-accurate) and otherwise on the
// CUDA cores (q8_gemm_kernel); both convert the int8 weight rows exactly when
// staging them in shared memory, apply the row scale to the finished sum and
// split the reduction across blocks with atomic adds when the output tiles
// alone would not fill the GPU.
#pragma once

#include "s6_common.cuh"

namespace s6 {

// SiLU(v) = v / (1 + e^-v), with the fast division (about 2 ulp; 0 for v
// below about -88, where e^-v overflows and SiLU is 0 to float precision)
__device__ __forceinline__ float silu_exact(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

// Four int8 values (bytes of w, lowest first) as floats without the
// conversion unit: each byte, biased to unsigned (b + 128), is placed under the
// exponent of 2^23 -- the float 2^23 + b + 128, exact -- and 2^23 + 128 is
// subtracted.
__device__ __forceinline__ float4 i8x4_to_f32x4(int w) {
    const unsigned u = static_cast<unsigned>(w) ^ 0x80808080u;
    constexpr float kBias = 8388608.0f + 128.0f;
    return make_float4(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7440)) - kBias,
                       __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7441)) - kBias,
                       __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7442)) - kBias,
                       __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7443)) - kBias);
}

// ------------------------------------------------------------ LayerNorm
constexpr int kLnThreads = 256;  // 8 rows per block, a warp per row

constexpr int kLnPerLane = 32;   // rows up to 1024 values are held in registers
constexpr int kLnVec = 4;        // float4 per lane of the vector path (rows up to 512 values)

// out[m] = (x[m] - mean) / sqrt(var + eps) * w + b (biased variance).  The
// row is read once into registers (two-pass statistics from them); longer
// rows are read again for each pass.  Rows of up to 512 values in whole
// 16-byte units move as float4, with the weights and biases loaded alongside.
__global__ void __launch_bounds__(kLnThreads) block_layernorm_kernel(const float *x, const float *w, const float *b,
                                                                     float *out, int M, int K, float eps) {
    const int m = blockIdx.x * (kLnThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (m >= M)
        return;
    const float *xr = x + static_cast<size_t>(m) * K;
    float *orow = out + static_cast<size_t>(m) * K;
    if (K % 4 == 0 && K <= 32 * 4 * kLnVec &&
        ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(b) |
          reinterpret_cast<uintptr_t>(out)) & 15u) == 0) {
        // the row, the weights and the biases as float4, all loads issued first
        const int K4 = K / 4;
        const float4 *x4 = reinterpret_cast<const float4 *>(xr);
        float4 v[kLnVec], wv[kLnVec], bv[kLnVec];
        const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < kLnVec; ++i) {
            const int k4 = lane + 32 * i;
            const bool in = k4 < K4;
            v[i] = in ? x4[k4] : zero;
            wv[i] = in ? reinterpret_cast<const float4 *>(w)[k4] : zero;
            bv[i] = in ? reinterpret_cast<const float4 *>(b)[k4] : zero;
        }
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < kLnVec; ++i)
            s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
#pragma unroll
        for (int o = 16; o; o >>= 1)
            s += __shfl_xor_sync(0xffffffffu, s, o);
        const float mean = s / K;
        float q = 0.f;
#pragma unroll
        for (int i = 0; i < kLnVec; ++i) {
            if (lane + 32 * i < K4) {
                const float d0 = v[i].x - mean, d1 = v[i].y - mean, d2 = v[i].z - mean, d3 = v[i].w - mean;
                q = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, fmaf(d3, d3, q))));
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1)
            q += __shfl_xor_sync(0xffffffffu, q, o);
        const float r = rsqrtf(q / K + eps);
        float4 *o4 = reinterpret_cast<float4 *>(orow);
#pragma unroll
        for (int i = 0; i < kLnVec; ++i) {
            const int k4 = lane + 32 * i;
            if (k4 < K4)
                o4[k4] = make_float4(fmaf((v[i].x - mean) * r, wv[i].x, bv[i].x),
                                     fmaf((v[i].y - mean) * r, wv[i].y, bv[i].y),
                                     fmaf((v[i].z - mean) * r, wv[i].z, bv[i].z),
                                     fmaf((v[i].w - mean) * r, wv[i].w, bv[i].w));
        }
        return;
    }
    if (K <= 32 * kLnPerLane) {
        float v[kLnPerLane];
#pragma unroll
        for (int i = 0; i < kLnPerLane; ++i) {
            const int k = lane + 32 * i;
            v[i] = k < K ? xr[k] : 0.f;
        }
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < kLnPerLane; ++i)
            s += v[i];
#pragma unroll
        for (int o = 16; o; o >>= 1)
            s += __shfl_xor_sync(0xffffffffu, s, o);
        const float mean = s / K;
        float q = 0.f;
#pragma unroll
        for (int i = 0; i < kLnPerLane; ++i) {
            const int k = lane + 32 * i;
            const float d = k < K ? v[i] - mean : 0.f;
            q = fmaf(d, d, q);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1)
            q += __shfl_xor_sync(0xffffffffu, q, o);
        const float r = rsqrtf(q / K + eps);
#pragma unroll
        for (int i = 0; i < kLnPerLane; ++i) {
            const int k = lane + 32 * i;
            if (k < K)
                orow[k] = fmaf((v[i] - mean) * r, w[k], b[k]);
        }
        return;
    }
    float s = 0.f;
    for (int k = lane; k < K; k += 32)
        s += xr[k];
#pragma unroll
    for (int o = 16; o; o >>= 1)
        s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / K;
    float q = 0.f;
    for (int k = lane; k < K; k += 32) {
        const float d = xr[k] - mean;
        q = fmaf(d, d, q);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        q += __shfl_xor_sync(0xffffffffu, q, o);
    const float r = rsqrtf(q / K + eps);
    for (int k = lane; k < K; k += 32)
        orow[k] = fmaf((xr[k] - mean) * r, w[k], b[k]);
}

// ------------------------------------------------------------ conv + x_proj
struct BlockSsmArgs {
    int Bt, di, N, R;
    const float *xz;   // [Bt][xz_ld]: xin | z
    const float *xc;   // [Bt][xc_ld]: SiLU(conv(xin))
    int xz_ld, xc_ld, g_ld;
    const float *dbc;  // [Bt][dbc_ld]: dt | B | C (the x_proj rows, R + 2N used)
    int dbc_ld;
    const int8_t *dt_q;
    const float *dt_s, *dt_bias;  // [di][R], [di], [di]
    const float *A_log, *D;       // [di][N], [di]
    float *h;  // [Bt][di][N] state, updated in place
    float *g;  // [Bt][g_ld] gated readout y * SiLU(z)
};

constexpr int kConvXThreads = 256;
constexpr int kXprojIt = 12;  // x_proj weight words a lane holds per row (rows of up to 12 x 128 channels)

// Asks the L2 to fetch [p, p + bytes) ahead of use: p 16-byte aligned, bytes a
// multiple of 16, the range inside one allocation.
__device__ __forceinline__ void bulk_prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// One block per sequence m: xc[c] = SiLU(conv_b + sum_{j<K-1} w[j] hist[j] +
// w[K-1] xin[c]) for every channel (the history drops its oldest input and
// appends xin), kept in shared memory and written out; then the x_proj rows
// dbc[m][o] = xp_s[o] * sum_c xp_q[o][c] xc[c], each row split over four
// consecutive threads (a quarter of the channels each) and summed by shuffles.
// SSM: the recurrence of the sequence follows in the same block (N = 16,
// 16-byte aligned h and A_log rows): xc and the x_proj row stay in shared
// memory, and xc, dbc are not written out; the sequence's state row is sent
// to the L2 when the block starts, so the recurrence does not wait on HBM.
// With rows of up to 12 x 128 channels (a multiple of 4), a lane holds a
// row's weight words in registers and fetches the next row's while it sums
// this one.
template <bool SSM>
__global__ void __launch_bounds__(kConvXThreads, 2) block_conv_xproj_kernel(
    const float *__restrict__ xz, int ldxz, const float *__restrict__ conv_w, const float *__restrict__ conv_b,
    float *__restrict__ hist, float *__restrict__ xc, int ldxc, const int8_t *__restrict__ xp_q,
    const float *__restrict__ xp_s, float *__restrict__ dbc, int ld_dbc, int di, int Kc, int n_out,
    const BlockSsmArgs sa) {
    extern __shared__ __align__(16) float xcs[];  // di floats, rounded up to 4 (+ the x_proj row with SSM)
    const int m = blockIdx.x;
    if constexpr (SSM) {
        // the state row h[m] (di x 16 floats), in pieces of at most 16 KB
        constexpr uint32_t kPiece = 16384;
        const uint32_t bytes = static_cast<uint32_t>(di) * 16u * sizeof(float);
        const char *row = reinterpret_cast<const char *>(sa.h + static_cast<size_t>(m) * di * 16);
        for (uint32_t off = threadIdx.x * kPiece; off < bytes; off += kConvXThreads * kPiece)
            bulk_prefetch_l2(row + off, min(kPiece, bytes - off));
    }
    // conv: a thread's channels in groups of 4, every load of a group issued first
    for (int c0 = threadIdx.x; c0 < di; c0 += 4 * kConvXThreads) {
        float xin[4], hv[4][3], wv[4][4], bv[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int c = c0 + g * kConvXThreads;
            xin[g] = 0.f;
            bv[g] = 0.f;
#pragma unroll
            for (int j = 0; j < 3; ++j)
                hv[g][j] = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                wv[g][j] = 0.f;
            if (c < di) {
                xin[g] = xz[static_cast<size_t>(m) * ldxz + c];
                const float *hs = hist + (static_cast<size_t>(m) * di + c) * (Kc - 1);
#pragma unroll
                for (int j = 0; j < 3; ++j)
                    if (j < Kc - 1)
                        hv[g][j] = hs[j];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (j < Kc)
                        wv[g][j] = conv_w[static_cast<size_t>(c) * Kc + j];
                bv[g] = conv_b ? conv_b[c] : 0.f;
            }
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int c = c0 + g * kConvXThreads;
            if (c >= di)
                continue;
            // taps: w[j] on the history (oldest first), w[Kc-1] on xin
            float pre = bv[g];
#pragma unroll
            for (int j = 0; j < 3; ++j)
                if (j < Kc - 1)
                    pre = fmaf(wv[g][j], hv[g][j], pre);
            float wlast = wv[g][3];
            if (Kc == 3)
                wlast = wv[g][2];
            else if (Kc == 2)
                wlast = wv[g][1];
            pre = fmaf(wlast, xin[g], pre);
            float *hs = hist + (static_cast<size_t>(m) * di + c) * (Kc - 1);
#pragma unroll
            for (int j = 0; j < 2; ++j)
                if (j + 1 < Kc - 1)
                    hs[j] = hv[g][j + 1];
            hs[Kc - 2] = xin[g];
            const float v = silu_exact(pre);
            xcs[c] = v;
            if (!SSM)
                xc[static_cast<size_t>(m) * ldxc + c] = v;
        }
    }
    __syncthreads();
    // x_proj: a warp per output row, lanes over 4-channel groups (coalesced
    // weight rows, consecutive float4 of xc)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool vec = (di % 4) == 0 && (reinterpret_cast<uintptr_t>(xp_q) & 3) == 0;
    const int n4 = di / 4;
    if (vec && n4 <= 32 * kXprojIt) {
        // a row's words in registers; the next row's loads go out before this row's sums
        const float4 *x4 = reinterpret_cast<const float4 *>(xcs);
        int wq[kXprojIt], wn[kXprojIt];
        auto fetch = [&](int o, int (&w)[kXprojIt]) {
            const int *qw = reinterpret_cast<const int *>(xp_q + static_cast<size_t>(o) * di);
#pragma unroll
            for (int k = 0; k < kXprojIt; ++k) {
                const int c4 = lane + 32 * k;
                w[k] = c4 < n4 ? __ldg(qw + c4) : 0;
            }
        };
        if (warp < n_out)
            fetch(warp, wq);
        for (int o = warp; o < n_out; o += kConvXThreads / 32) {
            if (o + kConvXThreads / 32 < n_out)
                fetch(o + kConvXThreads / 32, wn);
            // the four column accumulators as two packed pairs
            f2_t acc01 = f2_pack(0.f, 0.f), acc23 = acc01;
#pragma unroll
            for (int k = 0; k < kXprojIt; ++k) {
                const int c4 = lane + 32 * k;
                if (c4 < n4) {
                    const float4 wv = i8x4_to_f32x4(wq[k]);
                    const float4 xv = x4[c4];
                    acc01 = f2_fma(f2_pack(wv.x, wv.y), f2_pack(xv.x, xv.y), acc01);
                    acc23 = f2_fma(f2_pack(wv.z, wv.w), f2_pack(xv.z, xv.w), acc23);
                }
            }
            float a0, a1, a2, a3;
            f2_unpack(acc01, a0, a1);
            f2_unpack(acc23, a2, a3);
            float sum = (a0 + a1) + (a2 + a3);
#pragma unroll
            for (int off = 16; off; off >>= 1)
                sum += __shfl_xor_sync(0xffffffffu, sum, off);
            if (lane == 0) {
                if (SSM)
                    xcs[((di + 3) & ~3) + o] = sum * xp_s[o];
                else
                    dbc[static_cast<size_t>(m) * ld_dbc + o] = sum * xp_s[o];
            }
#pragma unroll
            for (int k = 0; k < kXprojIt; ++k)
                wq[k] = wn[k];
        }
    }
    for (int o = warp; !(vec && n4 <= 32 * kXprojIt) && o < n_out; o += kConvXThreads / 32) {
        const int8_t *q = xp_q + static_cast<size_t>(o) * di;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (vec) {
            const int *qw = reinterpret_cast<const int *>(q);
            const float4 *x4 = reinterpret_cast<const float4 *>(xcs);
#pragma unroll 4
            for (int c4 = lane; c4 < di / 4; c4 += 32) {
                const float4 wv = i8x4_to_f32x4(qw[c4]);
                const float4 xv = x4[c4];
                acc[0] = fmaf(wv.x, xv.x, acc[0]);
                acc[1] = fmaf(wv.y, xv.y, acc[1]);
                acc[2] = fmaf(wv.z, xv.z, acc[2]);
                acc[3] = fmaf(wv.w, xv.w, acc[3]);
            }
        } else {
#pragma unroll 4
            for (int c = lane; c < di; c += 32)
                acc[c & 3] = fmaf(static_cast<float>(q[c]), xcs[c], acc[c & 3]);
        }
        float sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
#pragma unroll
        for (int off = 16; off; off >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0) {
            if (SSM)
                xcs[((di + 3) & ~3) + o] = sum * xp_s[o];
            else
                dbc[static_cast<size_t>(m) * ld_dbc + o] = sum * xp_s[o];
        }
    }
    if constexpr (SSM) {
        // the recurrence of this sequence, two channels per step with all of
        // their loads issued first: dt_proj (R int8 weights on the dt part of
        // the x_proj row), softplus, the 16 state updates, readout and gate
        __syncthreads();
        const float *srow = xcs + ((di + 3) & ~3);
        const float *Bm = srow + sa.R, *Cm = srow + sa.R + 16;
        const bool vec_dt = (sa.R % 4) == 0 && (reinterpret_cast<uintptr_t>(sa.dt_q) & 3) == 0;
        const bool vec_bc = (sa.R % 4) == 0;  // the x_proj row in shared memory starts 16-byte aligned
        for (int c0 = threadIdx.x; c0 < di; c0 += 2 * kConvXThreads) {
            float4 h4[2][4], a4[2][4];
            float zv[2];
            int cc[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int c = c0 + k * kConvXThreads;
                cc[k] = c < di ? c : di - 1;  // a spare lane repeats a channel it does not store
                const float4 *hp = reinterpret_cast<const float4 *>(sa.h + (static_cast<size_t>(m) * di + cc[k]) * 16);
                const float4 *ap = reinterpret_cast<const float4 *>(sa.A_log + static_cast<size_t>(cc[k]) * 16);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    h4[k][q4] = hp[q4];
                    a4[k][q4] = ap[q4];
                }
                zv[k] = sa.xz[static_cast<size_t>(m) * sa.xz_ld + di + cc[k]];
            }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int c = c0 + k * kConvXThreads;
                const int8_t *q = sa.dt_q + static_cast<size_t>(cc[k]) * sa.R;
                float dtv = 0.f;
                if (vec_dt) {
                    const int *qw = reinterpret_cast<const int *>(q);
                    for (int r4 = 0; r4 < sa.R / 4; ++r4) {
                        const float4 w = i8x4_to_f32x4(qw[r4]);
                        dtv = fmaf(w.x, srow[4 * r4], dtv);
                        dtv = fmaf(w.y, srow[4 * r4 + 1], dtv);
                        dtv = fmaf(w.z, srow[4 * r4 + 2], dtv);
                        dtv = fmaf(w.w, srow[4 * r4 + 3], dtv);
                    }
                } else {
                    for (int r = 0; r < sa.R; ++r)
                        dtv = fmaf(static_cast<float>(q[r]), srow[r], dtv);
                }
                const float v = fmaf(dtv, sa.dt_s[cc[k]], sa.dt_bias[cc[k]]);
                const float delta = fmaxf(v, 0.f) + log1pf(__expf(-fabsf(v)));  // softplus
                const float x_c = xcs[cc[k]];
                const float du = delta * x_c;
                const float dl2 = -delta * kLog2e;
                const f2_t l2e2 = f2_pack(kLog2e, kLog2e), dl22 = f2_pack(dl2, dl2), du2 = f2_pack(du, du);
                f2_t acc2 = f2_pack(0.f, 0.f);
                float4 *hp = reinterpret_cast<float4 *>(sa.h + (static_cast<size_t>(m) * di + cc[k]) * 16);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float hh[4] = {h4[k][q4].x, h4[k][q4].y, h4[k][q4].z, h4[k][q4].w};
                    const float aa[4] = {a4[k][q4].x, a4[k][q4].y, a4[k][q4].z, a4[k][q4].w};
                    float bq[4], cq[4];
                    if (vec_bc) {  // B and C rows as 16-byte reads (R a multiple of 4)
                        const float4 b4 = reinterpret_cast<const float4 *>(Bm)[q4];
                        const float4 c4 = reinterpret_cast<const float4 *>(Cm)[q4];
                        bq[0] = b4.x, bq[1] = b4.y, bq[2] = b4.z, bq[3] = b4.w;
                        cq[0] = c4.x, cq[1] = c4.y, cq[2] = c4.z, cq[3] = c4.w;
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            bq[e] = Bm[4 * q4 + e];
                            cq[e] = Cm[4 * q4 + e];
                        }
                    }
                    // two states at a time: exp(A_log) = 2^(A_log log2 e) = -A, then
                    // exp(Delta A) = 2^(-Delta log2 e exp(A_log)); update and readout
#pragma unroll
                    for (int e = 0; e < 4; e += 2) {
                        float t0, t1;
                        f2_unpack(f2_mul(f2_pack(aa[e], aa[e + 1]), l2e2), t0, t1);
                        f2_unpack(f2_mul(dl22, f2_pack(ex2_approx(t0), ex2_approx(t1))), t0, t1);
                        const f2_t ab = f2_pack(ex2_approx(t0), ex2_approx(t1));
                        const f2_t h2 = f2_fma(ab, f2_pack(hh[e], hh[e + 1]), f2_mul(du2, f2_pack(bq[e], bq[e + 1])));
                        acc2 = f2_fma(h2, f2_pack(cq[e], cq[e + 1]), acc2);
                        f2_unpack(h2, hh[e], hh[e + 1]);
                    }
                    if (c < di)
                        hp[q4] = make_float4(hh[0], hh[1], hh[2], hh[3]);
                }
                float acc0, acc1;
                f2_unpack(acc2, acc0, acc1);
                if (c < di)
                    sa.g[static_cast<size_t>(m) * sa.g_ld + c] = fmaf(sa.D[c], x_c, acc0 + acc1) * silu_exact(zv[k]);
            }
        }
    }
}

// ------------------------------------------------------------ int8 products
constexpr int kGemmBM = 64;  // rows (sequences) per block tile
constexpr int kGemmBN = 64;  // outputs per block tile
constexpr int kGemmBK = 32;  // reduction slice staged per step
constexpr int kGemmThreads = 256;

struct Q8GemmArgs {
    int M, N, K;
    const float *x;  // [M][ldx]
    int ldx;
    const int8_t *wq;  // [N][K] int8 rows
    const float *ws;   // [N] row scales
    float *y;          // [M][ldy]
    int ldy;
    int accumulate;  // 1: y += (atomic adds, for a split reduction), 0: y =
    int k_split;     // reduction length per blockIdx.z (a multiple of kGemmBK)
};

// dynamic shared memory of q8_gemm_kernel: two slices of X and of W
constexpr size_t kGemmSmem = 2 * (kGemmBM + kGemmBN) * (kGemmBK + 4) * sizeof(float);

// Y[m][n] (+)= ws[n] * sum_k wq[n][k] X[m][k].  A 64 x 64 output tile per
// block; thread (tm, tn) owns rows tm + 16 i and outputs tn + 16 j (i, j < 4),
// so that the 128-bit shared-memory reads of a quarter warp hit distinct banks.
// 32-wide K slices are staged row-major with a 4-float pad, the next slice
// read into registers while the current one is multiplied.  VEC: every X row
// start is 16-byte aligned and every W row 8-byte aligned (ldx % 4 == 0,
// K % 8 == 0, aligned bases), so slices move as float4 / 8-byte vectors.
template <bool VEC>
__global__ void __launch_bounds__(kGemmThreads) q8_gemm_kernel(const Q8GemmArgs a) {
    constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK, LD = BK + 4;
    extern __shared__ __align__(16) float gemm_smem[];
    float(*Xs)[BM][LD] = reinterpret_cast<float(*)[BM][LD]>(gemm_smem);             // [2][BM][LD]
    float(*Ws)[BN][LD] = reinterpret_cast<float(*)[BN][LD]>(gemm_smem + 2 * BM * LD);  // [2][BN][LD]
    const int tid = threadIdx.x;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int kb = blockIdx.z * a.k_split;
    const int ke = min(a.K, kb + a.k_split);
    const int tm = tid >> 4, tn = tid & 15;
    // staging: each thread moves 8 consecutive k of one X row and of one W row
    constexpr int G = BK / 32;                   // groups of 8 per thread
    const int lr = tid >> 2;                     // row within the tile (0..63)
    const int lk = (tid & 3) * (8 * G);          // first k of its 8 G
    float xr[8 * G], wr[8 * G];
    auto fetch = [&](int k0) {
        const int m = m0 + lr, n = n0 + lr;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int k = k0 + lk + 8 * g;
            float *xo = xr + 8 * g, *wo = wr + 8 * g;
            if (VEC && k + 8 <= ke) {
                if (m < a.M) {
                    const float4 *src = reinterpret_cast<const float4 *>(a.x + static_cast<size_t>(m) * a.ldx + k);
                    const float4 v0 = src[0], v1 = src[1];
                    xo[0] = v0.x;
                    xo[1] = v0.y;
                    xo[2] = v0.z;
                    xo[3] = v0.w;
                    xo[4] = v1.x;
                    xo[5] = v1.y;
                    xo[6] = v1.z;
                    xo[7] = v1.w;
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        xo[e] = 0.f;
                }
                if (n < a.N) {
                    const uint2 q = *reinterpret_cast<const uint2 *>(a.wq + static_cast<size_t>(n) * a.K + k);
                    const float4 w0 = i8x4_to_f32x4(static_cast<int>(q.x)), w1 = i8x4_to_f32x4(static_cast<int>(q.y));
                    wo[0] = w0.x;
                    wo[1] = w0.y;
                    wo[2] = w0.z;
                    wo[3] = w0.w;
                    wo[4] = w1.x;
                    wo[5] = w1.y;
                    wo[6] = w1.z;
                    wo[7] = w1.w;
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        wo[e] = 0.f;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int kk = k + e;
                    xo[e] = (m < a.M && kk < ke) ? a.x[static_cast<size_t>(m) * a.ldx + kk] : 0.f;
                    wo[e] = (n < a.N && kk < ke) ? static_cast<float>(a.wq[static_cast<size_t>(n) * a.K + kk]) : 0.f;
                }
            }
        }
    };
    auto stage = [&](int buf) {
#pragma unroll
        for (int q = 0; q < 2 * G; ++q) {
            *reinterpret_cast<float4 *>(&Xs[buf][lr][lk + 4 * q]) =
                make_float4(xr[4 * q], xr[4 * q + 1], xr[4 * q + 2], xr[4 * q + 3]);
            *reinterpret_cast<float4 *>(&Ws[buf][lr][lk + 4 * q]) =
                make_float4(wr[4 * q], wr[4 * q + 1], wr[4 * q + 2], wr[4 * q + 3]);
        }
    };

    f2_t acc[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        acc[i][0] = acc[i][1] = f2_pack(0.f, 0.f);

    int buf = 0;
    if (kb < ke) {
        fetch(kb);
        stage(0);
    }
    __syncthreads();
    for (int k0 = kb; k0 < ke; k0 += BK) {
        const bool more = k0 + BK < ke;
        if (more)
            fetch(k0 + BK);  // in flight while this slice is multiplied
#pragma unroll
        for (int kq = 0; kq < BK; kq += 4) {
            float xk[4][4], wk[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 xv = *reinterpret_cast<const float4 *>(&Xs[buf][tm + 16 * i][kq]);
                const float4 wv = *reinterpret_cast<const float4 *>(&Ws[buf][tn + 16 * i][kq]);
                xk[i][0] = xv.x;
                xk[i][1] = xv.y;
                xk[i][2] = xv.z;
                xk[i][3] = xv.w;
                wk[i][0] = wv.x;
                wk[i][1] = wv.y;
                wk[i][2] = wv.z;
                wk[i][3] = wv.w;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const f2_t w01 = f2_pack(wk[0][e], wk[1][e]);
                const f2_t w23 = f2_pack(wk[2][e], wk[3][e]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const f2_t xx = f2_pack(xk[i][e], xk[i][e]);
                    acc[i][0] = f2_fma(xx, w01, acc[i][0]);
                    acc[i][1] = f2_fma(xx, w23, acc[i][1]);
                }
            }
        }
        if (more) {
            stage(buf ^ 1);
            __syncthreads();
            buf ^= 1;
        }
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + tm + 16 * i;
        if (m >= a.M)
            continue;
        float v[4];
        f2_unpack(acc[i][0], v[0], v[1]);
        f2_unpack(acc[i][1], v[2], v[3]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tn + 16 * j;
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

// ------------------------------------------ int8 products on the tensor cores
// The same product, Y[m][n] (+)= ws[n] * sum_k wq[n][k] X[m][k], with
// mma.sync m16n8k8 in TF32.  An int8 weight is exact in TF32; an activation
// is split as x = hi + lo, both TF32 (hi = x rounded to TF32, lo = the rest
// rounded again), so hi*w + lo*w carries x*w to about 2^-22 of its size -- the
// float32 product, from two tensor-core products instead of one.
//
// A 64 x 64 output tile per block of four warps, each warp 32 x 32 (2 x 4
// m16n8 tiles); 32-wide K slices staged in shared memory as (hi, lo, w) rows
// with a 4-float pad, which puts the eight rows x four columns of a fragment
// load on 32 distinct banks; the next slice is read into registers while the
// current one is multiplied.  Needs the VEC layout of q8_gemm_kernel and
// K % 16 == 0 (16-byte weight loads).
constexpr int kTcThreads = 128;
constexpr int kTcLD = kGemmBK + 4;
constexpr size_t kTcSmem = 2 * 3 * 64 * kTcLD * sizeof(float);

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kTcThreads) q8_tc_gemm_kernel(const Q8GemmArgs a) {
    constexpr int BK = kGemmBK, LD = kTcLD;
    extern __shared__ __align__(16) float tc_smem[];
    // [buf][0: hi, 1: lo, 2: w][row][LD]
    auto sm = [&](int buf, int part, int row, int col) -> float * {
        return tc_smem + ((buf * 3 + part) * 64 + row) * LD + col;
    };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    const int kb = blockIdx.z * a.k_split;
    const int ke = min(a.K, kb + a.k_split);
    // staging: thread -> tile row tid / 2, 16 consecutive k from (tid & 1) * 16
    const int lr = tid >> 1, lk = (tid & 1) * 16;
    float4 xr[4];
    int4 wr;
    auto fetch = [&](int k0) {
        const int m = m0 + lr, n = n0 + lr, k = k0 + lk;
        const bool kin = k + 16 <= ke;  // slices are whole (K, k_split multiples of 16)
        if (m < a.M && kin) {
            const float4 *src = reinterpret_cast<const float4 *>(a.x + static_cast<size_t>(m) * a.ldx + k);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                xr[q] = src[q];
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                xr[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        wr = (n < a.N && kin) ? *reinterpret_cast<const int4 *>(a.wq + static_cast<size_t>(n) * a.K + k)
                              : make_int4(0, 0, 0, 0);
    };
    auto stage = [&](int buf) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float v[4] = {xr[q].x, xr[q].y, xr[q].z, xr[q].w};
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                hi[e] = to_tf32(v[e]);
                lo[e] = to_tf32(v[e] - __uint_as_float(hi[e]));
            }
            *reinterpret_cast<uint4 *>(sm(buf, 0, lr, lk + 4 * q)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(sm(buf, 1, lr, lk + 4 * q)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        const int wv[4] = {wr.x, wr.y, wr.z, wr.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
            *reinterpret_cast<float4 *>(sm(buf, 2, lr, lk + 4 * q)) = i8x4_to_f32x4(wv[q]);
    };

    float acc[2][4][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                acc[i][j][e] = 0.f;

    int buf = 0;
    if (kb < ke) {
        fetch(kb);
        stage(0);
    }
    __syncthreads();
    for (int k0 = kb; k0 < ke; k0 += BK) {
        const bool more = k0 + BK < ke;
        if (more)
            fetch(k0 + BK);  // in flight while this slice is multiplied
#pragma unroll
        for (int kk = 0; kk < BK; kk += 8) {
            uint32_t ah[2][4], al[2][4], bw[4][2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int r = wm + 16 * i + g;
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const float *h = sm(buf, p, r, kk + t);
                    uint32_t(&f)[4] = p ? al[i] : ah[i];
                    f[0] = __float_as_uint(h[0]);
                    f[1] = __float_as_uint(h[8 * LD]);
                    f[2] = __float_as_uint(h[4]);
                    f[3] = __float_as_uint(h[8 * LD + 4]);
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float *wp = sm(buf, 2, wn + 8 * j + g, kk + t);
                bw[j][0] = __float_as_uint(wp[0]);
                bw[j][1] = __float_as_uint(wp[4]);
            }
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    mma_tf32(acc[i][j], al[i], bw[j][0], bw[j][1]);
                    mma_tf32(acc[i][j], ah[i], bw[j][0], bw[j][1]);
                }
        }
        if (more) {
            // the other buffer was last read before the previous barrier
            stage(buf ^ 1);
            __syncthreads();
            buf ^= 1;
        }
    }

    // accumulator (i, j): rows wm + 16 i + g (+8), columns wn + 8 j + 2 t (+1);
    // a split reduction adds a thread's two adjacent columns with one 8-byte
    // atomic when the output rows allow it (half the atomic operations; 16-byte
    // atomics after a lane-pair exchange measured slower)
    const bool pairs =
        a.accumulate && ((reinterpret_cast<uintptr_t>(a.y) | static_cast<uintptr_t>(a.ldy) * 4u) & 7u) == 0;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + wn + 8 * j + 2 * t;
#pragma unroll
            for (int hrow = 0; hrow < 2; ++hrow) {
                const int m = m0 + wm + 16 * i + g + 8 * hrow;
                if (m >= a.M)
                    continue;
                if (pairs && n + 1 < a.N) {
                    float2 *dst = reinterpret_cast<float2 *>(a.y + static_cast<size_t>(m) * a.ldy + n);
                    atomicAdd(dst, make_float2(acc[i][j][2 * hrow] * a.ws[n], acc[i][j][2 * hrow + 1] * a.ws[n + 1]));
                    continue;
                }
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    if (n + e >= a.N)
                        continue;
                    const float out = acc[i][j][2 * hrow + e] * a.ws[n + e];
                    float *dst = a.y + static_cast<size_t>(m) * a.ldy + n + e;
                    if (a.accumulate)
                        atomicAdd(dst, out);
                    else
                        *dst = out;
                }
            }
        }
}

constexpr int kSsmThreads = 256;

// One thread per (sequence, channel): dt_proj from the sequence's R dt values,
// softplus, the N state updates and the readout, gated.  HBM-bound on h (read
// and written once).  Block (x, y): channels 256 x .. of sequence y.
template <int NS>
__global__ void __launch_bounds__(kSsmThreads) block_ssm_kernel(const BlockSsmArgs a) {
    extern __shared__ float srow[];  // this sequence's x_proj row (R + 2N floats)
    const int rowlen = a.R + 2 * a.N;
    const int m = blockIdx.y;
    const int c = blockIdx.x * kSsmThreads + threadIdx.x;
    for (int i = threadIdx.x; i < rowlen; i += kSsmThreads)
        srow[i] = a.dbc[static_cast<size_t>(m) * a.dbc_ld + i];
    __syncthreads();
    if (c >= a.di)
        return;
    const float xc = a.xc[static_cast<size_t>(m) * a.xc_ld + c];
    const float zv = a.xz[static_cast<size_t>(m) * a.xz_ld + a.di + c];
    float *hp = a.h + (static_cast<size_t>(m) * a.di + c) * a.N;
    const float *al = a.A_log + static_cast<size_t>(c) * a.N;
    float4 h4[4], a4[4];
    if (NS == 16 && a.N == 16) {  // the state and its rates in flight first
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            h4[q4] = reinterpret_cast<const float4 *>(hp)[q4];
            a4[q4] = reinterpret_cast<const float4 *>(al)[q4];
        }
    }
    float dtv = 0.f;
    const int8_t *q = a.dt_q + static_cast<size_t>(c) * a.R;
    if ((a.R % 4) == 0 && (reinterpret_cast<uintptr_t>(a.dt_q) & 3) == 0) {
        const int *qw = reinterpret_cast<const int *>(q);
#pragma unroll 6
        for (int r4 = 0; r4 < a.R / 4; ++r4) {
            const int wv = qw[r4];
            dtv = fmaf(static_cast<float>(static_cast<int8_t>(wv & 0xff)), srow[4 * r4], dtv);
            dtv = fmaf(static_cast<float>(static_cast<int8_t>((wv >> 8) & 0xff)), srow[4 * r4 + 1], dtv);
            dtv = fmaf(static_cast<float>(static_cast<int8_t>((wv >> 16) & 0xff)), srow[4 * r4 + 2], dtv);
            dtv = fmaf(static_cast<float>(static_cast<int8_t>((wv >> 24) & 0xff)), srow[4 * r4 + 3], dtv);
        }
    } else {
        for (int r = 0; r < a.R; ++r)
            dtv = fmaf(static_cast<float>(q[r]), srow[r], dtv);
    }
    const float v = fmaf(dtv, a.dt_s[c], a.dt_bias[c]);
    const float delta = fmaxf(v, 0.f) + log1pf(__expf(-fabsf(v)));  // softplus
    const float *Bm = srow + a.R, *Cm = srow + a.R + a.N;
    float acc = 0.f;
    const float du = delta * xc;
    const float dl2 = -delta * kLog2e;
    if (NS == 16 && a.N == 16) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            float hh[4] = {h4[q4].x, h4[q4].y, h4[q4].z, h4[q4].w};
            const float aa[4] = {a4[q4].x, a4[q4].y, a4[q4].z, a4[q4].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int n = 4 * q4 + e;
                const float ab = ex2_approx(dl2 * __expf(aa[e]));  // exp(Delta A), A = -exp(A_log)
                hh[e] = fmaf(ab, hh[e], du * Bm[n]);
                acc = fmaf(hh[e], Cm[n], acc);
            }
            reinterpret_cast<float4 *>(hp)[q4] = make_float4(hh[0], hh[1], hh[2], hh[3]);
        }
    } else {
        for (int n = 0; n < a.N; ++n) {
            const float ab = ex2_approx(dl2 * __expf(al[n]));
            const float hn = fmaf(ab, hp[n], du * Bm[n]);
            hp[n] = hn;
            acc = fmaf(hn, Cm[n], acc);
        }
    }
    const float y = fmaf(a.D[c], xc, acc);
    a.g[static_cast<size_t>(m) * a.g_ld + c] = y * silu_exact(zv);
}

}  // namespace s6
