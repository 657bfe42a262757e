/*
 * s6_oracle.c -- float64 CPU oracle for the S6 selective scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header, table or constant with the CUDA
 * path.  It is deliberately plain: one channel at a time, one token at a time,
 * one state coordinate at a time, every step in double precision, in the order
 * the pages state the method.
 *
 * What it follows (page title, then section):
 *  - "mamba, live" (soundlark.studio), "what is actually running": the block's
 *    streaming form -- causal depthwise conv of width 4 + SiLU, dt = softplus(.),
 *    A = -exp(A_log), h <- exp(dt*A)*h + (dt*B)*xc, y = <h, C> + D*xc, output
 *    gated by SiLU(z).
 *  - "the s6 cell" (soundlark.studio), "the recurrence": the same three lines
 *    with the decay written as a power of two; Delta*A <= 0.
 *  - "Carry context through a selective state" (tensorviz.dev), "Recorded
 *    numerical example" and the model manifest's `steps` ("local", "select",
 *    "state", "read"): exact diagonal zero-order hold,
 *    B_bar = (exp(Delta*A) - 1) / A * B, the conv left-padded with zeros so it
 *    reads the current and the K-1 earlier tokens, C reading the UPDATED state,
 *    and D multiplying the conv output.
 *
 * Readings where the pages leave a step open:
 *  - softplus is log(1 + e^v) exactly (no large-v identity switch); written as
 *    max(v,0) + log1p(exp(-|v|)) so that it neither overflows nor cancels.
 *  - the conv has a bias (nullable by passing 0).
 *  - the scan starts from a zero state and a zero conv history unless a state
 *    is passed in (the streaming step and the resume case).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#define S6O_ABI_VERSION 1

int s6o_abi_version(void) { return S6O_ABI_VERSION; }

/* softplus(v) = log(1 + e^v) ("mamba, live": dt = softplus(dt_proj(.)) > 0). */
double s6o_softplus(double v)
{
    double m = v > 0.0 ? v : 0.0;
    return m + log1p(exp(-fabs(v)));
}

/* SiLU(v) = v * sigmoid(v) = v / (1 + e^-v). */
double s6o_silu(double v)
{
    if (v >= 0.0)
        return v / (1.0 + exp(-v));
    /* same value, written so e^-v cannot overflow for very negative v */
    double e = exp(v);
    return v * e / (1.0 + e);
}

/* A = -exp(A_log) < 0 ("mamba, live"; "the s6 cell", "the recurrence"). */
double s6o_A(double A_log) { return -exp(A_log); }

/* Decay factor A_bar = exp(Delta * A). */
double s6o_decay(double delta, double A_log) { return exp(delta * s6o_A(A_log)); }

/* Input term multiplying B*u.
 *  simplified (zoh = 0): Delta            ("mamba, live"; "the s6 cell")
 *  exact ZOH  (zoh = 1): (exp(Delta*A) - 1) / A   (the TinyMamba example,
 *              Mamba paper Eq. 4, as quoted on "Carry context ...").     */
double s6o_write_gain(double delta, double A_log, int zoh)
{
    if (!zoh)
        return delta;
    double A = s6o_A(A_log);
    return expm1(delta * A) / A;
}

/* h <- A_bar * h + write ("Decay the old state and add the current write"). */
double s6o_update(double h, double a_bar, double write) { return a_bar * h + write; }

/* Causal depthwise conv at one token:
 *   pre = bias + sum_{k<K-1} w[k] * hist[k] + w[K-1] * x_t
 * hist holds the K-1 previous pre-conv inputs, oldest first (zeros before the
 * first token).  Returns the pre-activation; the caller applies SiLU.        */
double s6o_conv_pre(int K, const double *w, double bias, const double *hist, double x_t)
{
    double acc = bias;
    for (int k = 0; k < K - 1; ++k)
        acc += w[k] * hist[k];
    acc += w[K - 1] * x_t;
    return acc;
}

/*
 * One channel over L tokens.
 *
 *   x       [L]     pre-conv input when K > 0, else the scan input u itself
 *   dt_raw  [L]     raw step size (before bias and softplus)
 *   z       [L]     gate input, or NULL for no gate
 *   Bm, Cm  [L*N]   per-token B_t and C_t rows of this channel's sequence
 *   A_log   [N]     this channel's A_log row
 *   D, dt_bias      this channel's skip weight and step-size bias
 *   K               conv width (0 = no conv: x is u)
 *   conv_w  [K]     taps, oldest first; conv_b the bias
 *   hist    [K-1]   in: conv history (oldest first), or NULL for zeros;
 *                   out (if hist_out != NULL): history after the last token
 *   h       [N]     in: initial state, or NULL for zeros
 *   y       [L]     out
 *   h_out   [N]     out (may be NULL)
 *   xc_out  [L]     out: the conv output u_t (may be NULL)
 *   delta_out [L]   out: Delta_t (may be NULL)
 */
void s6o_scan_channel(int64_t L, int N, int K, int zoh,
                      const double *x, const double *dt_raw, const double *z,
                      const double *Bm, const double *Cm,
                      const double *A_log, double D, double dt_bias,
                      const double *conv_w, double conv_b,
                      const double *hist_in, const double *h_in,
                      double *y, double *h_out, double *hist_out,
                      double *xc_out, double *delta_out)
{
    double hist[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    double h[64];
    for (int n = 0; n < N; ++n)
        h[n] = h_in ? h_in[n] : 0.0;
    if (K > 1 && hist_in)
        for (int k = 0; k < K - 1; ++k)
            hist[k] = hist_in[k];

    for (int64_t t = 0; t < L; ++t) {
        /* conv + SiLU ("Gather local context before the scan") */
        double u;
        if (K > 0) {
            double pre = s6o_conv_pre(K, conv_w, conv_b, hist, x[t]);
            for (int k = 0; k + 1 < K - 1; ++k)
                hist[k] = hist[k + 1];
            if (K > 1)
                hist[K - 2] = x[t];
            u = s6o_silu(pre);
        } else {
            u = x[t];
        }
        /* Delta ("Choose dynamics from the current input") */
        double delta = s6o_softplus(dt_raw[t] + dt_bias);
        if (xc_out)
            xc_out[t] = u;
        if (delta_out)
            delta_out[t] = delta;
        /* state update and readout ("Decay the old state ...", "Read, gate ...") */
        double acc = 0.0;
        for (int n = 0; n < N; ++n) {
            double a_bar = s6o_decay(delta, A_log[n]);
            double write = s6o_write_gain(delta, A_log[n], zoh) * Bm[t * N + n] * u;
            h[n] = s6o_update(h[n], a_bar, write);
            acc += h[n] * Cm[t * N + n];
        }
        double out = acc + D * u;
        if (z)
            out *= s6o_silu(z[t]);
        y[t] = out;
    }
    if (h_out)
        for (int n = 0; n < N; ++n)
            h_out[n] = h[n];
    if (hist_out && K > 1)
        for (int k = 0; k < K - 1; ++k)
            hist_out[k] = hist[k];
}

/*
 * Many independent channels in one call (no arithmetic beyond the loop above).
 * Channel c reads its sequences at x + c*L etc., its B/C rows at
 * Bm + bc_row[c]*L*N, its parameters at A_log + c*N, D[c], dt_bias[c],
 * conv_w + c*K, conv_b[c].  Optional per-channel state in/out follows the same
 * c-major layout.  NULL optional arrays mean "absent".
 */
void s6o_scan_channels(int64_t n_ch, int64_t L, int N, int K, int zoh,
                       const double *x, const double *dt_raw, const double *z,
                       const double *Bm, const double *Cm, const int64_t *bc_row,
                       const double *A_log, const double *D, const double *dt_bias,
                       const double *conv_w, const double *conv_b,
                       const double *hist_in, const double *h_in,
                       double *y, double *h_out, double *hist_out)
{
    int km1 = K > 1 ? K - 1 : 0;
    for (int64_t c = 0; c < n_ch; ++c) {
        s6o_scan_channel(L, N, K, zoh,
                         x + c * L, dt_raw + c * L, z ? z + c * L : NULL,
                         Bm + bc_row[c] * L * N, Cm + bc_row[c] * L * N,
                         A_log + c * N, D[c], dt_bias ? dt_bias[c] : 0.0,
                         K > 0 ? conv_w + c * K : NULL, (K > 0 && conv_b) ? conv_b[c] : 0.0,
                         hist_in ? hist_in + c * km1 : NULL, h_in ? h_in + c * N : NULL,
                         y + c * L, h_out ? h_out + c * N : NULL,
                         hist_out ? hist_out + c * km1 : NULL, NULL, NULL);
    }
}

/* Standalone conv + SiLU over many channels: xc[c*L + t]. */
void s6o_conv_silu_channels(int64_t n_ch, int64_t L, int K, const double *x,
                            const double *conv_w, const double *conv_b, double *xc)
{
    for (int64_t c = 0; c < n_ch; ++c) {
        double hist[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int64_t t = 0; t < L; ++t) {
            double pre = s6o_conv_pre(K, conv_w + c * K, conv_b ? conv_b[c] : 0.0, hist, x[c * L + t]);
            for (int k = 0; k + 1 < K - 1; ++k)
                hist[k] = hist[k + 1];
            if (K > 1)
                hist[K - 2] = x[c * L + t];
            xc[c * L + t] = s6o_silu(pre);
        }
    }
}

/* ------------------------------------------------------------ gradients
 * The backward pass of the scan (no conv: u given), for training through the
 * block ("Carry context through a selective state": the recurrence is what
 * makes training slow, since every timestep touches N states).  Reverse-mode
 * differentiation of exactly the forward steps above, for the loss
 * sum_t dy[t] * y[t]; no reading of the pages is needed beyond the forward.
 */

/* sigmoid(v) = 1 / (1 + e^-v), the derivative of softplus. */
double s6o_sigmoid(double v)
{
    if (v >= 0.0)
        return 1.0 / (1.0 + exp(-v));
    double e = exp(v);
    return e / (1.0 + e);
}

/* d SiLU(v) / dv = sigmoid(v) * (1 + v * (1 - sigmoid(v))). */
double s6o_dsilu(double v)
{
    double s = s6o_sigmoid(v);
    return s * (1.0 + v * (1.0 - s));
}

/*
 * One channel's gradients.  Inputs as s6o_scan_channel with K = 0, plus
 *   dy      [L]     gradient of the loss with respect to y
 *   hs      [(L+1)*N]  work: the states h_{-1} .. h_{L-1}
 * Outputs, written:     du[L], ddt[L] (with respect to dt_raw), dz[L] (if z)
 * Outputs, accumulated: dB[L*N], dC[L*N] (this channel's share of the
 *   sequence's rows), dA_log[N], dD[0], ddt_bias[0], dh_in[N] (if not NULL).
 */
void s6o_scan_bwd_channel(int64_t L, int N, int zoh,
                          const double *u, const double *dt_raw, const double *z,
                          const double *Bm, const double *Cm,
                          const double *A_log, double D, double dt_bias,
                          const double *h_in, const double *dy,
                          double *du, double *ddt, double *dz,
                          double *dB, double *dC, double *dA_log, double *dD, double *ddt_bias,
                          double *dh_in, double *hs)
{
    /* forward, keeping every state: hs[(t+1)*N + n] = h_t[n] */
    for (int n = 0; n < N; ++n)
        hs[n] = h_in ? h_in[n] : 0.0;
    for (int64_t t = 0; t < L; ++t) {
        double delta = s6o_softplus(dt_raw[t] + dt_bias);
        for (int n = 0; n < N; ++n) {
            double a_bar = s6o_decay(delta, A_log[n]);
            double write = s6o_write_gain(delta, A_log[n], zoh) * Bm[t * N + n] * u[t];
            hs[(t + 1) * N + n] = s6o_update(hs[t * N + n], a_bar, write);
        }
    }

    /* reverse: g[n] = dLoss/dh_t[n] arriving from tokens after t */
    double g[64];
    for (int n = 0; n < N; ++n)
        g[n] = 0.0;
    for (int64_t t = L - 1; t >= 0; --t) {
        const double *h_t = hs + (t + 1) * N;
        const double *h_prev = hs + t * N;
        double v = dt_raw[t] + dt_bias;
        double delta = s6o_softplus(v);
        double s = D * u[t];
        for (int n = 0; n < N; ++n)
            s += h_t[n] * Cm[t * N + n];
        double gate = z ? s6o_silu(z[t]) : 1.0;
        double ds = dy[t] * gate;  /* d/ds of y = s * gate */
        if (z)
            dz[t] = dy[t] * s * s6o_dsilu(z[t]);
        *dD += ds * u[t];
        double dut = ds * D;
        double ddelta = 0.0;
        for (int n = 0; n < N; ++n) {
            double A = s6o_A(A_log[n]);
            double a_bar = s6o_decay(delta, A_log[n]);
            double gain = s6o_write_gain(delta, A_log[n], zoh);
            double b = Bm[t * N + n];
            dC[t * N + n] += ds * h_t[n];
            double dh = ds * Cm[t * N + n] + g[n];  /* total dLoss/dh_t[n] */
            /* h_t = a_bar h_{t-1} + gain * b * u */
            double da = dh * h_prev[n];
            double dgain = dh * b * u[t];
            dB[t * N + n] += dh * gain * u[t];
            dut += dh * gain * b;
            /* a_bar = exp(delta * A) */
            ddelta += da * a_bar * A;
            double dA = da * a_bar * delta;
            if (zoh) {
                /* gain = expm1(delta A) / A */
                ddelta += dgain * a_bar;
                dA += dgain * (delta * a_bar * A - expm1(delta * A)) / (A * A);
            } else {
                /* gain = delta */
                ddelta += dgain;
            }
            dA_log[n] += dA * A; /* A = -exp(A_log): dA/dA_log = A */
            g[n] = dh * a_bar;   /* to h_{t-1} */
        }
        du[t] = dut;
        double dv = ddelta * s6o_sigmoid(v);  /* softplus'(v) = sigmoid(v) */
        ddt[t] = dv;
        *ddt_bias += dv;
    }
    if (dh_in)
        for (int n = 0; n < N; ++n)
            dh_in[n] += g[n];
}

/*
 * Many channels: channel c reads u + c*L etc. and its B/C rows at
 * Bm + bc_row[c]*L*N; it accumulates into dB/dC at dBm + c*L*N (one private
 * block per channel; the caller sums the channels of a sequence), its
 * parameter gradients at dA_log + c*N, dD[c], ddt_bias[c], dh_in + c*N.
 */
void s6o_scan_bwd_channels(int64_t n_ch, int64_t L, int N, int zoh,
                           const double *u, const double *dt_raw, const double *z,
                           const double *Bm, const double *Cm, const int64_t *bc_row,
                           const double *A_log, const double *D, const double *dt_bias,
                           const double *h_in, const double *dy,
                           double *du, double *ddt, double *dz, double *dBm, double *dCm,
                           double *dA_log, double *dD, double *ddt_bias, double *dh_in, double *work)
{
    for (int64_t c = 0; c < n_ch; ++c) {
        s6o_scan_bwd_channel(L, N, zoh, u + c * L, dt_raw + c * L, z ? z + c * L : NULL,
                             Bm + bc_row[c] * L * N, Cm + bc_row[c] * L * N,
                             A_log + c * N, D[c], dt_bias ? dt_bias[c] : 0.0,
                             h_in ? h_in + c * N : NULL, dy + c * L,
                             du + c * L, ddt + c * L, z ? dz + c * L : NULL,
                             dBm + c * L * N, dCm + c * L * N, dA_log + c * N, dD + c,
                             ddt_bias + c, dh_in ? dh_in + c * N : NULL, work);
    }
}

/*
 * Backward of the causal conv + SiLU in front of the scan, one channel at a
 * time: given dxc[t] (the gradient with respect to the conv output u_t, e.g.
 * du of s6o_scan_bwd_channels), pre_t = bias + sum_k w[k] x[t-K+1+k] with
 * zero left padding, u_t = SiLU(pre_t):
 *   dpre_t = dxc[t] * SiLU'(pre_t);  dx[t-K+1+k] += w[k] dpre_t (in range);
 *   dw[k] += dpre_t x[t-K+1+k];  db += dpre_t.
 * dx is written; dw (K values per channel) and db are accumulated.
 */
void s6o_conv_silu_bwd_channels(int64_t n_ch, int64_t L, int K, const double *x,
                                const double *conv_w, const double *conv_b, const double *dxc,
                                double *dx, double *dw, double *db)
{
    for (int64_t c = 0; c < n_ch; ++c) {
        const double *xc = x + c * L;
        const double *w = conv_w + c * K;
        double *dxo = dx + c * L;
        for (int64_t t = 0; t < L; ++t)
            dxo[t] = 0.0;
        double hist[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int64_t t = 0; t < L; ++t) {
            double pre = s6o_conv_pre(K, w, conv_b ? conv_b[c] : 0.0, hist, xc[t]);
            double dpre = dxc[c * L + t] * s6o_dsilu(pre);
            for (int k = 0; k < K; ++k) {
                int64_t src = t - (K - 1) + k;
                if (src >= 0) {
                    dxo[src] += w[k] * dpre;
                    dw[c * K + k] += dpre * xc[src];
                }
            }
            db[c] += dpre;
            for (int k = 0; k + 1 < K - 1; ++k)
                hist[k] = hist[k + 1];
            if (K > 1)
                hist[K - 2] = xc[t];
        }
    }
}

/* Streaming state size of a block stack: channels x states x blocks
 * ("mamba, live": 1,536 x 16 x 6 = 147,456; the TinyMamba example: 8 x 3 = 24). */
int64_t s6o_ssm_state_values(int64_t d_inner, int64_t d_state, int64_t blocks)
{
    return d_inner * d_state * blocks;
}

/* Conv history values: K-1 past inputs per channel (TinyMamba: 8 x 2 = 16). */
int64_t s6o_conv_history_values(int64_t d_inner, int64_t K, int64_t blocks)
{
    return d_inner * (K - 1) * blocks;
}

/* ------------------------------------------------ constant-decay recurrence
 * The diagonal recurrence cell of "the s6 cell", sections "one cell, two
 * architectures" and "the difference that no engineering removes": the same
 * line h <- a*h + b*u with a = 2^(negative), but the decay taken from a
 * constant instead of computed per token.  With state width N per channel:
 *   a[n] = 2^w[n]  (w[n] <= 0, a per-channel constant, precomputed once)
 *   h[n] <- a[n] * h[n] + B_t[n] * u_t          (no step size: b = B_t)
 *   y_t  = (<h, C_t> + D * u_t) * SiLU(z_t)     (the S6 cell's readout; z optional)
 * RWKV's normaliser branch is not part of this cell (the pages give it no
 * formula).
 */
void s6o_diag_const_channel(int64_t L, int N, const double *u, const double *z,
                            const double *Bm, const double *Cm, const double *log2_decay,
                            double D, const double *h_in, double *y, double *h_out)
{
    double h[64], a[64];
    for (int n = 0; n < N; ++n) {
        h[n] = h_in ? h_in[n] : 0.0;
        a[n] = exp2(log2_decay[n]);
    }
    for (int64_t t = 0; t < L; ++t) {
        double acc = 0.0;
        for (int n = 0; n < N; ++n) {
            h[n] = s6o_update(h[n], a[n], Bm[t * N + n] * u[t]);
            acc += h[n] * Cm[t * N + n];
        }
        double out = acc + D * u[t];
        if (z)
            out *= s6o_silu(z[t]);
        y[t] = out;
    }
    if (h_out)
        for (int n = 0; n < N; ++n)
            h_out[n] = h[n];
}

/* Many channels, laid out as in s6o_scan_channels (log2_decay + c*N). */
void s6o_diag_const_channels(int64_t n_ch, int64_t L, int N, const double *u, const double *z,
                             const double *Bm, const double *Cm, const int64_t *bc_row,
                             const double *log2_decay, const double *D, const double *h_in,
                             double *y, double *h_out)
{
    for (int64_t c = 0; c < n_ch; ++c)
        s6o_diag_const_channel(L, N, u + c * L, z ? z + c * L : NULL, Bm + bc_row[c] * L * N,
                               Cm + bc_row[c] * L * N, log2_decay + c * N, D[c],
                               h_in ? h_in + c * N : NULL, y + c * L, h_out ? h_out + c * N : NULL);
}

/* ------------------------------------------------------ the decode block
 * One Mamba-mini block for one token of one sequence, in the streaming form of
 * "mamba, live", section "what is actually running" (the per-block listing),
 * with the weights stored as that page's "Weights" paragraph says: per-row
 * symmetric int8, w = int8_row x scale_row, A_log kept in float32.
 *
 *   hn      = LayerNorm(x)                          (biased variance, eps, affine)
 *   [xin,z] = in_proj(hn)                           dm -> 2 di  (rows 0..di-1: xin)
 *   xc      = SiLU(conv_K(xin))                     with the (K-1)-token history
 *   [dt,B,C]= x_proj(xc)                            di -> R + N + N
 *   Delta   = softplus(dt_proj(dt) + dt_bias)       R -> di
 *   h       = exp(Delta A) h + (Delta B) xc,  A = -exp(A_log)
 *   y       = <h, C> + D xc
 *   x      += out_proj(y SiLU(z))                   di -> dm
 *
 * Readings: in_proj, x_proj and out_proj carry no bias (the TinyMamba
 * manifest's Linears say bias false); dt_proj's bias is dt_bias; LayerNorm is
 * PyTorch's (weight and bias, biased variance).
 */

/* LayerNorm of one row: (x - mean) / sqrt(var + eps) * w + b. */
void s6o_layernorm(int n, const double *x, const double *w, const double *b, double eps, double *out)
{
    double mean = 0.0;
    for (int i = 0; i < n; ++i)
        mean += x[i];
    mean /= n;
    double var = 0.0;
    for (int i = 0; i < n; ++i)
        var += (x[i] - mean) * (x[i] - mean);
    var /= n;
    double r = 1.0 / sqrt(var + eps);
    for (int i = 0; i < n; ++i)
        out[i] = (x[i] - mean) * r * w[i] + b[i];
}

/* y[o] = scale[o] * sum_i q[o][i] x[i]: a Linear with per-row int8 weights. */
void s6o_linear_q8(int n_out, int n_in, const int8_t *q, const double *scale, const double *x, double *y)
{
    for (int o = 0; o < n_out; ++o) {
        double acc = 0.0;
        for (int i = 0; i < n_in; ++i)
            acc += (double)q[(int64_t)o * n_in + i] * x[i];
        y[o] = scale[o] * acc;
    }
}

/* The block's weights (all row-major, [out][in]). */
typedef struct {
    int dm, di, N, R, K;
    double eps;
    const double *ln_w, *ln_b;             /* [dm] */
    const int8_t *in_q;                    /* [2 di][dm] */
    const double *in_s;                    /* [2 di] */
    const double *conv_w, *conv_b;         /* [di][K], [di] */
    const int8_t *xp_q;                    /* [R + 2N][di] */
    const double *xp_s;                    /* [R + 2N] */
    const int8_t *dt_q;                    /* [di][R] */
    const double *dt_s, *dt_bias;          /* [di], [di] */
    const double *A_log, *D;               /* [di][N], [di] */
    const int8_t *out_q;                   /* [dm][di] */
    const double *out_s;                   /* [dm] */
} s6o_block;

/* One token through one block.  x [dm] is updated in place (the residual
 * stream); conv_state [di][K-1] (oldest first) and h [di][N] too.  work holds
 * 6 di + dm + R + 2N doubles. */
void s6o_block_step(const s6o_block *p, double *x, double *conv_state, double *h, double *work)
{
    int dm = p->dm, di = p->di, N = p->N, R = p->R, K = p->K;
    double *hn = work;                 /* dm */
    double *xz = hn + dm;              /* 2 di */
    double *xc = xz + 2 * di;          /* di */
    double *dbc = xc + di;             /* R + 2N */
    double *dtr = dbc + R + 2 * N;     /* di */
    double *g = dtr + di;              /* di */
    s6o_layernorm(dm, x, p->ln_w, p->ln_b, p->eps, hn);
    s6o_linear_q8(2 * di, dm, p->in_q, p->in_s, hn, xz);
    for (int c = 0; c < di; ++c) {
        double *hist = conv_state + (int64_t)c * (K - 1);
        double pre = s6o_conv_pre(K, p->conv_w + (int64_t)c * K, p->conv_b ? p->conv_b[c] : 0.0, hist, xz[c]);
        for (int k = 0; k + 1 < K - 1; ++k)
            hist[k] = hist[k + 1];
        if (K > 1)
            hist[K - 2] = xz[c];
        xc[c] = s6o_silu(pre);
    }
    s6o_linear_q8(R + 2 * N, di, p->xp_q, p->xp_s, xc, dbc);
    s6o_linear_q8(di, R, p->dt_q, p->dt_s, dbc, dtr);
    const double *Bt = dbc + R, *Ct = dbc + R + N;
    for (int c = 0; c < di; ++c) {
        double delta = s6o_softplus(dtr[c] + p->dt_bias[c]);
        double acc = 0.0;
        for (int n = 0; n < N; ++n) {
            double a_bar = s6o_decay(delta, p->A_log[(int64_t)c * N + n]);
            double *hc = h + (int64_t)c * N + n;
            *hc = s6o_update(*hc, a_bar, delta * Bt[n] * xc[c]);
            acc += *hc * Ct[n];
        }
        double yv = acc + p->D[c] * xc[c];
        g[c] = yv * s6o_silu(xz[di + c]);
    }
    double *o = hn; /* reuse: dm outputs */
    s6o_linear_q8(dm, di, p->out_q, p->out_s, g, o);
    for (int i = 0; i < dm; ++i)
        x[i] += o[i];
}

/* The block for n_seq independent sequences (x, conv_state, h per sequence). */
void s6o_block_step_seqs(int64_t n_seq, int dm, int di, int N, int R, int K, double eps,
                         const double *ln_w, const double *ln_b, const int8_t *in_q, const double *in_s,
                         const double *conv_w, const double *conv_b, const int8_t *xp_q, const double *xp_s,
                         const int8_t *dt_q, const double *dt_s, const double *dt_bias, const double *A_log,
                         const double *D, const int8_t *out_q, const double *out_s,
                         double *x, double *conv_state, double *h, double *work)
{
    s6o_block p = {dm, di, N, R, K, eps, ln_w, ln_b, in_q, in_s, conv_w, conv_b, xp_q, xp_s,
                   dt_q, dt_s, dt_bias, A_log, D, out_q, out_s};
    for (int64_t s = 0; s < n_seq; ++s)
        s6o_block_step(&p, x + s * dm, conv_state + s * (int64_t)di * (K - 1), h + s * (int64_t)di * N, work);
}
