/*
 * s6.h -- C ABI of the B200 (sm_100a) selective-scan library (libs6_b200.so).
 *
 * The library computes the S6 selective state-space recurrence of Mamba, as the
 * pages state it:
 *   "mamba, live" (soundlark.studio), section "what is actually running":
 *       xc = SiLU(depthwise_conv4(x))          4-tap causal, per channel
 *       dt = softplus(dt_raw + dt_bias) > 0    per inner channel
 *       A  = -exp(A_log) < 0                    d_inner x N
 *       h  = exp(dt*A) * h + (dt*B) * xc        the recurrence
 *       y  = <h, C> + D*xc,  output y * SiLU(z)
 *   "the s6 cell" (soundlark.studio), section "the recurrence": the decay is
 *       the power of two 2^(dt*A*log2 e), with dt*A <= 0.
 *   "Carry context through a selective state" (tensorviz.dev), "Recorded
 *       numerical example" and the manifest's steps "state"/"read": the exact
 *       zero-order hold B_bar = (exp(dt*A) - 1)/A * B, and C reading the
 *       UPDATED state.
 * Entry points: the full-sequence scans (plain, fused with the conv, without
 * allocation, or from a given state), the standalone conv, the single-token
 * streaming step, and the gradients of the scans (reverse-mode
 * differentiation of the same steps).
 *
 * Conventions shared by every call
 * --------------------------------
 *  Sizes: Bt = batch, L = seqlen, d = d_inner, N = d_state (1..16),
 *         K = conv_width (2..4 where a conv is applied).
 *  Layouts (row-major, C order, no padding between rows):
 *     sequence tensors  x, u, dt, z, y : [Bt, L, d]   (channels contiguous)
 *     per-token rows    B, C           : [Bt, L, N]
 *     A_log                            : [d, N]   float32
 *     D, dt_bias, conv_b               : [d]      float32
 *     conv_w                           : [d, K]   float32, oldest tap first
 *     h_final, h_ssm                   : [Bt, d, N] float32
 *     conv_state                       : [Bt, d, K-1] in the I/O dtype,
 *                                        oldest input first
 *  I/O dtype (dims.io_dtype) applies to x/u, dt, z, B, C, y and conv_state:
 *     S6_F32 (float) or S6_BF16 (bfloat16).  All arithmetic and all states are
 *     float32 on the device.
 *  Pointers: DEVICE pointers owned by the caller; the library keeps none of
 *     them after the call returns.  Outputs must not alias inputs.
 *  Alignment: for the full-sequence calls, x/u, dt, z, y (and out) must be
 *     16-byte aligned and d * sizeof(io) a multiple of 16 bytes (d % 4 == 0
 *     for float32, d % 8 == 0 for bfloat16): their rows are moved by the
 *     tensor-memory accelerator or in 16-byte vectors.  For s6_step, h_ssm and
 *     A_log must be 16-byte aligned when N is 4, 8 or 16.  Every other
 *     pointer must be aligned to its element size.  Violations return
 *     S6_ERR_ALIGNMENT.
 *  Streams: every call is asynchronous on `stream` (NULL = legacy default
 *     stream) and returns once the work is enqueued.
 *  Errors: arguments are checked on the host before anything is enqueued;
 *     a failed check returns a negative s6_status and enqueues nothing.  A
 *     launch failure returns S6_ERR_CUDA.  No call aborts, traps or prints.
 *  Start state: a full-sequence call starts from h = 0 and a zero conv
 *     history (the conv is left-padded with zeros); the _from_state calls
 *     take both as arguments.
 *  Scratch: s6_scan_fwd, s6_conv_scan_fwd and their _from_state forms may
 *     use a library-owned device
 *     buffer for carries between thread blocks (allocated with cudaMalloc on
 *     the first call on a device that needs it, grown on demand, kept until
 *     process exit).  Make that first call before capturing a stream.  Calls
 *     that share a device must not run concurrently on different streams.
 */
#ifndef S6_B200_H
#define S6_B200_H

#include <stdint.h>

#if defined(__GNUC__)
#define S6_API __attribute__((visibility("default")))
#else
#define S6_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream; declared here so that callers need
 * no CUDA header. */
typedef struct CUstream_st *s6_stream_t;

typedef enum { S6_F32 = 0, S6_BF16 = 1 } s6_dtype;

typedef struct {
    int64_t batch;      /* Bt >= 0 (0: nothing to do)                          */
    int64_t seqlen;     /* L  >= 0 (0: nothing to scan); ignored by s6_step    */
    int64_t d_inner;    /* d  >= 1                                             */
    int64_t d_state;    /* N  in [1, 16]                                       */
    int64_t conv_width; /* K  in [2, 4] for calls that apply the conv          */
    int32_t io_dtype;   /* s6_dtype                                            */
} s6_dims;

typedef enum {
    S6_OK = 0,
    S6_ERR_INVALID_ARG = -1, /* null pointer, negative or inconsistent size     */
    S6_ERR_UNSUPPORTED = -2, /* N > 16, K outside [2,4], unknown dtype          */
    S6_ERR_ALIGNMENT = -3,   /* pointer or row not 16-byte aligned              */
    S6_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed            */
    S6_ERR_TIMEOUT = -5,     /* a bounded device-side wait gave up              */
    S6_ERR_SCRATCH_LIMIT = -6 /* fixed scratch too small (s6_conv_scan_fwd_noalloc) */
} s6_status;

/*
 * s6_scan_fwd -- full-sequence selective scan, u already convolved.
 * ("mamba, live": the three lines h = ..., y = ..., y * SiLU(z).)
 *
 *  u        [Bt,L,d] io   scan input (the conv + SiLU output xc)
 *  dt       [Bt,L,d] io   raw step size; Delta = softplus(dt + dt_bias)
 *  A_log    [d,N]    f32  A = -exp(A_log)
 *  B, C     [Bt,L,N] io   per-token input and readout vectors
 *  D        [d]      f32  skip weight, y += D * u
 *  z        [Bt,L,d] io   gate input, y *= SiLU(z); NULL = no gate
 *  dt_bias  [d]      f32  NULL = zeros
 *  zoh_mode int           0: write (Delta*B)*u (the streaming page's form);
 *                         1: exact ZOH write (exp(Delta*A)-1)/A * B * u
 *  y        [Bt,L,d] io   output (written)
 *  h_final  [Bt,d,N] f32  state after token L-1 (written); NULL = not wanted
 */
S6_API int s6_scan_fwd(const s6_dims *dims, const void *u, const void *dt, const float *A_log,
                const void *B, const void *C, const float *D, const void *z,
                const float *dt_bias, int zoh_mode, void *y, float *h_final,
                s6_stream_t stream);

/*
 * s6_conv_scan_fwd -- the fused block path: causal depthwise conv of width K
 * + SiLU on x, then the selective scan of s6_scan_fwd on the result, which
 * never leaves the chip.  ("mamba, live": xc = SiLU(depthwise_conv4(xin)) and
 * the recurrence; "Carry context ...", step "local": the conv is left-padded
 * and reads the current and K-1 earlier inputs.)
 *
 *  x        [Bt,L,d] io   pre-conv input
 *  conv_w   [d,K]    f32  taps, oldest first: pre_t = conv_b + sum_k w[k] x[t-K+1+k]
 *  conv_b   [d]      f32  NULL = zeros
 *  the rest as s6_scan_fwd, with u := SiLU(pre) kept in float32 (not rounded
 *  to the I/O dtype), so the result equals causal_conv1d_silu_fwd followed by
 *  s6_scan_fwd only up to that rounding.
 */
S6_API int s6_conv_scan_fwd(const s6_dims *dims, const void *x, const float *conv_w, const float *conv_b,
                     const void *dt, const float *A_log, const void *B, const void *C,
                     const float *D, const void *z, const float *dt_bias, int zoh_mode,
                     void *y, float *h_final, s6_stream_t stream);

/*
 * s6_conv_scan_fwd_noalloc -- s6_conv_scan_fwd for callers that must not
 * allocate device memory.  The pages have no counterpart: this is a deployment
 * variant of the same computation, not a step of the method.
 *
 * Who needs it: a caller whose device memory is entirely owned by its own
 * allocator (a framework's caching pool that has reserved the GPU), or a
 * latency-critical process with a fixed memory plan, cannot let a library call
 * cudaMalloc on its behalf -- the allocation may fail, block, or synchronise
 * the device.  s6_conv_scan_fwd may allocate (its carry scratch, on first use
 * and when a larger problem arrives); this entry point never does.
 *
 * Same arguments, layouts and results as s6_conv_scan_fwd.  When the schedule
 * splits sequences into segments it keeps the segment carries in one fixed
 * 4 MiB array compiled into the library (every GPU that loads the library holds
 * it until the process exits), instead of allocated memory.  The carries need
 * about 4 KiB per (sequence, 64-channel tile) at N = 16; a problem that would
 * need more than the array holds returns S6_ERR_SCRATCH_LIMIT and enqueues
 * nothing.  Problems with enough (sequence, tile) pairs to be scheduled without
 * segments use no scratch at all.
 *
 * The first call on a device looks up the array's device address (once per
 * device); make that first call before capturing a stream.  The array is
 * shared by every call on the device and keeps the last call's contents; the
 * call clears on its stream what must start at zero.  Calls whose executions
 * overlap on the GPU (different streams, or different host threads) race on
 * the array and must be serialised by the caller.
 */
S6_API int s6_conv_scan_fwd_noalloc(const s6_dims *dims, const void *x, const float *conv_w,
                                    const float *conv_b, const void *dt, const float *A_log,
                                    const void *B, const void *C, const float *D, const void *z,
                                    const float *dt_bias, int zoh_mode, void *y, float *h_final,
                                    s6_stream_t stream);

/*
 * s6_scan_fwd_from_state, s6_conv_scan_fwd_from_state -- s6_scan_fwd and
 * s6_conv_scan_fwd continued from a given state instead of zeros: the chunked
 * form of a prefill, and the bridge between the scan and s6_step.  The state
 * is what the streaming page carries between tokens ("mamba, live": the
 * model's memory is h_ssm plus a (K-1)-token conv history per channel;
 * "Carry context through a selective state", token streaming matching the full
 * forward): scanning tokens [0, L1) and then [L1, L) from (h_final, the last
 * K-1 inputs) equals one scan over [0, L).
 *
 *  h_init    [Bt,d,N]   f32  state before token 0; NULL = zeros
 *  conv_hist [Bt,d,K-1] io   the K-1 inputs before token 0, oldest first (the
 *                            layout of conv_state); NULL = zeros.  Fused form
 *                            only.
 *  the rest as s6_scan_fwd / s6_conv_scan_fwd.  h_init and conv_hist need
 *  only element alignment and must not alias outputs.  With L = 0, h_final
 *  receives h_init.
 */
S6_API int s6_scan_fwd_from_state(const s6_dims *dims, const void *u, const void *dt, const float *A_log,
                                  const void *B, const void *C, const float *D, const void *z,
                                  const float *dt_bias, int zoh_mode, const float *h_init, void *y,
                                  float *h_final, s6_stream_t stream);
S6_API int s6_conv_scan_fwd_from_state(const s6_dims *dims, const void *x, const float *conv_w,
                                       const float *conv_b, const void *dt, const float *A_log,
                                       const void *B, const void *C, const float *D, const void *z,
                                       const float *dt_bias, int zoh_mode, const float *h_init,
                                       const void *conv_hist, void *y, float *h_final,
                                       s6_stream_t stream);

/*
 * s6_diag_recurrence_fwd -- the diagonal recurrence cell with the decay source
 * as a parameter ("the s6 cell", sections "one cell, two architectures" and
 * "the difference that no engineering removes"): both recurrences reduce to
 * h <- a*h + b*u with a = 2^(negative); the decay is either computed per token
 * from the input (live, the selective scan) or a per-channel constant that is
 * precomputed once (no exponential per token).  State width N = d_state.
 *
 *  decay_source  S6_DECAY_LIVE:  a = 2^(Delta*A*log2 e), Delta = softplus(dt +
 *                                dt_bias), A = -exp(A_log), b = Delta*B_t --
 *                                exactly s6_scan_fwd_from_state with
 *                                zoh_mode = 0 (dt, A_log required; log2_decay
 *                                ignored)
 *                S6_DECAY_CONST: a[d,n] = 2^log2_decay[d,n] (log2_decay <= 0
 *                                for a decay in (0, 1]), b = B_t: per state n,
 *                                h[n] <- a[n] h[n] + B_t[n] u_t
 *                                (dt, A_log and dt_bias ignored, may be NULL)
 *  u        [Bt,L,d] io   input
 *  log2_decay [d,N]  f32  log2 of the constant decays (S6_DECAY_CONST)
 *  B, C     [Bt,L,N] io   per-token write and readout vectors
 *  D        [d]      f32  y = (<h, C_t> + D*u) * SiLU(z)
 *  z        [Bt,L,d] io   NULL = no gate
 *  h_init   [Bt,d,N] f32  start state, NULL = zeros
 *  y, h_final              as s6_scan_fwd
 * RWKV's normaliser branch (the page's other difference) is not part of this
 * cell: the pages give it no formula.  Alignment and scratch as s6_scan_fwd;
 * an unknown decay_source returns S6_ERR_INVALID_ARG.
 */
#define S6_DECAY_LIVE 0
#define S6_DECAY_CONST 1
S6_API int s6_diag_recurrence_fwd(const s6_dims *dims, int decay_source, const void *u, const void *dt,
                                  const float *A_log, const float *dt_bias, const float *log2_decay,
                                  const void *B, const void *C, const float *D, const void *z,
                                  const float *h_init, void *y, float *h_final, s6_stream_t stream);

/*
 * s6_scan_bwd -- gradients of s6_scan_fwd (no conv: u given) for the loss
 * sum(dy * y): reverse-mode differentiation of the same steps (the recurrence
 * the pages single out as what makes training slow, "Carry context through a
 * selective state"; "mamba, live" for the forward).  Inputs as
 * s6_scan_fwd_from_state, plus
 *
 *  dy        [Bt,L,d] io   gradient with respect to y
 *  h_init    [Bt,d,N] f32  start state of the forward, NULL = zeros
 * Written (float32):
 *  du, ddt   [Bt,L,d]      with respect to u and the raw dt
 *  dz        [Bt,L,d]      with respect to z (required when z is given)
 *  dB, dC    [Bt,L,N]      summed over the d channels of each sequence
 *  dA_log    [d,N], dD [d], ddt_bias [d] (NULL = not wanted)
 *                          summed over the sequences and tokens
 *  dh_init   [Bt,d,N]      with respect to h_init (NULL = not wanted)
 * dB, dC, dA_log, dD and ddt_bias are zeroed by the call, then accumulated
 * with atomics, so their last bits depend on the order of the additions.  The
 * call uses the library-owned scratch buffer.  At N = 16 with 16-byte aligned
 * u, dt, z, dy, B, C and d * sizeof(io) a multiple of 16 (the pipelined
 * backward) it holds the state before every 16th token (ceil(L/16) * Bt * d *
 * 16 floats) and per-tile dB / dC rows (ceil(d/64) * Bt * L * 32 floats);
 * otherwise the state every 64 tokens plus one chunk of states ((ceil(L/64) +
 * 64) * Bt * d * N floats).  Pointers need only element alignment.
 */
S6_API int s6_scan_bwd(const s6_dims *dims, const void *u, const void *dt, const float *A_log,
                       const void *B, const void *C, const float *D, const void *z,
                       const float *dt_bias, int zoh_mode, const float *h_init, const void *dy,
                       float *du, float *ddt, float *dz, float *dB, float *dC, float *dA_log,
                       float *dD, float *ddt_bias, float *dh_init, s6_stream_t stream);

/*
 * s6_conv_scan_bwd -- gradients of the fused path (s6_conv_scan_fwd_from_state
 * with a zero conv history) for the loss sum(dy * y): the scan's gradients as
 * in s6_scan_bwd, carried through SiLU and the causal conv.  In addition to
 * s6_scan_bwd's arguments (with x, the pre-conv input, in place of u):
 *
 *  conv_w  [d,K] f32, conv_b [d] f32 (NULL = zeros)   as in the forward
 *  dx      [Bt,L,d]  f32  with respect to x (written; replaces du)
 *  dconv_w [d,K]     f32  with respect to conv_w (zeroed, then accumulated)
 *  dconv_b [d]       f32  with respect to conv_b (NULL = not wanted)
 */
S6_API int s6_conv_scan_bwd(const s6_dims *dims, const void *x, const float *conv_w,
                            const float *conv_b, const void *dt, const float *A_log,
                            const void *B, const void *C, const float *D, const void *z,
                            const float *dt_bias, int zoh_mode, const float *h_init,
                            const void *dy, float *dx, float *dconv_w, float *dconv_b,
                            float *ddt, float *dz, float *dB, float *dC, float *dA_log,
                            float *dD, float *ddt_bias, float *dh_init, s6_stream_t stream);

/*
 * s6_scan_fwd_ckpt, s6_conv_scan_fwd_ckpt -- the forward of a training step:
 * s6_scan_fwd_from_state / s6_conv_scan_fwd (zero conv history) that also
 * keeps what the backward would otherwise recompute, so that the backward
 * does not run the forward again ("Carry context through a selective state":
 * the recurrence is what makes training slow).  Arguments as those calls
 * (h_init [Bt,d,N] f32, NULL = zeros), plus
 *
 *  ckpt  [Bt][ceil(L/16)][d][16] f32  written: ckpt[b][k] is the state before
 *        token 16 k (h_init, or zeros, at k = 0); 16-byte aligned
 *
 * N = 16 only (S6_ERR_UNSUPPORTED otherwise).  The SiLUs are evaluated as the
 * backward evaluates them (the exponential form), so with bfloat16 I/O y may
 * differ from s6_conv_scan_fwd's in its last bit.  The checkpoints stay valid
 * for the inputs they were computed from.
 */
S6_API int s6_scan_fwd_ckpt(const s6_dims *dims, const void *u, const void *dt, const float *A_log,
                            const void *B, const void *C, const float *D, const void *z,
                            const float *dt_bias, int zoh_mode, const float *h_init, void *y,
                            float *h_final, float *ckpt, s6_stream_t stream);
S6_API int s6_conv_scan_fwd_ckpt(const s6_dims *dims, const void *x, const float *conv_w,
                                 const float *conv_b, const void *dt, const float *A_log,
                                 const void *B, const void *C, const float *D, const void *z,
                                 const float *dt_bias, int zoh_mode, const float *h_init, void *y,
                                 float *h_final, float *ckpt, s6_stream_t stream);

/*
 * s6_scan_bwd_ckpt, s6_conv_scan_bwd_ckpt -- s6_scan_bwd / s6_conv_scan_bwd
 * given the checkpoints that the matching _ckpt forward wrote for the same
 * inputs: the arguments of those calls with ckpt (read only) in place of
 * h_init, which the checkpoints already hold.  Only the pipelined backward
 * takes checkpoints: N = 16 (S6_ERR_UNSUPPORTED otherwise), and u / x, dt, z,
 * dy, B, C and ckpt 16-byte aligned with d * sizeof(io) a multiple of 16
 * (S6_ERR_ALIGNMENT otherwise).  The scratch holds only the dB / dC rows.
 */
S6_API int s6_scan_bwd_ckpt(const s6_dims *dims, const void *u, const void *dt, const float *A_log,
                            const void *B, const void *C, const float *D, const void *z,
                            const float *dt_bias, int zoh_mode, const float *ckpt, const void *dy,
                            float *du, float *ddt, float *dz, float *dB, float *dC, float *dA_log,
                            float *dD, float *ddt_bias, float *dh_init, s6_stream_t stream);
S6_API int s6_conv_scan_bwd_ckpt(const s6_dims *dims, const void *x, const float *conv_w,
                                 const float *conv_b, const void *dt, const float *A_log,
                                 const void *B, const void *C, const float *D, const void *z,
                                 const float *dt_bias, int zoh_mode, const float *ckpt,
                                 const void *dy, float *dx, float *dconv_w, float *dconv_b,
                                 float *ddt, float *dz, float *dB, float *dC, float *dA_log,
                                 float *dD, float *ddt_bias, float *dh_init, s6_stream_t stream);

/*
 * causal_conv1d_silu_fwd -- the conv + SiLU alone ("mamba, live":
 * depthwise_conv4 then SiLU; "Carry context ...", step "local").
 *
 *  x        [Bt,L,d] io   input
 *  conv_w   [d,K]    f32  taps, oldest first
 *  conv_b   [d]      f32  NULL = zeros
 *  out      [Bt,L,d] io   SiLU(conv_b + sum_k w[k] x[t-K+1+k]), x[<0] = 0
 */
S6_API int causal_conv1d_silu_fwd(const s6_dims *dims, const void *x, const float *conv_w,
                           const float *conv_b, void *out, s6_stream_t stream);

/*
 * s6_step -- one streaming token for Bt independent sequences, state updated
 * in place ("mamba, live": one token in, one token out, constant work; the
 * model's memory is h_ssm plus a (K-1)-token conv history per channel).
 * dims.seqlen is ignored.
 *
 *  A_log [d,N], D [d], dt_bias [d] (NULL = zeros), conv_w [d,K],
 *  conv_b [d] (NULL = zeros), zoh_mode  -- as above
 *  u_t        [Bt,d]      io   pre-conv input of this token
 *  dt_t       [Bt,d]      io   raw step size
 *  B_t, C_t   [Bt,N]      io
 *  z_t        [Bt,d]      io   NULL = no gate
 *  h_ssm      [Bt,d,N]    f32  read and overwritten with the new state
 *  conv_state [Bt,d,K-1]  io   read and overwritten: drops the oldest input,
 *                              appends u_t
 *  y_t        [Bt,d]      io   output (written)
 */
S6_API int s6_step(const s6_dims *dims, const float *A_log, const float *D, const float *dt_bias,
            const float *conv_w, const float *conv_b, int zoh_mode, const void *u_t,
            const void *dt_t, const void *B_t, const void *C_t, const void *z_t, float *h_ssm,
            void *conv_state, void *y_t, s6_stream_t stream);

/*
 * s6_block_step -- one token through one Mamba-mini decode block for Bt
 * independent sequences ("mamba, live", section "what is actually running":
 * the per-block listing; its "Weights" paragraph: per-row symmetric int8,
 * w = int8_row x scale_row, A_log kept in float32):
 *
 *     hn = LayerNorm(x);  [xin, z] = in_proj(hn);  xc = SiLU(conv_K(xin))
 *     [dt, B, C] = x_proj(xc);  Delta = softplus(dt_proj(dt) + dt_bias)
 *     h = exp(Delta A) h + (Delta B) xc,  A = -exp(A_log);  y = <h, C> + D xc
 *     x += out_proj(y * SiLU(z))
 *
 * Readings: in_proj, x_proj and out_proj have no bias; dt_proj's bias is
 * dt_bias; LayerNorm uses the biased variance, eps = dims.eps, weight and bias.
 *
 *  dims      batch Bt >= 0, d_model dm >= 1, d_inner di >= 1, d_state N in
 *            [1, 16], dt_rank R >= 1, conv_width K in [2, 4], eps
 *  w         the block's weights (device pointers, row-major [out][in]):
 *              ln_w, ln_b [dm] f32; in_q [2 di][dm] int8, in_s [2 di] f32
 *              (rows 0..di-1 give xin, di..2di-1 give z); conv_w [di][K] f32,
 *              conv_b [di] f32 (NULL = zeros); xp_q [R + 2N][di] int8, xp_s
 *              [R + 2N] f32 (rows: dt, then B, then C); dt_q [di][R] int8, dt_s
 *              [di] f32, dt_bias [di] f32; A_log [di][N] f32, D [di] f32;
 *              out_q [dm][di] int8, out_s [dm] f32.  w_row = q_row * s_row.
 *  x          [Bt][dm]      f32  the residual stream: read, and out_proj's
 *                                output added in place
 *  conv_state [Bt][di][K-1] f32  the K-1 previous xin, oldest first (in place)
 *  h_ssm      [Bt][di][N]   f32  the state (in place)
 * All float pointers need 4-byte alignment (A_log and h_ssm 16-byte when
 * N = 16).  Uses a library-owned scratch buffer for the intermediate rows
 * (xin|z, the x_proj rows, the gated readout): allocated on the first call on
 * a device, grown on demand; make that call before capturing a stream.
 * in_proj and out_proj split their reductions across blocks and add the
 * partial sums with float atomics, so the last bits of x can vary between
 * runs.  Their products keep float32 accuracy: the int8 weights are exact, and
 * where d_model and d_inner are multiples of 16 they run on the tensor cores
 * with each float32 activation split into two TF32 terms.
 */
typedef struct {
    int64_t batch;      /* Bt >= 0 */
    int64_t d_model;    /* dm */
    int64_t d_inner;    /* di */
    int64_t d_state;    /* N in [1, 16] */
    int64_t dt_rank;    /* R */
    int64_t conv_width; /* K in [2, 4] */
    float eps;          /* LayerNorm epsilon */
} s6_block_dims;

typedef struct {
    const float *ln_w, *ln_b;
    const int8_t *in_q;
    const float *in_s;
    const float *conv_w, *conv_b;
    const int8_t *xp_q;
    const float *xp_s;
    const int8_t *dt_q;
    const float *dt_s, *dt_bias;
    const float *A_log, *D;
    const int8_t *out_q;
    const float *out_s;
} s6_block_weights;

S6_API int s6_block_step(const s6_block_dims *dims, const s6_block_weights *w, float *x, float *conv_state,
                         float *h_ssm, s6_stream_t stream);

/*
 * s6_device_status -- synchronises `stream`, then reads and clears the
 * library's device-side error word.  Returns S6_ERR_TIMEOUT if a kernel gave
 * up a bounded wait (its outputs are then incomplete), S6_ERR_CUDA if the
 * stream or the copy failed, else S6_OK.
 */
S6_API int s6_device_status(s6_stream_t stream);

/*
 * s6_debug_carry_fault -- fault injection for tests of the failure path; the
 * pages have no counterpart.  Off by default; a process that never calls it is
 * unaffected.
 *
 * After the call, every scan that splits its sequences into segments gives up
 * a wait for a predecessor's carry after `carry_polls` polls (0 restores the
 * default, about 4M polls spaced by 64 ns sleeps), and the unit with index
 * `skip_publish_unit` (-1: none) publishes no carry, so its successor's wait
 * runs out: that kernel sets the device error word, continues from an
 * undefined start state and exits normally, and s6_device_status then returns
 * S6_ERR_TIMEOUT.  Nothing faults, traps or hangs.  Process-wide host state,
 * read when a scan is enqueued; not for concurrent use with other scans.
 */
S6_API int s6_debug_carry_fault(int skip_publish_unit, unsigned int carry_polls);

/* Human-readable name of an s6_status value (static string; never NULL). */
S6_API const char *s6_status_string(int status);

/* Library version, (major << 16) | minor. */
S6_API int s6_version(void);

#ifdef __cplusplus
}
#endif

#endif /* S6_B200_H */
