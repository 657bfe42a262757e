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
 * call uses the library-owned scratch buffer (state checkpoints every 64
 * tokens plus one chunk of states: (ceil(L/64) + 64) * Bt * d * 16 floats at
 * N = 16).  Pointers need only element alignment.
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
 * s6_device_status -- synchronises `stream`, then reads and clears the
 * library's device-side error word.  Returns S6_ERR_TIMEOUT if a kernel gave
 * up a bounded wait (its outputs are then incomplete), S6_ERR_CUDA if the
 * stream or the copy failed, else S6_OK.
 */
S6_API int s6_device_status(s6_stream_t stream);

/* Human-readable name of an s6_status value (static string; never NULL). */
S6_API const char *s6_status_string(int status);

/* Library version, (major << 16) | minor. */
S6_API int s6_version(void);

#ifdef __cplusplus
}
#endif

#endif /* S6_B200_H */
