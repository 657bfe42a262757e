"""float64 CPU oracle for the S6 selective scan -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product library never loads it and
shares no code with it: the arithmetic lives in ``s6_oracle.c`` (plain C,
double precision, one channel / token / state coordinate at a time), and this
file only marshals numpy arrays into it and fans independent channels out over
host threads.

What the oracle computes (page titles and sections):

* "mamba, live", *what is actually running* -- the streaming block:
  ``xc = SiLU(conv4(x))``, ``dt = softplus(.)``, ``A = -exp(A_log)``,
  ``h <- exp(dt*A)*h + (dt*B)*xc``, ``y = <h, C> + D*xc``, gated by ``SiLU(z)``.
* "the s6 cell", *the recurrence* -- the same update with the decay written
  ``2^(dt*A*log2 e)``; ``dt*A <= 0``.
* "Carry context through a selective state" (the TinyMamba example and its
  model manifest, ``steps`` *local/select/state/read*) -- exact diagonal
  zero-order hold ``B_bar = (exp(dt*A) - 1)/A * B``, a zero-left-padded causal
  conv, C reading the updated state, D multiplying the conv output.
* ``diag_const`` -- "the s6 cell", *one cell, two architectures*: the same
  diagonal recurrence with a constant decay 2^w per (channel, state) instead of
  a per-token one, written B_t * u_t.
* ``block_step`` -- one token through one Mamba-mini block ("mamba, live",
  the per-block listing and *Weights*): LayerNorm, int8 per-row in_proj,
  conv + SiLU, x_proj, dt_proj + softplus, the recurrence, readout, gate,
  out_proj and the residual add.
* ``scan_bwd`` -- the gradients of that scan (no conv), by reverse-mode
  differentiation of the same steps; pinned by central differences of the
  forward oracle.

Every function here is pinned by ``tests/test_oracle_pins.py`` to values the
pages print or to closed forms; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "s6_oracle.c")
_LIB = os.path.join(_HERE, "libs6_oracle.so")

_c_double_p = ctypes.POINTER(ctypes.c_double)
_c_i64_p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile ``s6_oracle.c`` with gcc into ``libs6_oracle.so`` (in place)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def bind(path: str):
    """Load a compiled oracle library from ``path`` and declare its C signatures."""
    lib = ctypes.CDLL(path)
    d, i, i64 = ctypes.c_double, ctypes.c_int, ctypes.c_int64
    for name, args in (("s6o_softplus", [d]), ("s6o_silu", [d]), ("s6o_A", [d]),
                       ("s6o_decay", [d, d]), ("s6o_write_gain", [d, d, i]),
                       ("s6o_update", [d, d, d]), ("s6o_sigmoid", [d]), ("s6o_dsilu", [d])):
        f = getattr(lib, name)
        f.argtypes, f.restype = args, d
    lib.s6o_conv_pre.argtypes = [i, _c_double_p, d, _c_double_p, d]
    lib.s6o_conv_pre.restype = d
    lib.s6o_scan_channels.argtypes = [i64, i64, i, i, i] + [_c_double_p] * 5 + [_c_i64_p] + \
        [_c_double_p] * 10
    lib.s6o_scan_channels.restype = None
    lib.s6o_conv_silu_channels.argtypes = [i64, i64, i, _c_double_p, _c_double_p, _c_double_p,
                                           _c_double_p]
    lib.s6o_conv_silu_channels.restype = None
    lib.s6o_scan_bwd_channels.argtypes = [i64, i64, i, i] + [_c_double_p] * 5 + [_c_i64_p] + \
        [_c_double_p] * 15
    lib.s6o_scan_bwd_channels.restype = None
    lib.s6o_conv_silu_bwd_channels.argtypes = [i64, i64, i] + [_c_double_p] * 7
    lib.s6o_conv_silu_bwd_channels.restype = None
    lib.s6o_diag_const_channels.argtypes = [i64, i64, i] + [_c_double_p] * 4 + [_c_i64_p] + [_c_double_p] * 5
    lib.s6o_diag_const_channels.restype = None
    _c_i8_p = ctypes.POINTER(ctypes.c_int8)
    lib.s6o_layernorm.argtypes = [i, _c_double_p, _c_double_p, _c_double_p, d, _c_double_p]
    lib.s6o_layernorm.restype = None
    lib.s6o_linear_q8.argtypes = [i, i, _c_i8_p, _c_double_p, _c_double_p, _c_double_p]
    lib.s6o_linear_q8.restype = None
    lib.s6o_block_step_seqs.argtypes = ([i64, i, i, i, i, i, d, _c_double_p, _c_double_p, _c_i8_p, _c_double_p,
                                         _c_double_p, _c_double_p, _c_i8_p, _c_double_p, _c_i8_p, _c_double_p,
                                         _c_double_p, _c_double_p, _c_double_p, _c_i8_p, _c_double_p] +
                                        [_c_double_p] * 4)
    lib.s6o_block_step_seqs.restype = None
    for name in ("s6o_ssm_state_values", "s6o_conv_history_values"):
        f = getattr(lib, name)
        f.argtypes, f.restype = [i64, i64, i64], i64
    lib.s6o_abi_version.restype = i
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(build())
    return _lib


class use_library:
    """Context manager: route every oracle call through another build (tests only)."""

    def __init__(self, path: str):
        self.lib = bind(path)

    def __enter__(self):
        global _lib
        self.prev, _lib = _load(), self.lib
        return self.lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.prev


# ---------------------------------------------------------------- scalar steps
def softplus(v: float) -> float:
    return _load().s6o_softplus(float(v))


def silu(v: float) -> float:
    return _load().s6o_silu(float(v))


def A_of(A_log: float) -> float:
    return _load().s6o_A(float(A_log))


def decay(delta: float, A_log: float) -> float:
    return _load().s6o_decay(float(delta), float(A_log))


def write_gain(delta: float, A_log: float, zoh: bool) -> float:
    return _load().s6o_write_gain(float(delta), float(A_log), int(bool(zoh)))


def update(h: float, a_bar: float, write: float) -> float:
    return _load().s6o_update(float(h), float(a_bar), float(write))


def sigmoid(v: float) -> float:
    return _load().s6o_sigmoid(float(v))


def dsilu(v: float) -> float:
    return _load().s6o_dsilu(float(v))


def conv_pre(w, bias: float, hist, x_t: float) -> float:
    w = np.ascontiguousarray(w, dtype=np.float64)
    hist = np.ascontiguousarray(hist, dtype=np.float64)
    if hist.size == 0:
        hist = np.zeros(1)
    return _load().s6o_conv_pre(int(w.size), _ptr(w), float(bias), _ptr(hist), float(x_t))


def ssm_state_values(d_inner: int, d_state: int, blocks: int = 1) -> int:
    return _load().s6o_ssm_state_values(d_inner, d_state, blocks)


def conv_history_values(d_inner: int, K: int, blocks: int = 1) -> int:
    return _load().s6o_conv_history_values(d_inner, K, blocks)


# ------------------------------------------------------------------ marshalling
def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(_c_double_p)


def _f64(a):
    """Any stored input -> float64.  uint16 arrays hold bfloat16 bit patterns."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _threads(n_items: int, threads) -> int:
    if threads is None:
        threads = os.cpu_count() or 1
    return max(1, min(int(threads), n_items))


def scan(x, dt_raw, A_log, B, C, D, z=None, dt_bias=None, zoh=False, conv_w=None, conv_b=None,
         channels=None, h_init=None, conv_hist=None, threads=None, return_state=False):
    """Selective scan over [Bt, L, d] inputs, one independent channel at a time.

    x: pre-conv input when ``conv_w`` is given, else the scan input u.
    dt_raw, z: [Bt, L, d]; B, C: [Bt, L, N]; A_log: [d, N]; D, dt_bias,
    conv_b: [d]; conv_w: [d, K].  ``channels``: None for all, or an int array
    of shape [n, 2] of (b, d) pairs.  ``h_init`` [.., N] and ``conv_hist``
    [.., K-1] (same leading layout as the result) start from a given state.

    Returns (y, h_final) as float64: [Bt, L, d] and [Bt, d, N] for all
    channels, or [n, L] and [n, N] for a channel list.  With
    ``return_state`` also returns the conv history after the last token.
    """
    x = np.asarray(x)
    Bt, L, d = x.shape
    N = np.asarray(A_log).shape[1]
    K = 0 if conv_w is None else np.asarray(conv_w).shape[1]
    km1 = max(K - 1, 0)
    full = channels is None
    if full:
        bb, dd = np.meshgrid(np.arange(Bt), np.arange(d), indexing="ij")
        channels = np.stack([bb.ravel(), dd.ravel()], axis=1)
    channels = np.asarray(channels, dtype=np.int64).reshape(-1, 2)
    n = channels.shape[0]
    cb, cd = channels[:, 0], channels[:, 1]

    def gather_seq(a):
        return np.ascontiguousarray(_f64(np.asarray(a)[cb, :, cd]).reshape(n, L))

    xs = gather_seq(x)
    dts = gather_seq(dt_raw)
    zs = gather_seq(z) if z is not None else None
    Bm = np.ascontiguousarray(_f64(B)).reshape(-1)
    Cm = np.ascontiguousarray(_f64(C)).reshape(-1)
    bc_row = np.ascontiguousarray(cb)
    Al = np.ascontiguousarray(_f64(A_log)[cd])
    Dv = np.ascontiguousarray(_f64(D)[cd])
    bias = np.ascontiguousarray(_f64(dt_bias)[cd]) if dt_bias is not None else None
    cw = np.ascontiguousarray(_f64(conv_w)[cd]) if K > 0 else None
    cbias = np.ascontiguousarray(_f64(conv_b)[cd]) if (K > 0 and conv_b is not None) else None
    hin = None
    if h_init is not None:
        hin = np.ascontiguousarray(_f64(h_init)[cb, cd] if full else _f64(h_init)).reshape(n, N)
    hist = None
    if conv_hist is not None and km1 > 0:
        hist = np.ascontiguousarray(_f64(conv_hist)[cb, cd] if full else _f64(conv_hist)).reshape(n, km1)

    y = np.zeros((n, L))
    hout = np.zeros((n, N))
    histout = np.zeros((n, max(km1, 1)))
    lib = _load()

    def run(lo, hi):
        sl = slice(lo, hi)

        def p(a):
            return None if a is None else _ptr(a[sl])

        lib.s6o_scan_channels(hi - lo, L, N, K, int(bool(zoh)),
                              p(xs), p(dts), p(zs), _ptr(Bm), _ptr(Cm),
                              bc_row[sl].ctypes.data_as(_c_i64_p),
                              p(Al), p(Dv), p(bias), p(cw), p(cbias), p(hist), p(hin),
                              p(y), p(hout), p(histout) if km1 > 0 else None)

    nt = _threads(n, threads)
    bounds = np.linspace(0, n, nt + 1).astype(np.int64)
    if nt == 1:
        run(0, n)
    else:
        with ThreadPoolExecutor(nt) as ex:
            list(ex.map(lambda i: run(int(bounds[i]), int(bounds[i + 1])), range(nt)))

    if full:
        y_full = np.zeros((Bt, L, d))
        y_full[cb, :, cd] = y
        h_full = hout.reshape(Bt, d, N)
        hs = histout[:, :km1].reshape(Bt, d, km1)
        return (y_full, h_full, hs) if return_state else (y_full, h_full)
    return (y, hout, histout[:, :km1]) if return_state else (y, hout)


def diag_const(u, log2_decay, B, C, D, z=None, channels=None, h_init=None, threads=None):
    """The constant-decay diagonal recurrence ("the s6 cell", *one cell, two
    architectures*): h <- 2^w * h + B_t * u_t per state, y = (<h, C_t> + D u) * SiLU(z).

    u, z: [Bt, L, d]; B, C: [Bt, L, N]; log2_decay (w <= 0): [d, N]; D: [d];
    h_init: [Bt, d, N] or None.  ``channels`` as in ``scan``.  Returns (y, h_final)
    in float64: [Bt, L, d] / [Bt, d, N], or [n, L] / [n, N] for a channel list.
    """
    u = np.asarray(u)
    Bt, L, d = u.shape
    N = np.asarray(log2_decay).shape[1]
    full = channels is None
    if full:
        bb, dd = np.meshgrid(np.arange(Bt), np.arange(d), indexing="ij")
        channels = np.stack([bb.ravel(), dd.ravel()], axis=1)
    channels = np.asarray(channels, dtype=np.int64).reshape(-1, 2)
    n = channels.shape[0]
    cb, cd = channels[:, 0], channels[:, 1]

    def gather_seq(a):
        return np.ascontiguousarray(_f64(np.asarray(a)[cb, :, cd]).reshape(n, L))

    us = gather_seq(u)
    zs = gather_seq(z) if z is not None else None
    Bm = np.ascontiguousarray(_f64(B)).reshape(-1)
    Cm = np.ascontiguousarray(_f64(C)).reshape(-1)
    bc_row = np.ascontiguousarray(cb)
    W = np.ascontiguousarray(_f64(log2_decay)[cd])
    Dv = np.ascontiguousarray(_f64(D)[cd])
    hin = None
    if h_init is not None:
        hin = np.ascontiguousarray(_f64(h_init)[cb, cd] if full else _f64(h_init)).reshape(n, N)
    y = np.zeros((n, L))
    hout = np.zeros((n, N))
    lib = _load()

    def run(lo, hi):
        sl = slice(lo, hi)

        def p(a):
            return None if a is None else _ptr(a[sl])

        lib.s6o_diag_const_channels(hi - lo, L, N, p(us), p(zs), _ptr(Bm), _ptr(Cm),
                                    bc_row[sl].ctypes.data_as(_c_i64_p), p(W), p(Dv), p(hin), p(y), p(hout))

    nt = _threads(n, threads)
    bounds = np.linspace(0, n, nt + 1).astype(np.int64)
    with ThreadPoolExecutor(nt) as ex:
        list(ex.map(lambda i: run(int(bounds[i]), int(bounds[i + 1])), range(nt)))
    if full:
        y_full = np.zeros((Bt, L, d))
        y_full[cb, :, cd] = y
        return y_full, hout.reshape(Bt, d, N)
    return y, hout


def layernorm(x, w, b, eps=1e-5):
    """LayerNorm of each row of x (the last axis), biased variance, affine."""
    x = np.ascontiguousarray(_f64(x))
    rows = x.reshape(-1, x.shape[-1])
    out = np.zeros_like(rows)
    wv, bv = np.ascontiguousarray(_f64(w)), np.ascontiguousarray(_f64(b))
    for r in range(rows.shape[0]):
        _load().s6o_layernorm(rows.shape[1], _ptr(rows[r]), _ptr(wv), _ptr(bv), float(eps), _ptr(out[r]))
    return out.reshape(x.shape)


def linear_q8(q, scale, x):
    """y = scale[o] * sum_i q[o, i] x[i] for each row of x: a Linear with per-row int8 weights."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    sc = np.ascontiguousarray(_f64(scale))
    x = np.ascontiguousarray(_f64(x))
    rows = x.reshape(-1, x.shape[-1])
    out = np.zeros((rows.shape[0], q.shape[0]))
    for r in range(rows.shape[0]):
        _load().s6o_linear_q8(q.shape[0], q.shape[1], q.ctypes.data_as(ctypes.POINTER(ctypes.c_int8)), _ptr(sc),
                              _ptr(rows[r]), _ptr(out[r]))
    return out.reshape(x.shape[:-1] + (q.shape[0],))


_BLOCK_KEYS = ("ln_w", "ln_b", "in_q", "in_s", "conv_w", "conv_b", "xp_q", "xp_s", "dt_q", "dt_s", "dt_bias",
               "A_log", "D", "out_q", "out_s")


def block_step(x, conv_state, h, w, eps=1e-5, threads=None):
    """One token through one decode block ("mamba, live", the per-block listing)
    for each sequence: x [Bt, dm], conv_state [Bt, di, K-1], h [Bt, di, N];
    ``w`` the block's weights (s6_inputs.block_weights).  Returns new
    (x, conv_state, h) as float64 arrays; the inputs are not modified."""
    x = np.array(_f64(x), copy=True)
    cs = np.array(_f64(conv_state), copy=True)
    hh = np.array(_f64(h), copy=True)
    Bt, dm = x.shape
    di, N = np.asarray(w["A_log"]).shape
    K = np.asarray(w["conv_w"]).shape[1]
    R = np.asarray(w["dt_q"]).shape[1]
    arrs = {}
    for k in _BLOCK_KEYS:
        v = np.asarray(w[k])
        arrs[k] = np.ascontiguousarray(v, dtype=np.int8) if v.dtype == np.int8 else np.ascontiguousarray(_f64(v))
    i8 = ctypes.POINTER(ctypes.c_int8)

    def p(k):
        a = arrs[k]
        return a.ctypes.data_as(i8) if a.dtype == np.int8 else _ptr(a)

    nt = _threads(Bt, threads)
    bounds = np.linspace(0, Bt, nt + 1).astype(np.int64)

    def run(i):
        lo, hi = int(bounds[i]), int(bounds[i + 1])
        work = np.zeros(6 * di + dm + R + 2 * N)
        _load().s6o_block_step_seqs(hi - lo, dm, di, N, R, K, float(eps), *[p(k) for k in _BLOCK_KEYS],
                                    _ptr(x[lo:hi]), _ptr(cs[lo:hi]), _ptr(hh[lo:hi]), _ptr(work))

    with ThreadPoolExecutor(nt) as ex:
        list(ex.map(run, range(nt)))
    return x, cs, hh


def scan_bwd(u, dt_raw, A_log, B, C, D, dy, z=None, dt_bias=None, zoh=False, h_init=None, threads=None):
    """Gradients of the scan without conv (u given) for the loss sum(dy * y).

    u, dt_raw, z, dy: [Bt, L, d]; B, C: [Bt, L, N]; A_log: [d, N]; D, dt_bias:
    [d]; h_init: [Bt, d, N] or None (zeros).  Returns a dict of float64 arrays:
    du, ddt, dz (None without z) [Bt, L, d]; dB, dC [Bt, L, N]; dA_log [d, N];
    dD, ddt_bias [d]; dh_init [Bt, d, N].
    """
    u = np.asarray(u)
    Bt, L, d = u.shape
    N = np.asarray(A_log).shape[1]
    bb, dd = np.meshgrid(np.arange(Bt), np.arange(d), indexing="ij")
    cb, cd = bb.ravel(), dd.ravel()
    n = Bt * d

    def seq(a):
        return np.ascontiguousarray(np.transpose(_f64(a), (0, 2, 1))).reshape(n, L)

    us, dts, dys = seq(u), seq(dt_raw), seq(dy)
    zs = seq(z) if z is not None else None
    Bm = np.ascontiguousarray(_f64(B)).reshape(-1)
    Cm = np.ascontiguousarray(_f64(C)).reshape(-1)
    bc_row = np.ascontiguousarray(cb.astype(np.int64))
    Al = np.ascontiguousarray(_f64(A_log)[cd])
    Dv = np.ascontiguousarray(_f64(D)[cd])
    bias = np.ascontiguousarray(_f64(dt_bias)[cd]) if dt_bias is not None else None
    hin = np.ascontiguousarray(_f64(h_init).reshape(n, N)) if h_init is not None else None
    du, ddt = np.zeros((n, L)), np.zeros((n, L))
    dz = np.zeros((n, L)) if z is not None else None
    dBc, dCc = np.zeros((n, L, N)), np.zeros((n, L, N))
    dAl, dDc, dbc, dh = np.zeros((n, N)), np.zeros(n), np.zeros(n), np.zeros((n, N))
    lib = _load()
    nt = _threads(n, threads)
    bounds = np.linspace(0, n, nt + 1).astype(np.int64)

    def run(i):
        lo, hi = int(bounds[i]), int(bounds[i + 1])
        sl = slice(lo, hi)

        def p(a):
            return None if a is None else _ptr(a[sl])

        work = np.zeros((L + 1) * N)
        lib.s6o_scan_bwd_channels(hi - lo, L, N, int(bool(zoh)), p(us), p(dts), p(zs), _ptr(Bm), _ptr(Cm),
                                  bc_row[sl].ctypes.data_as(_c_i64_p), p(Al), p(Dv), p(bias), p(hin), p(dys),
                                  p(du), p(ddt), p(dz), p(dBc), p(dCc), p(dAl), p(dDc), p(dbc), p(dh), _ptr(work))

    with ThreadPoolExecutor(nt) as ex:
        list(ex.map(run, range(nt)))

    def back(a):
        return np.transpose(a.reshape(Bt, d, L), (0, 2, 1))

    return {"du": back(du), "ddt": back(ddt), "dz": back(dz) if dz is not None else None,
            # B and C rows are shared by the d channels of a sequence: sum their shares
            "dB": dBc.reshape(Bt, d, L, N).sum(axis=1), "dC": dCc.reshape(Bt, d, L, N).sum(axis=1),
            "dA_log": dAl.reshape(Bt, d, N).sum(axis=0), "dD": dDc.reshape(Bt, d).sum(axis=0),
            "ddt_bias": dbc.reshape(Bt, d).sum(axis=0), "dh_init": dh.reshape(Bt, d, N)}


def conv_scan_bwd(x, conv_w, conv_b, dt_raw, A_log, B, C, D, dy, z=None, dt_bias=None, zoh=False, h_init=None,
                  threads=None):
    """Gradients of the fused path (causal conv + SiLU, then the scan) for the loss
    sum(dy * y): the scan's backward on u = SiLU(conv(x)), then the conv's
    backward on du.  Returns the dict of scan_bwd with du replaced by dx
    [Bt, L, d], plus dconv_w [d, K] and dconv_b [d]."""
    x = np.asarray(x)
    Bt, L, d = x.shape
    K = np.asarray(conv_w).shape[1]
    u = conv_silu(x, conv_w, conv_b, threads=threads)
    g = scan_bwd(u, dt_raw, A_log, B, C, D, dy, z=z, dt_bias=dt_bias, zoh=zoh, h_init=h_init, threads=threads)
    n = Bt * d
    xs = np.ascontiguousarray(np.transpose(_f64(x), (0, 2, 1))).reshape(n, L)
    dxc = np.ascontiguousarray(np.transpose(g.pop("du"), (0, 2, 1))).reshape(n, L)
    cw = np.ascontiguousarray(np.tile(_f64(conv_w), (Bt, 1)))
    cbias = np.ascontiguousarray(np.tile(_f64(conv_b), Bt)) if conv_b is not None else None
    dx, dw, db = np.zeros((n, L)), np.zeros((n, K)), np.zeros(n)
    _load().s6o_conv_silu_bwd_channels(n, L, K, _ptr(xs), _ptr(cw), _ptr(cbias), _ptr(dxc), _ptr(dx), _ptr(dw),
                                      _ptr(db))
    g["dx"] = np.transpose(dx.reshape(Bt, d, L), (0, 2, 1))
    g["dconv_w"] = dw.reshape(Bt, d, K).sum(axis=0)
    g["dconv_b"] = db.reshape(Bt, d).sum(axis=0)
    return g


def conv_silu(x, conv_w, conv_b=None, threads=None):
    """Standalone causal depthwise conv + SiLU: [Bt, L, d] -> [Bt, L, d] float64."""
    x = np.asarray(x)
    Bt, L, d = x.shape
    K = np.asarray(conv_w).shape[1]
    xs = np.ascontiguousarray(np.transpose(_f64(x), (0, 2, 1))).reshape(Bt * d, L)
    cw = np.ascontiguousarray(np.tile(_f64(conv_w), (Bt, 1)))
    cbias = np.ascontiguousarray(np.tile(_f64(conv_b), Bt)) if conv_b is not None else None
    out = np.zeros((Bt * d, L))
    lib = _load()
    n = Bt * d
    nt = _threads(n, threads)
    bounds = np.linspace(0, n, nt + 1).astype(np.int64)

    def run(i):
        lo, hi = int(bounds[i]), int(bounds[i + 1])
        lib.s6o_conv_silu_channels(hi - lo, L, K, _ptr(xs[lo:hi]), _ptr(cw[lo:hi]),
                                   _ptr(cbias[lo:hi]) if cbias is not None else None,
                                   _ptr(out[lo:hi]))

    with ThreadPoolExecutor(nt) as ex:
        list(ex.map(run, range(nt)))
    return np.transpose(out.reshape(Bt, d, L), (0, 2, 1))


def step(x_t, dt_t, B_t, C_t, A_log, D, dt_bias, conv_w, conv_b, h, conv_state, z_t=None,
         zoh=False, threads=None):
    """One streaming token for Bt sequences (the block's streaming form).

    x_t, dt_t, z_t: [Bt, d]; B_t, C_t: [Bt, N]; h: [Bt, d, N];
    conv_state: [Bt, d, K-1] (oldest first).  Returns (y_t [Bt, d],
    h' [Bt, d, N], conv_state' [Bt, d, K-1]) in float64.  The body is the scan's
    body applied to one token with the carried state.
    """
    x_t = np.asarray(x_t)
    Bt, d = x_t.shape
    y, hn, hist = scan(x_t[:, None, :], np.asarray(dt_t)[:, None, :], A_log,
                       np.asarray(B_t)[:, None, :], np.asarray(C_t)[:, None, :], D,
                       z=None if z_t is None else np.asarray(z_t)[:, None, :], dt_bias=dt_bias,
                       zoh=zoh, conv_w=conv_w, conv_b=conv_b, h_init=h, conv_hist=conv_state,
                       threads=threads, return_state=True)
    return y[:, 0, :], hn, hist
