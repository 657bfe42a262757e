"""B200 (sm_100a) selective scan (Mamba S6) -- Python binding of libs6_b200.so.

This module only marshals arguments: it checks dtype / device / contiguity of
torch tensors, allocates outputs with torch when the caller passes none, and
hands raw device pointers plus the current CUDA stream to the C ABI declared in
``include/s6.h``.  Every arithmetic step runs in the library's CUDA kernels.
There is no CPU fallback: if the library is missing, the first call raises.

Functions (same names as the C ABI):
    s6_scan_fwd, s6_conv_scan_fwd, s6_conv_scan_fwd_noalloc, s6_scan_fwd_from_state,
    s6_conv_scan_fwd_from_state, s6_diag_recurrence_fwd, s6_scan_bwd, s6_conv_scan_bwd,
    causal_conv1d_silu_fwd, s6_step, s6_block_step, s6_device_status, s6_status_string, s6_version,
    s6_debug_carry_fault (tests only)
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "S6Error", "lib", "s6_scan_fwd", "s6_conv_scan_fwd", "s6_conv_scan_fwd_noalloc", "s6_scan_fwd_from_state",
    "s6_conv_scan_fwd_from_state", "s6_scan_fwd_ckpt", "s6_conv_scan_fwd_ckpt", "CKPT_EVERY",
    "s6_diag_recurrence_fwd", "S6_DECAY_LIVE", "S6_DECAY_CONST", "s6_scan_bwd", "s6_conv_scan_bwd",
    "causal_conv1d_silu_fwd", "s6_step",
    "s6_block_step", "BlockDims", "BlockWeights", "BLOCK_WEIGHT_KEYS",
    "s6_device_status", "s6_status_string", "s6_version", "s6_debug_carry_fault", "S6_F32", "S6_BF16", "Dims",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libs6_b200.so")

S6_F32, S6_BF16 = 0, 1
S6_OK, S6_ERR_INVALID_ARG, S6_ERR_UNSUPPORTED, S6_ERR_ALIGNMENT, S6_ERR_CUDA, S6_ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
S6_ERR_SCRATCH_LIMIT = -6
S6_DECAY_LIVE, S6_DECAY_CONST = 0, 1
CKPT_EVERY = 16  # tokens between the states a training forward keeps for the backward


class Dims(ctypes.Structure):
    """Mirror of ``s6_dims``."""
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("d_inner", ctypes.c_int64),
                ("d_state", ctypes.c_int64), ("conv_width", ctypes.c_int64), ("io_dtype", ctypes.c_int32)]


class BlockDims(ctypes.Structure):
    """Mirror of ``s6_block_dims``."""
    _fields_ = [("batch", ctypes.c_int64), ("d_model", ctypes.c_int64), ("d_inner", ctypes.c_int64),
                ("d_state", ctypes.c_int64), ("dt_rank", ctypes.c_int64), ("conv_width", ctypes.c_int64),
                ("eps", ctypes.c_float)]


BLOCK_WEIGHT_KEYS = ("ln_w", "ln_b", "in_q", "in_s", "conv_w", "conv_b", "xp_q", "xp_s", "dt_q", "dt_s", "dt_bias",
                     "A_log", "D", "out_q", "out_s")


class BlockWeights(ctypes.Structure):
    """Mirror of ``s6_block_weights`` (device pointers)."""
    _fields_ = [(k, ctypes.c_void_p) for k in BLOCK_WEIGHT_KEYS]


class S6Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {s6_status_string(status)} ({status})")


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"CUDA library {LIB_PATH} is missing: build it with `python -m selective_state_space_19_b200._build`"
                " (or __graft_entry__.build()); there is no CPU fallback")
        L = ctypes.CDLL(LIB_PATH)
        DP = ctypes.POINTER(Dims)
        L.s6_scan_fwd.argtypes = [DP, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P]
        L.s6_conv_scan_fwd.argtypes = [DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P]
        L.s6_conv_scan_fwd_noalloc.argtypes = [DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P]
        L.s6_scan_fwd_from_state.argtypes = [DP, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P]
        L.s6_conv_scan_fwd_from_state.argtypes = [DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P]
        L.s6_diag_recurrence_fwd.argtypes = [DP, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]
        L.s6_scan_bwd.argtypes = [DP, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P] + [_P] * 9 + [_P]
        L.s6_conv_scan_bwd.argtypes = [DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P] + [_P] * 11 + [_P]
        L.s6_scan_fwd_ckpt.argtypes = [DP, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P]
        L.s6_conv_scan_fwd_ckpt.argtypes = [DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P]
        L.s6_scan_bwd_ckpt.argtypes = L.s6_scan_bwd.argtypes
        L.s6_conv_scan_bwd_ckpt.argtypes = L.s6_conv_scan_bwd.argtypes
        L.causal_conv1d_silu_fwd.argtypes = [DP, _P, _P, _P, _P, _P]
        L.s6_step.argtypes = [DP, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]
        L.s6_device_status.argtypes = [_P]
        L.s6_status_string.argtypes = [_I]
        L.s6_status_string.restype = ctypes.c_char_p
        L.s6_version.argtypes = []
        L.s6_debug_carry_fault.argtypes = [_I, ctypes.c_uint]
        L.s6_block_step.argtypes = [ctypes.POINTER(BlockDims), ctypes.POINTER(BlockWeights), _P, _P, _P, _P]
        L.s6_block_step.restype = _I
        L.s6_debug_carry_fault.restype = _I
        for f in (L.s6_scan_fwd, L.s6_conv_scan_fwd, L.s6_conv_scan_fwd_noalloc, L.s6_scan_fwd_from_state,
                  L.s6_conv_scan_fwd_from_state, L.s6_diag_recurrence_fwd, L.s6_scan_bwd, L.s6_conv_scan_bwd, L.causal_conv1d_silu_fwd, L.s6_step,
                  L.s6_device_status, L.s6_version):
            f.restype = _I
        _lib = L
    return _lib


def s6_status_string(status: int) -> str:
    return lib().s6_status_string(int(status)).decode()


def s6_version() -> int:
    return lib().s6_version()


def _torch():
    import torch
    return torch


def _io_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return S6_F32
    if t.dtype == torch.bfloat16:
        return S6_BF16
    raise TypeError(f"I/O tensors must be float32 or bfloat16, got {t.dtype}")


def _ptr(t, name, dtype=None, shape=None, device=None):
    if t is None:
        return None
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def _stream(stream, device):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status, where):
    if status != S6_OK:
        raise S6Error(status, where)


def _scan(fn, x, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final, conv_w, conv_b, want_h, stream,
          from_state=False, h_init=None, conv_hist=None, ckpt_mode=False, ckpt=None):
    torch = _torch()
    if x.dim() != 3:
        raise ValueError("x/u must be [batch, seqlen, d_inner]")
    Bt, L, d = x.shape
    io = _io_code(x)
    N = A_log.shape[-1]
    dev = x.device
    f32 = torch.float32
    K = conv_w.shape[-1] if conv_w is not None else 0
    if y is None:
        y = torch.empty_like(x)
    if h_final is None and want_h:
        h_final = torch.empty((Bt, d, N), dtype=f32, device=dev)
    dims = Dims(Bt, L, d, N, K, io)
    args = [ctypes.byref(dims)]
    seq = (Bt, L, d)
    xp = _ptr(x, "x", x.dtype, seq, dev)
    if conv_w is not None:
        args += [xp, _ptr(conv_w, "conv_w", f32, (d, K), dev), _ptr(conv_b, "conv_b", f32, (d,), dev)]
    else:
        args += [xp]
    args += [_ptr(dt, "dt", x.dtype, seq, dev), _ptr(A_log, "A_log", f32, (d, N), dev),
             _ptr(B, "B", x.dtype, (Bt, L, N), dev), _ptr(C, "C", x.dtype, (Bt, L, N), dev),
             _ptr(D, "D", f32, (d,), dev), _ptr(z, "z", x.dtype, seq, dev),
             _ptr(dt_bias, "dt_bias", f32, (d,), dev), int(zoh_mode)]
    if from_state or ckpt_mode:
        args += [_ptr(h_init, "h_init", f32, (Bt, d, N), dev)]
        if conv_w is not None and not ckpt_mode:
            args += [_ptr(conv_hist, "conv_hist", x.dtype, (Bt, d, K - 1), dev)]
    args += [_ptr(y, "y", x.dtype, seq, dev), _ptr(h_final, "h_final", f32, (Bt, d, N), dev)]
    if ckpt_mode:
        if ckpt is None:
            ckpt = torch.empty((Bt, (L + CKPT_EVERY - 1) // CKPT_EVERY, d, N), dtype=f32, device=dev)
        args += [_ptr(ckpt, "ckpt", f32, (Bt, (L + CKPT_EVERY - 1) // CKPT_EVERY, d, N), dev)]
    args += [_stream(stream, dev)]
    _check(fn(*args), fn.__name__)
    if ckpt_mode:
        return y, h_final, ckpt
    return y, h_final


def s6_scan_fwd(u, dt, A_log, B, C, D, z=None, dt_bias=None, zoh_mode=0, y=None, h_final=None,
                want_h_final=True, stream=None):
    """Selective scan of an already-convolved input u.  Returns (y, h_final)."""
    return _scan(lib().s6_scan_fwd, u, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final, None, None,
                 want_h_final, stream)


def s6_conv_scan_fwd(x, conv_w, conv_b, dt, A_log, B, C, D, z=None, dt_bias=None, zoh_mode=0, y=None,
                     h_final=None, want_h_final=True, stream=None):
    """Fused causal conv + SiLU + selective scan + gate.  Returns (y, h_final)."""
    return _scan(lib().s6_conv_scan_fwd, x, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final, conv_w,
                 conv_b, want_h_final, stream)


def s6_conv_scan_fwd_noalloc(x, conv_w, conv_b, dt, A_log, B, C, D, z=None, dt_bias=None, zoh_mode=0, y=None,
                             h_final=None, want_h_final=True, stream=None):
    """s6_conv_scan_fwd for callers that cannot let the library allocate device
    memory: the segment carries live in a fixed array inside the library.  Pass
    y and h_final to keep this call free of allocations on the torch side too."""
    return _scan(lib().s6_conv_scan_fwd_noalloc, x, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final, conv_w,
                 conv_b, want_h_final, stream)


def s6_scan_fwd_from_state(u, dt, A_log, B, C, D, z=None, dt_bias=None, zoh_mode=0, h_init=None, y=None,
                           h_final=None, want_h_final=True, stream=None):
    """s6_scan_fwd started from the state h_init [Bt, d, N] (None = zeros).  Returns (y, h_final)."""
    return _scan(lib().s6_scan_fwd_from_state, u, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final, None, None,
                 want_h_final, stream, from_state=True, h_init=h_init)


def s6_conv_scan_fwd_from_state(x, conv_w, conv_b, dt, A_log, B, C, D, z=None, dt_bias=None, zoh_mode=0,
                                h_init=None, conv_hist=None, y=None, h_final=None, want_h_final=True, stream=None):
    """s6_conv_scan_fwd started from the state h_init [Bt, d, N] and the conv history
    conv_hist [Bt, d, K-1] (the K-1 inputs before token 0, oldest first; None = zeros).
    Returns (y, h_final)."""
    return _scan(lib().s6_conv_scan_fwd_from_state, x, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final, conv_w,
                 conv_b, want_h_final, stream, from_state=True, h_init=h_init, conv_hist=conv_hist)


def s6_scan_fwd_ckpt(u, dt, A_log, B, C, D, z=None, dt_bias=None, zoh_mode=0, h_init=None, y=None, h_final=None,
                     ckpt=None, want_h_final=True, stream=None):
    """The forward of a training step: s6_scan_fwd_from_state that also keeps the
    state before every 16th token, ckpt [Bt, ceil(L/16), d, 16] float32, for
    s6_scan_bwd(..., ckpt=ckpt).  N = 16.  Returns (y, h_final, ckpt)."""
    return _scan(lib().s6_scan_fwd_ckpt, u, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final, None, None,
                 want_h_final, stream, h_init=h_init, ckpt_mode=True, ckpt=ckpt)


def s6_conv_scan_fwd_ckpt(x, conv_w, conv_b, dt, A_log, B, C, D, z=None, dt_bias=None, zoh_mode=0, h_init=None,
                          y=None, h_final=None, ckpt=None, want_h_final=True, stream=None):
    """The forward of a training step on the fused path (zero conv history): also
    keeps the state before every 16th token for s6_conv_scan_bwd(..., ckpt=ckpt).
    N = 16.  Returns (y, h_final, ckpt)."""
    return _scan(lib().s6_conv_scan_fwd_ckpt, x, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final, conv_w,
                 conv_b, want_h_final, stream, h_init=h_init, ckpt_mode=True, ckpt=ckpt)


def s6_diag_recurrence_fwd(u, B, C, D, decay_source=S6_DECAY_CONST, log2_decay=None, dt=None, A_log=None,
                           dt_bias=None, z=None, h_init=None, y=None, h_final=None, want_h_final=True, stream=None):
    """The diagonal recurrence with the decay source as a parameter: constant
    (h <- 2^log2_decay * h + B_t u_t; log2_decay [d, N]) or live (the selective
    scan, dt and A_log given).  Returns (y, h_final)."""
    torch = _torch()
    if u.dim() != 3:
        raise ValueError("u must be [batch, seqlen, d_inner]")
    Bt, L, d = u.shape
    par = A_log if decay_source == S6_DECAY_LIVE else log2_decay
    if par is None:
        par = A_log if A_log is not None else log2_decay
    if par is None:
        raise ValueError("log2_decay (constant decay) or A_log (live decay) is required")
    N = par.shape[-1]
    dev = u.device
    f32 = torch.float32
    if y is None:
        y = torch.empty_like(u)
    if h_final is None and want_h_final:
        h_final = torch.empty((Bt, d, N), dtype=f32, device=dev)
    dims = Dims(Bt, L, d, N, 0, _io_code(u))
    seq = (Bt, L, d)
    st = lib().s6_diag_recurrence_fwd(
        ctypes.byref(dims), int(decay_source), _ptr(u, "u", u.dtype, seq, dev), _ptr(dt, "dt", u.dtype, seq, dev),
        _ptr(A_log, "A_log", f32, (d, N), dev), _ptr(dt_bias, "dt_bias", f32, (d,), dev),
        _ptr(log2_decay, "log2_decay", f32, (d, N), dev), _ptr(B, "B", u.dtype, (Bt, L, N), dev),
        _ptr(C, "C", u.dtype, (Bt, L, N), dev), _ptr(D, "D", f32, (d,), dev), _ptr(z, "z", u.dtype, seq, dev),
        _ptr(h_init, "h_init", f32, (Bt, d, N), dev), _ptr(y, "y", u.dtype, seq, dev),
        _ptr(h_final, "h_final", f32, (Bt, d, N), dev), _stream(stream, dev))
    _check(st, "s6_diag_recurrence_fwd")
    return y, h_final


def _bwd_start(fn, fn_ckpt, h_init, ckpt, Bt, L, d, N, dev):
    """The backward entry point and its start argument: h_init, or the checkpoints
    of a training forward (which hold the start state)."""
    if ckpt is None:
        return fn, _ptr(h_init, "h_init", _torch().float32, (Bt, d, N), dev)
    if h_init is not None:
        raise ValueError("with ckpt, the start state is in the checkpoints: pass h_init to the forward")
    return fn_ckpt, _ptr(ckpt, "ckpt", _torch().float32, (Bt, (L + CKPT_EVERY - 1) // CKPT_EVERY, d, N), dev)


def s6_scan_bwd(u, dt, A_log, B, C, D, dy, z=None, dt_bias=None, zoh_mode=0, h_init=None, want_dh_init=False,
                stream=None, ckpt=None):
    """Gradients of s6_scan_fwd for the loss sum(dy * y).  Returns a dict of float32
    tensors: du, ddt, dz (None without z) [Bt, L, d]; dB, dC [Bt, L, N]; dA_log [d, N];
    dD, ddt_bias (None without dt_bias) [d]; dh_init [Bt, d, N] (None unless wanted).
    ckpt: the checkpoints of s6_scan_fwd_ckpt on the same inputs (its h_init is
    in them, so h_init must then be None); the backward then skips its own forward."""
    torch = _torch()
    if u.dim() != 3:
        raise ValueError("u must be [batch, seqlen, d_inner]")
    Bt, L, d = u.shape
    N = A_log.shape[-1]
    dev = u.device
    f32 = torch.float32
    seq = (Bt, L, d)
    g = {"du": torch.empty(seq, dtype=f32, device=dev), "ddt": torch.empty(seq, dtype=f32, device=dev),
         "dz": torch.empty(seq, dtype=f32, device=dev) if z is not None else None,
         "dB": torch.empty((Bt, L, N), dtype=f32, device=dev), "dC": torch.empty((Bt, L, N), dtype=f32, device=dev),
         "dA_log": torch.empty((d, N), dtype=f32, device=dev), "dD": torch.empty((d,), dtype=f32, device=dev),
         "ddt_bias": torch.empty((d,), dtype=f32, device=dev) if dt_bias is not None else None,
         "dh_init": torch.empty((Bt, d, N), dtype=f32, device=dev) if want_dh_init else None}
    dims = Dims(Bt, L, d, N, 0, _io_code(u))
    io = u.dtype
    fn, start = _bwd_start(lib().s6_scan_bwd, lib().s6_scan_bwd_ckpt, h_init, ckpt, Bt, L, d, N, dev)
    st = fn(ctypes.byref(dims), _ptr(u, "u", io, seq, dev), _ptr(dt, "dt", io, seq, dev),
                           _ptr(A_log, "A_log", f32, (d, N), dev), _ptr(B, "B", io, (Bt, L, N), dev),
                           _ptr(C, "C", io, (Bt, L, N), dev), _ptr(D, "D", f32, (d,), dev),
                           _ptr(z, "z", io, seq, dev), _ptr(dt_bias, "dt_bias", f32, (d,), dev), int(zoh_mode),
                           start, _ptr(dy, "dy", io, seq, dev),
                           *[_ptr(g[k], k) for k in ("du", "ddt", "dz", "dB", "dC", "dA_log", "dD", "ddt_bias",
                                                     "dh_init")],
                           _stream(stream, dev))
    _check(st, fn.__name__)
    return g


def s6_conv_scan_bwd(x, conv_w, conv_b, dt, A_log, B, C, D, dy, z=None, dt_bias=None, zoh_mode=0, h_init=None,
                     want_dh_init=False, stream=None, ckpt=None):
    """Gradients of s6_conv_scan_fwd for the loss sum(dy * y).  Returns the dict of
    s6_scan_bwd with dx [Bt, L, d] in place of du, plus dconv_w [d, K] and dconv_b
    [d] (None without conv_b).  ckpt: the checkpoints of s6_conv_scan_fwd_ckpt on
    the same inputs (h_init must then be None)."""
    torch = _torch()
    if x.dim() != 3:
        raise ValueError("x must be [batch, seqlen, d_inner]")
    Bt, L, d = x.shape
    N = A_log.shape[-1]
    K = conv_w.shape[-1]
    dev = x.device
    f32 = torch.float32
    seq = (Bt, L, d)
    g = {"dx": torch.empty(seq, dtype=f32, device=dev),
         "dconv_w": torch.empty((d, K), dtype=f32, device=dev),
         "dconv_b": torch.empty((d,), dtype=f32, device=dev) if conv_b is not None else None,
         "ddt": torch.empty(seq, dtype=f32, device=dev),
         "dz": torch.empty(seq, dtype=f32, device=dev) if z is not None else None,
         "dB": torch.empty((Bt, L, N), dtype=f32, device=dev), "dC": torch.empty((Bt, L, N), dtype=f32, device=dev),
         "dA_log": torch.empty((d, N), dtype=f32, device=dev), "dD": torch.empty((d,), dtype=f32, device=dev),
         "ddt_bias": torch.empty((d,), dtype=f32, device=dev) if dt_bias is not None else None,
         "dh_init": torch.empty((Bt, d, N), dtype=f32, device=dev) if want_dh_init else None}
    dims = Dims(Bt, L, d, N, K, _io_code(x))
    io = x.dtype
    fn, start = _bwd_start(lib().s6_conv_scan_bwd, lib().s6_conv_scan_bwd_ckpt, h_init, ckpt, Bt, L, d, N, dev)
    st = fn(ctypes.byref(dims), _ptr(x, "x", io, seq, dev), _ptr(conv_w, "conv_w", f32, (d, K), dev),
                                _ptr(conv_b, "conv_b", f32, (d,), dev), _ptr(dt, "dt", io, seq, dev),
                                _ptr(A_log, "A_log", f32, (d, N), dev), _ptr(B, "B", io, (Bt, L, N), dev),
                                _ptr(C, "C", io, (Bt, L, N), dev), _ptr(D, "D", f32, (d,), dev),
                                _ptr(z, "z", io, seq, dev), _ptr(dt_bias, "dt_bias", f32, (d,), dev), int(zoh_mode),
                                start, _ptr(dy, "dy", io, seq, dev),
                                *[_ptr(g[k], k) for k in ("dx", "dconv_w", "dconv_b", "ddt", "dz", "dB", "dC",
                                                          "dA_log", "dD", "ddt_bias", "dh_init")],
                                _stream(stream, dev))
    _check(st, fn.__name__)
    return g


def causal_conv1d_silu_fwd(x, conv_w, conv_b=None, out=None, stream=None):
    """SiLU(causal depthwise conv(x)) over [batch, seqlen, d_inner]."""
    torch = _torch()
    Bt, L, d = x.shape
    K = conv_w.shape[-1]
    if out is None:
        out = torch.empty_like(x)
    dims = Dims(Bt, L, d, 1, K, _io_code(x))
    dev = x.device
    st = lib().causal_conv1d_silu_fwd(ctypes.byref(dims), _ptr(x, "x", x.dtype, (Bt, L, d), dev),
                                      _ptr(conv_w, "conv_w", torch.float32, (d, K), dev),
                                      _ptr(conv_b, "conv_b", torch.float32, (d,), dev),
                                      _ptr(out, "out", x.dtype, (Bt, L, d), dev), _stream(stream, dev))
    _check(st, "causal_conv1d_silu_fwd")
    return out


def s6_step(u_t, dt_t, B_t, C_t, A_log, D, conv_w, h_ssm, conv_state, z_t=None, dt_bias=None, conv_b=None,
            zoh_mode=0, y_t=None, stream=None):
    """One streaming token for a batch of sequences; h_ssm and conv_state are updated in place."""
    torch = _torch()
    Bt, d = u_t.shape
    N = A_log.shape[-1]
    K = conv_w.shape[-1]
    io = _io_code(u_t)
    dev = u_t.device
    if y_t is None:
        y_t = torch.empty_like(u_t)
    f32 = torch.float32
    dims = Dims(Bt, 1, d, N, K, io)
    st = lib().s6_step(ctypes.byref(dims), _ptr(A_log, "A_log", f32, (d, N), dev), _ptr(D, "D", f32, (d,), dev),
                       _ptr(dt_bias, "dt_bias", f32, (d,), dev), _ptr(conv_w, "conv_w", f32, (d, K), dev),
                       _ptr(conv_b, "conv_b", f32, (d,), dev), int(zoh_mode),
                       _ptr(u_t, "u_t", u_t.dtype, (Bt, d), dev), _ptr(dt_t, "dt_t", u_t.dtype, (Bt, d), dev),
                       _ptr(B_t, "B_t", u_t.dtype, (Bt, N), dev), _ptr(C_t, "C_t", u_t.dtype, (Bt, N), dev),
                       _ptr(z_t, "z_t", u_t.dtype, (Bt, d), dev), _ptr(h_ssm, "h_ssm", f32, (Bt, d, N), dev),
                       _ptr(conv_state, "conv_state", u_t.dtype, (Bt, d, K - 1), dev),
                       _ptr(y_t, "y_t", u_t.dtype, (Bt, d), dev), _stream(stream, dev))
    _check(st, "s6_step")
    return y_t


def s6_block_step(x, conv_state, h_ssm, w, eps=1e-5, stream=None):
    """One token through one decode block for every sequence of the batch:
    x [Bt, dm] (the residual stream, updated in place), conv_state [Bt, di, K-1]
    and h_ssm [Bt, di, N] (float32, in place); ``w`` a dict of the block's device
    weights (BLOCK_WEIGHT_KEYS: int8 rows *_q with float32 row scales *_s).  The
    weight structure is kept on the dict (key "_abi") for later calls."""
    torch = _torch()
    Bt, dm = x.shape
    di, N = w["A_log"].shape
    K = w["conv_w"].shape[1]
    R = w["dt_q"].shape[1]
    dev = x.device
    f32, i8 = torch.float32, torch.int8
    shapes = {"ln_w": ((dm,), f32), "ln_b": ((dm,), f32), "in_q": ((2 * di, dm), i8), "in_s": ((2 * di,), f32),
              "conv_w": ((di, K), f32), "conv_b": ((di,), f32), "xp_q": ((R + 2 * N, di), i8),
              "xp_s": ((R + 2 * N,), f32), "dt_q": ((di, R), i8), "dt_s": ((di,), f32), "dt_bias": ((di,), f32),
              "A_log": ((di, N), f32), "D": ((di,), f32), "out_q": ((dm, di), i8), "out_s": ((dm,), f32)}
    abi = w.get("_abi")
    if abi is None:
        abi = BlockWeights(*[_ptr(w.get(k), k, shapes[k][1], shapes[k][0], dev) for k in BLOCK_WEIGHT_KEYS])
        w["_abi"] = abi
    dims = BlockDims(Bt, dm, di, N, R, K, float(eps))
    st = lib().s6_block_step(ctypes.byref(dims), ctypes.byref(abi), _ptr(x, "x", f32, (Bt, dm), dev),
                             _ptr(conv_state, "conv_state", f32, (Bt, di, K - 1), dev),
                             _ptr(h_ssm, "h_ssm", f32, (Bt, di, N), dev), _stream(stream, dev))
    _check(st, "s6_block_step")
    return x


def s6_device_status(stream=None, device=None) -> int:
    """Synchronise and return (and clear) the library's device-side error status."""
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    return lib().s6_device_status(_stream(stream, dev))


def s6_debug_carry_fault(skip_publish_unit: int = -1, carry_polls: int = 0) -> None:
    """Test-only fault injection: unit `skip_publish_unit` of the next segmented
    scans publishes no carry and carry waits give up after `carry_polls` polls
    (0 = default).  ``s6_debug_carry_fault()`` switches it off again."""
    _check(lib().s6_debug_carry_fault(int(skip_publish_unit), int(carry_polls)), "s6_debug_carry_fault")
