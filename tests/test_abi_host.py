"""CPU-only checks of the boundary: the library builds for sm_100a, loads without
a GPU, exports every function include/s6.h declares, and rejects bad arguments
on the host before touching the device.  No compute call is made here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "s6.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = "\n".join(l for l in src.splitlines() if not l.lstrip().startswith("#"))
    return re.findall(r"S6_API\s+(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", src)


@pytest.fixture(scope="module")
def lib():
    from selective_state_space_19_b200 import _build
    import selective_state_space_19_b200 as S
    _build.build()
    return S.lib()


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"s6_scan_fwd", "s6_conv_scan_fwd", "causal_conv1d_silu_fwd", "s6_step", "s6_status_string",
            "s6_device_status", "s6_version"} <= names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_library_is_built_for_sm100a_only():
    from selective_state_space_19_b200 import _build
    flags = " ".join(_build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert "sm_90" not in flags and "sm_80" not in flags


def test_status_strings(lib):
    import selective_state_space_19_b200 as S
    for st in (S.S6_OK, S.S6_ERR_INVALID_ARG, S.S6_ERR_UNSUPPORTED, S.S6_ERR_ALIGNMENT, S.S6_ERR_CUDA,
               S.S6_ERR_TIMEOUT):
        assert S.s6_status_string(st).startswith("S6_")
    assert "unknown" in S.s6_status_string(12345)
    assert S.s6_version() >> 16 == 1


def _dims(**kw):
    import selective_state_space_19_b200 as S
    d = dict(batch=2, seqlen=8, d_inner=64, d_state=16, conv_width=4, io_dtype=0)
    d.update(kw)
    return S.Dims(**d)


def _call_scan(lib, dims, **ptrs):
    P = ctypes.c_void_p
    args = dict(u=16, dt=16, A_log=16, B=16, C=16, D=16, z=None, dt_bias=None, zoh=0, y=16, h=None)
    args.update(ptrs)
    return lib.s6_scan_fwd(ctypes.byref(dims) if dims is not None else None, P(args["u"]), P(args["dt"]),
                           P(args["A_log"]), P(args["B"]), P(args["C"]), P(args["D"]), P(args["z"]),
                           P(args["dt_bias"]), args["zoh"], P(args["y"]), P(args["h"]), None)


def test_host_checks_reject_before_any_launch(lib):
    import selective_state_space_19_b200 as S
    assert _call_scan(lib, None) == S.S6_ERR_INVALID_ARG
    assert _call_scan(lib, _dims(d_state=17)) == S.S6_ERR_UNSUPPORTED
    assert _call_scan(lib, _dims(d_state=0)) == S.S6_ERR_INVALID_ARG
    assert _call_scan(lib, _dims(io_dtype=7)) == S.S6_ERR_UNSUPPORTED
    assert _call_scan(lib, _dims(batch=-1)) == S.S6_ERR_INVALID_ARG
    assert _call_scan(lib, _dims(), u=None) == S.S6_ERR_INVALID_ARG
    assert _call_scan(lib, _dims(), zoh=3) == S.S6_ERR_INVALID_ARG
    assert _call_scan(lib, _dims(d_inner=62)) == S.S6_ERR_ALIGNMENT          # 62*4 B rows
    assert _call_scan(lib, _dims(d_inner=60, io_dtype=1)) == S.S6_ERR_ALIGNMENT  # 60*2 B rows
    assert _call_scan(lib, _dims(), dt=24) == S.S6_ERR_ALIGNMENT
    # empty work is accepted and does nothing (no pointer is touched)
    assert _call_scan(lib, _dims(batch=0), u=None, dt=None, y=None) == S.S6_OK
    assert _call_scan(lib, _dims(seqlen=0), u=None, dt=None, y=None) == S.S6_OK


def test_conv_and_step_host_checks(lib):
    import selective_state_space_19_b200 as S
    P = ctypes.c_void_p
    d = _dims(conv_width=5)
    assert lib.causal_conv1d_silu_fwd(ctypes.byref(d), P(16), P(16), None, P(16), None) == S.S6_ERR_UNSUPPORTED
    d = _dims(conv_width=1)
    assert lib.causal_conv1d_silu_fwd(ctypes.byref(d), P(16), P(16), None, P(16), None) == S.S6_ERR_UNSUPPORTED
    d = _dims()
    assert lib.causal_conv1d_silu_fwd(ctypes.byref(d), None, P(16), None, P(16), None) == S.S6_ERR_INVALID_ARG
    ok = [P(16)] * 5
    assert lib.s6_step(ctypes.byref(_dims()), *ok, 0, None, *[P(16)] * 3, None, P(16), P(16), P(16),
                       None) == S.S6_ERR_INVALID_ARG
    assert lib.s6_step(ctypes.byref(_dims()), *ok, 2, *[P(16)] * 4, None, P(16), P(16), P(16),
                       None) == S.S6_ERR_INVALID_ARG
    assert lib.s6_step(ctypes.byref(_dims(d_state=20)), *ok, 0, *[P(16)] * 4, None, P(16), P(16), P(16),
                       None) == S.S6_ERR_UNSUPPORTED
    assert lib.s6_step(ctypes.byref(_dims()), *ok, 0, *[P(16)] * 4, None, P(20), P(16), P(16),
                       None) == S.S6_ERR_ALIGNMENT


def test_from_state_and_backward_host_checks(lib):
    import selective_state_space_19_b200 as S
    P = ctypes.c_void_p
    d = ctypes.byref(_dims())
    ok = P(16)

    def fs(zoh=0, h_init=ok, hist=ok):  # s6_conv_scan_fwd_from_state
        return lib.s6_conv_scan_fwd_from_state(d, ok, ok, None, ok, ok, ok, ok, ok, None, None, zoh, h_init, hist,
                                               ok, None, None)
    assert fs(zoh=2) == S.S6_ERR_INVALID_ARG
    assert fs(h_init=P(18)) == S.S6_ERR_ALIGNMENT   # float32 start state
    assert fs(hist=P(18)) == S.S6_ERR_ALIGNMENT     # float32 I/O conv history
    assert lib.s6_scan_fwd_from_state(d, ok, ok, ok, ok, ok, ok, None, None, 0, P(2), ok, None,
                                      None) == S.S6_ERR_ALIGNMENT

    def bwd(zoh=0, **kw):  # s6_scan_bwd
        a = dict(u=ok, dt=ok, A_log=ok, B=ok, C=ok, D=ok, z=None, dt_bias=None, h_init=None, dy=ok, du=ok,
                 ddt=ok, dz=None, dB=ok, dC=ok, dA_log=ok, dD=ok, ddt_bias=None, dh_init=None)
        a.update(kw)
        return lib.s6_scan_bwd(kw.pop("dims", d), a["u"], a["dt"], a["A_log"], a["B"], a["C"], a["D"], a["z"],
                               a["dt_bias"], zoh, a["h_init"], a["dy"], a["du"], a["ddt"], a["dz"], a["dB"],
                               a["dC"], a["dA_log"], a["dD"], a["ddt_bias"], a["dh_init"], None)
    assert bwd(zoh=5) == S.S6_ERR_INVALID_ARG
    assert bwd(dy=None) == S.S6_ERR_INVALID_ARG
    assert bwd(dB=None) == S.S6_ERR_INVALID_ARG
    assert bwd(z=ok) == S.S6_ERR_INVALID_ARG        # a gate needs dz
    assert bwd(u=P(18)) == S.S6_ERR_ALIGNMENT
    assert bwd(dA_log=P(2)) == S.S6_ERR_ALIGNMENT
    assert bwd(dims=ctypes.byref(_dims(d_state=17))) == S.S6_ERR_UNSUPPORTED
    assert bwd(dims=ctypes.byref(_dims(batch=0))) == S.S6_OK  # nothing to do, nothing touched

    def cbwd(dims=d, conv_w=ok, dconv_w=ok):  # s6_conv_scan_bwd
        return lib.s6_conv_scan_bwd(dims, ok, conv_w, None, ok, ok, ok, ok, ok, None, None, 0, None, ok, ok,
                                    dconv_w, None, ok, None, ok, ok, ok, ok, None, None, None)
    assert cbwd(dims=ctypes.byref(_dims(conv_width=5))) == S.S6_ERR_UNSUPPORTED
    assert cbwd(conv_w=None) == S.S6_ERR_INVALID_ARG
    assert cbwd(dconv_w=None) == S.S6_ERR_INVALID_ARG
    assert cbwd(conv_w=P(2)) == S.S6_ERR_ALIGNMENT


def test_training_forward_and_backward_host_checks(lib):
    """The checkpoint calls: N = 16 only, a checkpoint buffer that must be given
    and 16-byte aligned, and the pipelined backward's row alignment -- all
    refused before anything reaches the device."""
    import selective_state_space_19_b200 as S
    P = ctypes.c_void_p
    ok = P(16)

    def fwd(dims=None, zoh=0, ckpt=ok):  # s6_scan_fwd_ckpt
        dd = ctypes.byref(dims or _dims())
        return lib.s6_scan_fwd_ckpt(dd, ok, ok, ok, ok, ok, ok, None, None, zoh, None, ok, None, ckpt, None)
    assert fwd(zoh=3) == S.S6_ERR_INVALID_ARG
    assert fwd(dims=_dims(d_state=8)) == S.S6_ERR_UNSUPPORTED
    assert fwd(ckpt=None) == S.S6_ERR_INVALID_ARG
    assert fwd(ckpt=P(8)) == S.S6_ERR_ALIGNMENT
    assert fwd(dims=_dims(batch=0), ckpt=None) == S.S6_OK  # nothing to do, nothing touched

    def cfwd(ckpt=ok, conv_w=ok):  # s6_conv_scan_fwd_ckpt
        return lib.s6_conv_scan_fwd_ckpt(ctypes.byref(_dims()), ok, conv_w, None, ok, ok, ok, ok, ok, None, None,
                                         0, None, ok, None, ckpt, None)
    assert cfwd(ckpt=P(4)) == S.S6_ERR_ALIGNMENT
    assert cfwd(conv_w=None) == S.S6_ERR_INVALID_ARG

    def bwd(dims=None, ckpt=ok, u=ok):  # s6_scan_bwd_ckpt
        dd = ctypes.byref(dims or _dims())
        return lib.s6_scan_bwd_ckpt(dd, u, ok, ok, ok, ok, ok, None, None, 0, ckpt, ok, ok, ok, None, ok, ok, ok,
                                    ok, None, None, None)
    assert bwd(ckpt=None) == S.S6_ERR_INVALID_ARG
    assert bwd(dims=_dims(d_state=8)) == S.S6_ERR_UNSUPPORTED
    assert bwd(ckpt=P(8)) == S.S6_ERR_ALIGNMENT
    assert bwd(u=P(4)) == S.S6_ERR_ALIGNMENT               # rows the tensor unit moves
    assert bwd(dims=_dims(d_inner=66)) == S.S6_ERR_ALIGNMENT  # 66 float32 is not a whole number of 16 bytes

    def cbwd(ckpt=ok):  # s6_conv_scan_bwd_ckpt
        return lib.s6_conv_scan_bwd_ckpt(ctypes.byref(_dims()), ok, ok, None, ok, ok, ok, ok, ok, None, None, 0,
                                         ckpt, ok, ok, ok, None, ok, None, ok, ok, ok, ok, None, None, None)
    assert cbwd(ckpt=None) == S.S6_ERR_INVALID_ARG
    assert cbwd(ckpt=P(24)) == S.S6_ERR_ALIGNMENT


def test_diag_and_block_host_checks(lib):
    """The constant-decay cell and the decode block reject bad arguments before
    any device call."""
    import selective_state_space_19_b200 as S
    P = ctypes.c_void_p
    ok = P(16)

    def diag(src=S.S6_DECAY_CONST, dims=None, w=ok):
        return lib.s6_diag_recurrence_fwd(ctypes.byref(dims or _dims()), src, ok, None, None, None, w, ok, ok, ok,
                                          None, None, ok, None, None)
    assert diag(src=5) == S.S6_ERR_INVALID_ARG
    assert diag(w=None) == S.S6_ERR_INVALID_ARG                       # the decays are required
    assert diag(dims=_dims(d_state=17)) == S.S6_ERR_UNSUPPORTED
    assert diag(w=P(2)) == S.S6_ERR_ALIGNMENT                         # float32 decays
    assert diag(dims=_dims(batch=0)) == S.S6_OK

    def block(**over):
        dims = dict(batch=4, d_model=64, d_inner=128, d_state=16, dt_rank=8, conv_width=4, eps=1e-5)
        ptrs = {k: 16 for k in S.BLOCK_WEIGHT_KEYS}
        ptrs["conv_b"] = None
        x = over.pop("x", 16)
        for k in list(over):
            if k in ptrs:
                ptrs[k] = over.pop(k)
        dims.update(over)
        w = S.BlockWeights(**{k: v for k, v in ptrs.items()})
        return lib.s6_block_step(ctypes.byref(S.BlockDims(**dims)), ctypes.byref(w), P(x), ok, ok, None)
    assert lib.s6_block_step(None, None, ok, ok, ok, None) == S.S6_ERR_INVALID_ARG
    assert block(d_state=17) == S.S6_ERR_UNSUPPORTED
    assert block(conv_width=5) == S.S6_ERR_UNSUPPORTED
    assert block(dt_rank=0) == S.S6_ERR_INVALID_ARG
    assert block(eps=float("nan")) == S.S6_ERR_INVALID_ARG
    assert block(in_q=None) == S.S6_ERR_INVALID_ARG                   # every weight but conv_b is required
    assert block(x=None) == S.S6_ERR_INVALID_ARG
    assert block(A_log=20) == S.S6_ERR_ALIGNMENT                      # N = 16 rows move as 16-byte vectors
    assert block(ln_w=2) == S.S6_ERR_ALIGNMENT
    assert block(batch=0) == S.S6_OK                                  # nothing to do, nothing touched


def test_binding_refuses_cpu_tensors(lib):
    import torch
    import selective_state_space_19_b200 as S
    x = torch.zeros(1, 4, 8)
    with pytest.raises(ValueError):
        S.s6_scan_fwd(x, x, torch.zeros(8, 3), torch.zeros(1, 4, 3), torch.zeros(1, 4, 3), torch.zeros(8))


def test_product_path_does_not_use_the_oracle():
    """The package, its C sources and the header never refer to the oracle."""
    pkg = os.path.join(ROOT, "selective_state_space_19_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in txt.lower(), f
    assert "oracle" not in open(HEADER).read().lower()
