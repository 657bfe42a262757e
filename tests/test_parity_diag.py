"""GPU parity of s6_diag_recurrence_fwd against the float64 oracle.

The constant-decay cell ("the s6 cell", one cell, two architectures): per
state, h <- 2^w h + B_t u_t with w a per-(channel, state) constant, and the
readout of the S6 cell.  Compared element by element with oracle.diag_const
(y and h_final, max |got - ref| / (1 + |ref|)) over shapes that span several
chunks with a ragged tail, N = 3, 8, 16, with and without the gate and a start
state, and few enough channel tiles to take the associative split.  The
live-decay source must equal the selective scan.

Bound.  bfloat16 I/O: 1e-2, as for the scan.  float32 I/O: a constant decay a
keeps about 1/(1 - a) past writes in the state, and each float32 update
rounds the state by up to 2^-24 relative, so the state's relative error grows
to about 2 * 2^-24 / (1 - a); with the workload's decays up to 0.999 the bound
is taken as twice that, 4 * 2^-24 / (1 - 0.999) = 2.4e-4 (the scan's 1e-4
assumes memories of at most about 100 tokens).
"""
import numpy as np
import pytest

from oracle import s6_oracle as O
import s6_inputs as SI
from s6_testutil import as_f64, assert_close, dev_inputs, from_dev, note, rel_err, to_dev

pytestmark = pytest.mark.gpu

A_MAX = 0.999
TOL_F32 = 4 * 2.0 ** -24 / (1 - A_MAX)


def _close(got, ref, io, what):
    if io == "f32":
        err = rel_err(got, ref)
        note(f"{what} ({io})", err)
        assert err <= TOL_F32, f"{what}: max|got-ref|/(1+|ref|) = {err:.3e} > {TOL_F32:.1e}"
    else:
        assert_close(got, ref, io, what)


def _run(S, t, w, gate, h0=None):
    return S.s6_diag_recurrence_fwd(t["x"], t["B"], t["C"], t["D"], decay_source=S.S6_DECAY_CONST,
                                    log2_decay=w, z=t["z"] if gate else None, h_init=h0)


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("gate", [True, False])
@pytest.mark.parametrize("shape", [dict(Bt=8, L=300, d=1536, N=16),   # 192 channel tiles: no associative split
                                   dict(Bt=2, L=1000, d=136, N=16),   # associative split, ragged d
                                   dict(Bt=3, L=77, d=264, N=8),
                                   dict(Bt=2, L=70, d=40, N=3)])
def test_diag_const_matches_oracle(io, gate, shape):
    import selective_state_space_19_b200 as S
    import torch
    inp = SI.scan_inputs("mamba_mini", io=io, K=4, seed=shape["L"] + shape["d"], **shape)
    w = SI.diag_log2_decay(shape["d"], shape["N"])
    t = dev_inputs(inp)
    y, h = _run(S, t, to_dev(w), gate)
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    ry, rh = O.diag_const(inp["x"], w, inp["B"], inp["C"], inp["D"], z=inp["z"] if gate else None)
    _close(as_f64(from_dev(y)), ry, io, "diag y")
    _close(h.cpu().numpy(), rh, io, "diag h_final")


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_diag_const_from_state(io):
    import selective_state_space_19_b200 as S
    import torch
    Bt, L, d, N = 2, 600, 256, 16
    inp = SI.scan_inputs("mamba_mini", Bt=Bt, L=L, d=d, N=N, K=4, io=io, seed=81)
    w = SI.diag_log2_decay(d, N)
    h0 = np.random.default_rng(82).standard_normal((Bt, d, N)).astype(np.float32)
    t = dev_inputs(inp)
    y, h = _run(S, t, to_dev(w), True, to_dev(h0))
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    ry, rh = O.diag_const(inp["x"], w, inp["B"], inp["C"], inp["D"], z=inp["z"], h_init=h0)
    _close(as_f64(from_dev(y)), ry, io, "diag y")
    _close(h.cpu().numpy(), rh, io, "diag h_final")


def test_diag_const_long_seq_shape_full():
    """The long-sequence workload's shape (Bt16 L8192 d1536 N16, bf16) with
    constant decays, as the bench row runs it: every output element, the oracle
    sequence by sequence."""
    import selective_state_space_19_b200 as S
    import torch
    inp = SI.scan_inputs("long_seq", seed=83)
    w = SI.diag_log2_decay(1536, 16)
    t = dev_inputs(inp)
    y, h = _run(S, t, to_dev(w), True)
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    yg, hg = as_f64(from_dev(y)), h.cpu().numpy()
    for b in range(inp["Bt"]):
        sl = slice(b, b + 1)
        ry, rh = O.diag_const(inp["x"][sl], w, inp["B"][sl], inp["C"][sl], inp["D"], z=inp["z"][sl])
        assert_close(yg[sl], ry, "bf16", "diag full long-seq y")
        assert_close(hg[sl], rh, "bf16", "diag full long-seq h_final")


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_diag_live_source_is_the_selective_scan(io):
    import selective_state_space_19_b200 as S
    import torch
    inp = SI.scan_inputs("mamba_mini", Bt=2, L=200, d=128, N=16, io=io, seed=85)
    t = dev_inputs(inp)
    y, h = S.s6_diag_recurrence_fwd(t["x"], t["B"], t["C"], t["D"], decay_source=S.S6_DECAY_LIVE, dt=t["dt"],
                                    A_log=t["A_log"], dt_bias=t["dt_bias"], z=t["z"])
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    ry, rh = O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"],
                    dt_bias=inp["dt_bias"])
    assert_close(as_f64(from_dev(y)), ry, io, "diag live y")
    assert_close(h.cpu().numpy(), rh, io, "diag live h_final")


def test_diag_rejects_bad_arguments():
    import selective_state_space_19_b200 as S
    import torch
    u = torch.zeros(1, 8, 64, device="cuda")
    Bm = torch.zeros(1, 8, 16, device="cuda")
    Dv = torch.zeros(64, device="cuda")
    w = torch.zeros(64, 16, device="cuda")
    with pytest.raises(S.S6Error) as e:
        S.s6_diag_recurrence_fwd(u, Bm, Bm, Dv, decay_source=7, log2_decay=w)
    assert e.value.status == S.S6_ERR_INVALID_ARG
    with pytest.raises(S.S6Error) as e:  # live decay without dt
        S.s6_diag_recurrence_fwd(u, Bm, Bm, Dv, decay_source=S.S6_DECAY_LIVE, A_log=w)
    assert e.value.status == S.S6_ERR_INVALID_ARG
