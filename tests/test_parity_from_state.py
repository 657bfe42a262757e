"""GPU parity of s6_scan_fwd_from_state / s6_conv_scan_fwd_from_state against the
float64 oracle: a scan that starts from a given state (h_init and the K-1 conv
inputs before token 0) instead of zeros.

The oracle takes the same start state directly; the chunked-prefill checks also
compare against one oracle scan over the whole sequence, which pins the state
handed from one chunk to the next ("token streaming ... matches the full
forward").  Cases cover both I/O types and both write modes, the static and
the segmented schedules, a chunk boundary that is not a multiple of the
kernel's chunk, ragged channel tiles, K = 2, N = 3 and N = 8, and L = 0.
"""
import numpy as np
import pytest

from oracle import s6_oracle as O
import s6_inputs as SI
from s6_testutil import as_f64, assert_close, dev_inputs, from_dev, to_dev

pytestmark = pytest.mark.gpu


def _start_state(Bt, d, N, K, io, seed):
    rng = np.random.default_rng(seed)
    h0 = rng.standard_normal((Bt, d, N)).astype(np.float32)
    hist = SI.to_storage(rng.standard_normal((Bt, d, K - 1)).astype(np.float32), io)
    return h0, hist


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("shape", [dict(Bt=3, L=150, d=200, N=16, K=4),   # static schedule, ragged tile
                                   dict(Bt=1, L=2100, d=64, N=16, K=4),   # segmented schedule
                                   dict(Bt=2, L=70, d=72, N=8, K=2),
                                   dict(Bt=2, L=33, d=40, N=3, K=3)])
def test_fused_from_given_state(io, zoh, shape):
    """Random h_init and conv history: y and h_final equal the oracle started from
    the same state."""
    import selective_state_space_19_b200 as S
    Bt, L, d, N, K = (shape[k] for k in ("Bt", "L", "d", "N", "K"))
    inp = SI.scan_inputs("mamba_mini", io=io, seed=90 + L, **shape)
    h0, hist = _start_state(Bt, d, N, K, io, seed=L)
    ry, rh = O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"],
                    dt_bias=inp["dt_bias"], zoh=zoh, conv_w=inp["conv_w"], conv_b=inp["conv_b"],
                    h_init=h0, conv_hist=hist)
    t = dev_inputs(inp)
    y, h = S.s6_conv_scan_fwd_from_state(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"],
                                         t["D"], z=t["z"], dt_bias=t["dt_bias"], zoh_mode=int(zoh),
                                         h_init=to_dev(h0), conv_hist=to_dev(hist))
    assert S.s6_device_status() == 0
    assert_close(as_f64(from_dev(y)), ry, io, "y")
    assert_close(h.cpu().numpy(), rh, io, "h_final")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_unfused_from_given_state(io):
    """s6_scan_fwd_from_state (no conv): y and h_final equal the oracle from h_init."""
    import selective_state_space_19_b200 as S
    Bt, L, d, N = 2, 300, 136, 16
    inp = SI.scan_inputs("mamba_mini", Bt=Bt, L=L, d=d, N=N, io=io, seed=61)
    h0, _ = _start_state(Bt, d, N, 2, io, seed=62)
    ry, rh = O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"],
                    dt_bias=inp["dt_bias"], h_init=h0)
    t = dev_inputs(inp)
    y, h = S.s6_scan_fwd_from_state(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], z=t["z"],
                                    dt_bias=t["dt_bias"], h_init=to_dev(h0))
    assert S.s6_device_status() == 0
    assert_close(as_f64(from_dev(y)), ry, io, "y")
    assert_close(h.cpu().numpy(), rh, io, "h_final")


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("Bt,d,cuts", [(4, 192, (77, 200, 333)),     # static schedule
                                       (1, 64, (1000, 2222, 3001))])  # segmented schedule
def test_chunked_prefill_equals_one_scan(io, Bt, d, cuts):
    """Prefill in chunks, each from the previous chunk's h_final and its last K-1
    inputs, equals one oracle scan over the whole sequence."""
    import selective_state_space_19_b200 as S
    import torch
    L, N, K = cuts[-1], 16, 4
    inp = SI.scan_inputs("mamba_mini", Bt=Bt, L=L, d=d, N=N, K=K, io=io, seed=cuts[0])
    ry, rh = O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"],
                    dt_bias=inp["dt_bias"], conv_w=inp["conv_w"], conv_b=inp["conv_b"])
    t = dev_inputs(inp)
    h, hist, ys, lo = None, None, [], 0
    for hi in cuts:
        part = {k: t[k][:, lo:hi].contiguous() for k in ("x", "dt", "z", "B", "C")}
        y, h = S.s6_conv_scan_fwd_from_state(part["x"], t["conv_w"], t["conv_b"], part["dt"], t["A_log"],
                                             part["B"], part["C"], t["D"], z=part["z"], dt_bias=t["dt_bias"],
                                             h_init=h, conv_hist=hist)
        hist = t["x"][:, hi - (K - 1):hi].transpose(1, 2).contiguous()  # [Bt, d, K-1], oldest first
        ys.append(from_dev(y))
        lo = hi
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    assert_close(np.concatenate([as_f64(v) for v in ys], axis=1), ry, io, "y")
    assert_close(h.cpu().numpy(), rh, io, "h_final")


def test_chunked_prefill_full_long_seq_workload():
    """The bench's chunked-prefill row: the long-sequence workload in full
    (Bt16 L8192 d1536 bf16) in four 2048-token parts, each from the previous
    part's state and conv history, against one oracle scan per sequence: every
    element of y and the final state."""
    import selective_state_space_19_b200 as S
    import torch
    inp = SI.scan_inputs("long_seq")
    Bt, L, K = inp["Bt"], inp["L"], inp["K"]
    t = dev_inputs(inp)
    h, hist, ys = None, None, []
    cuts = [L * i // 4 for i in range(5)]
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        part = {k: t[k][:, lo:hi].contiguous() for k in ("x", "dt", "z", "B", "C")}
        y, h = S.s6_conv_scan_fwd_from_state(part["x"], t["conv_w"], t["conv_b"], part["dt"], t["A_log"],
                                             part["B"], part["C"], t["D"], z=part["z"], dt_bias=t["dt_bias"],
                                             h_init=h, conv_hist=hist)
        hist = t["x"][:, hi - (K - 1):hi].transpose(1, 2).contiguous()
        ys.append(from_dev(y))
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    hg = h.cpu().numpy()
    for b in range(Bt):
        sl = slice(b, b + 1)
        ry, rh = O.scan(inp["x"][sl], inp["dt"][sl], inp["A_log"], inp["B"][sl], inp["C"][sl], inp["D"],
                        z=inp["z"][sl], dt_bias=inp["dt_bias"], conv_w=inp["conv_w"], conv_b=inp["conv_b"])
        yb = np.concatenate([as_f64(v[b:b + 1]) for v in ys], axis=1)
        assert_close(yb, ry, "bf16", "prefill full long-seq y")
        assert_close(hg[b:b + 1], rh, "bf16", "prefill full long-seq h_final")


def test_empty_sequence_returns_the_start_state():
    import selective_state_space_19_b200 as S
    import torch
    Bt, d, N, K = 2, 64, 16, 4
    inp = SI.scan_inputs("mamba_mini", Bt=Bt, L=1, d=d, N=N, K=K, io="f32", seed=3)
    t = dev_inputs(inp)
    empty = {k: t[k][:, :0].contiguous() for k in ("x", "dt", "z", "B", "C")}
    h0 = torch.randn(Bt, d, N, device="cuda")
    hf = torch.full((Bt, d, N), 7.0, device="cuda")
    S.s6_conv_scan_fwd_from_state(empty["x"], t["conv_w"], t["conv_b"], empty["dt"], t["A_log"], empty["B"],
                                  empty["C"], t["D"], z=empty["z"], dt_bias=t["dt_bias"], h_init=h0, h_final=hf)
    torch.cuda.synchronize()
    assert torch.equal(hf, h0)
