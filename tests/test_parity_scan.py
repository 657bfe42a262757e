"""GPU parity of s6_scan_fwd / s6_conv_scan_fwd against the float64 oracle.

Every case draws seeded inputs (s6_inputs), runs the CUDA path through the C
ABI and the oracle on the same stored values, and checks y and h_final element
by element: max |got - ref| / (1 + |ref|) <= 1e-4 (float32 I/O) or 1e-2
(bfloat16 I/O, float32 state).
"""
import numpy as np
import pytest

from oracle import s6_oracle as O
import s6_inputs as SI
from s6_testutil import TOL, as_f64, assert_close, dev_inputs, from_dev, sample_channels

pytestmark = pytest.mark.gpu


def _gpu_scan(inp, zoh, fused=True, gate=True, bias=True, conv_b=True, want_h=True):
    import selective_state_space_19_b200 as S
    import torch
    t = dev_inputs(inp)
    if fused:
        y, h = S.s6_conv_scan_fwd(t["x"], t["conv_w"], t["conv_b"] if conv_b else None, t["dt"], t["A_log"], t["B"],
                                  t["C"], t["D"], z=t["z"] if gate else None, dt_bias=t["dt_bias"] if bias else None,
                                  zoh_mode=int(zoh), want_h_final=want_h)
    else:
        y, h = S.s6_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], z=t["z"] if gate else None,
                             dt_bias=t["dt_bias"] if bias else None, zoh_mode=int(zoh), want_h_final=want_h)
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    return from_dev(y), (h.cpu().numpy() if h is not None else None)


def _ref_scan(inp, zoh, fused=True, gate=True, bias=True, conv_b=True, channels=None):
    return O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"] if gate else None,
                  dt_bias=inp["dt_bias"] if bias else None, zoh=zoh, conv_w=inp["conv_w"] if fused else None,
                  conv_b=(inp["conv_b"] if conv_b else None) if fused else None, channels=channels)


def _check_full(inp, zoh, **kw):
    y, h = _gpu_scan(inp, zoh, **kw)
    ry, rh = _ref_scan(inp, zoh, **kw)
    io = inp["io"]
    ey = assert_close(as_f64(y), ry, io, "y")
    eh = assert_close(h, rh, io, "h_final")
    return ey, eh


# ------------------------------------------------------------ the named workloads
@pytest.mark.parametrize("zoh", [False, True])
def test_teaching_block(zoh):
    """TinyMamba teaching block: Bt1 L6 d8 N3, conv width 3, fp32; both write modes."""
    inp = SI.scan_inputs("teaching")
    _check_full(inp, zoh)


@pytest.mark.parametrize("zoh", [False, True])
def test_mamba_mini_block_full(zoh):
    """Mamba-mini block scan: Bt8 L256 d1536 N16 K4 fp32, every output element."""
    inp = SI.scan_inputs("mamba_mini")
    _check_full(inp, zoh)


def _check_full_size(name, zoh):
    """A workload at its full size: the GPU scan over the whole batch in one
    launch, every element of y and h_final against the oracle, computed
    sequence by sequence."""
    inp = SI.scan_inputs(name)
    y, h = _gpu_scan(inp, zoh)
    ey = eh = 0.0
    for b in range(inp["Bt"]):
        sl = slice(b, b + 1)
        sub = dict(inp, x=inp["x"][sl], z=inp["z"][sl], B=inp["B"][sl], C=inp["C"][sl], dt=inp["dt"][sl], Bt=1)
        ry, rh = _ref_scan(sub, zoh)
        ey = max(ey, assert_close(as_f64(y[b:b + 1]), ry, "bf16", f"{name} y"))
        eh = max(eh, assert_close(h[b:b + 1], rh, "bf16", f"{name} h_final"))
    return ey, eh


def test_long_seq_full_size():
    """Bt16 L8192 d1536 N16 K4 bf16 (simplified, fused conv + gate, h_final), the
    bench's workload in its launch configuration: every output element."""
    _check_full_size("long_seq", False)


def test_wide_full_size():
    """Bt4 L2048 d5120 N16 K4 bf16, exact ZOH, fused conv + gate: every output
    element."""
    _check_full_size("wide", True)


# ------------------------------------------------------------ shapes and options
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("L,d,N,K", [(1, 8, 16, 4), (37, 200, 16, 4), (50, 136, 3, 3), (70, 264, 8, 2),
                                     (33, 40, 1, 4), (129, 128, 12, 3), (16, 8, 5, 2)])
def test_ragged_shapes(io, zoh, L, d, N, K):
    """L not a multiple of the chunk, d not a multiple of the CTA tile, N below the
    register tile, every conv width."""
    inp = SI.scan_inputs("mamba_mini", Bt=3, L=L, d=d, N=N, K=K, io=io, seed=100 + L + d + N)
    _check_full(inp, zoh)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_unfused_scan(io):
    """s6_scan_fwd: u given directly (no conv)."""
    inp = SI.scan_inputs("mamba_mini", Bt=2, L=77, d=256, io=io, seed=7)
    _check_full(inp, False, fused=False)
    _check_full(inp, True, fused=False)


@pytest.mark.parametrize("gate,bias,conv_b", [(False, True, True), (True, False, True), (True, True, False),
                                              (False, False, False)])
def test_optional_inputs(gate, bias, conv_b):
    inp = SI.scan_inputs("mamba_mini", Bt=2, L=45, d=136, seed=8)
    _check_full(inp, False, gate=gate, bias=bias, conv_b=conv_b)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_random_A_log(io):
    """A_log drawn at random, so decays are not powers of one another."""
    inp = SI.scan_inputs("mamba_mini", Bt=2, L=300, d=256, io=io, seed=9, random_A=True)
    _check_full(inp, False)
    _check_full(inp, True)


def test_no_h_final():
    inp = SI.scan_inputs("mamba_mini", Bt=2, L=20, d=128, seed=10)
    y, h = _gpu_scan(inp, False, want_h=False)
    assert h is None
    ry, _ = _ref_scan(inp, False)
    assert_close(y, ry, "f32", "y")


def test_fused_equals_conv_then_scan():
    """The fused path equals causal_conv1d_silu_fwd then s6_scan_fwd, up to the
    rounding of the conv output to the I/O dtype (exact in float32 up to order)."""
    import selective_state_space_19_b200 as S
    import torch
    inp = SI.scan_inputs("mamba_mini", Bt=2, L=150, d=264, seed=11)
    t = dev_inputs(inp)
    y1, h1 = S.s6_conv_scan_fwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                                z=t["z"], dt_bias=t["dt_bias"])
    xc = S.causal_conv1d_silu_fwd(t["x"], t["conv_w"], t["conv_b"])
    y2, h2 = S.s6_scan_fwd(xc, t["dt"], t["A_log"], t["B"], t["C"], t["D"], z=t["z"], dt_bias=t["dt_bias"])
    torch.cuda.synchronize()
    assert torch.allclose(y1, y2, rtol=1e-5, atol=1e-6)
    assert torch.allclose(h1, h2, rtol=1e-5, atol=1e-6)


# ------------------------------------------------------------ edge cases
def test_empty_sequence_gives_zero_state():
    import selective_state_space_19_b200 as S
    import torch
    inp = SI.scan_inputs("mamba_mini", Bt=2, L=0, d=64, seed=12)
    t = dev_inputs(inp)
    h = torch.full((2, 64, 16), 7.0, device="cuda")
    y, h = S.s6_conv_scan_fwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                              z=t["z"], dt_bias=t["dt_bias"], h_final=h)
    torch.cuda.synchronize()
    assert y.numel() == 0
    assert torch.count_nonzero(h).item() == 0


def test_empty_batch_is_noop():
    import selective_state_space_19_b200 as S
    inp = SI.scan_inputs("mamba_mini", Bt=0, L=5, d=64, seed=13)
    t = dev_inputs(inp)
    y, h = S.s6_conv_scan_fwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                              z=t["z"], dt_bias=t["dt_bias"])
    assert y.numel() == 0 and h.numel() == 0


def test_rejects_bad_arguments():
    import selective_state_space_19_b200 as S
    import torch
    inp = SI.scan_inputs("mamba_mini", Bt=1, L=8, d=64, seed=14)
    t = dev_inputs(inp)
    # d * sizeof(float) not a multiple of 16 bytes
    with pytest.raises(S.S6Error) as e:
        S.s6_scan_fwd(t["x"][:, :, :62].contiguous(), t["dt"][:, :, :62].contiguous(), t["A_log"][:62].contiguous(),
                      t["B"], t["C"], t["D"][:62].contiguous())
    assert e.value.status == S.S6_ERR_ALIGNMENT
    # misaligned base pointer
    buf = torch.zeros(1 * 8 * 64 + 1, device="cuda")
    xm = buf[1:].view(1, 8, 64)
    with pytest.raises(S.S6Error) as e:
        S.s6_scan_fwd(xm, t["dt"], t["A_log"], t["B"], t["C"], t["D"])
    assert e.value.status == S.S6_ERR_ALIGNMENT
    # N > 16
    big = torch.zeros(64, 17, device="cuda")
    Bb = torch.zeros(1, 8, 17, device="cuda")
    with pytest.raises(S.S6Error) as e:
        S.s6_scan_fwd(t["x"], t["dt"], big, Bb, Bb, t["D"])
    assert e.value.status == S.S6_ERR_UNSUPPORTED
    # conv width 5
    w5 = torch.zeros(64, 5, device="cuda")
    with pytest.raises(S.S6Error) as e:
        S.s6_conv_scan_fwd(t["x"], w5, None, t["dt"], t["A_log"], t["B"], t["C"], t["D"])
    assert e.value.status == S.S6_ERR_UNSUPPORTED
    # zoh_mode outside {0, 1}
    with pytest.raises(S.S6Error) as e:
        S.s6_scan_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], zoh_mode=2)
    assert e.value.status == S.S6_ERR_INVALID_ARG
    assert S.s6_device_status() == 0


def test_tolerances_are_the_stated_ones():
    assert TOL == {"f32": 1e-4, "bf16": 1e-2}


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_static_schedule_many_chains(io):
    """Enough (sequence, channel-tile) chains that each CTA runs one whole chain
    (no carries between CTAs): sampled channels against the oracle."""
    inp = SI.scan_inputs("mamba_mini", Bt=96, L=70, d=2048, io=io, seed=15)
    y, h = _gpu_scan(inp, False)
    ch = sample_channels(inp["Bt"], inp["d"], 64, seed=3)
    ry, rh = _ref_scan(inp, False, channels=ch)
    assert_close(np.stack([as_f64(y[b, :, d]) for b, d in ch]), ry, io, "y")
    assert_close(np.stack([h[b, d] for b, d in ch]), rh, io, "h_final")


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("zoh", [False, True])
def test_long_chain_few_channels(io, zoh):
    """One sequence, few channels, a long sequence: the scan is split into many
    segments whose end states pass between CTAs; every output is compared."""
    inp = SI.scan_inputs("mamba_mini", Bt=1, L=5000, d=64, io=io, seed=16)
    _check_full(inp, zoh)


def test_repeated_calls_are_identical():
    """Dynamic scheduling hands units to CTAs in a different order each time;
    the result does not depend on it (bit-identical outputs)."""
    import selective_state_space_19_b200 as S
    import torch
    inp = SI.scan_inputs("long_seq", Bt=2, L=3000, d=512, seed=17)
    t = dev_inputs(inp)
    outs = []
    for _ in range(3):
        y, h = S.s6_conv_scan_fwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                                  z=t["z"], dt_bias=t["dt_bias"])
        outs.append((y.clone(), h.clone()))
    torch.cuda.synchronize()
    for y, h in outs[1:]:
        assert torch.equal(y, outs[0][0]) and torch.equal(h, outs[0][1])
