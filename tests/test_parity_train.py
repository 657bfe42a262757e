"""GPU parity of the training path against the float64 oracle.

The training forwards (s6_scan_fwd_ckpt, s6_conv_scan_fwd_ckpt) return y and
h_final like the other forwards and also keep the state before every 16th
token; the backwards given those states skip their own forward.  The pages
single out the recurrence as what makes training slow ("Carry context through
a selective state", About this example).

- y and h_final are compared with oracle.scan (1e-4 float32, 1e-2 bfloat16
  outputs; states 1e-4).
- Each kept state ckpt[b, k] is compared with the oracle's state after the
  first 16 k tokens, i.e. the h_final of oracle.scan on that prefix (the start
  state at k = 0).
- The gradients are compared with oracle.scan_bwd / oracle.conv_scan_bwd at
  the backward's bound, 2e-3.

The shapes have a ragged last group of 16 tokens, a start state, and one long
sequence that takes the forward's associative split.
"""
import numpy as np
import pytest

from oracle import s6_oracle as O
import s6_inputs as SI
from s6_testutil import TOL, dev_inputs, note, rel_err, to_dev

pytestmark = pytest.mark.gpu

GTOL = 2e-3
EVERY = 16


def _inputs(io, Bt, L, d, seed, K=4):
    inp = SI.scan_inputs("mamba_mini", Bt=Bt, L=L, d=d, N=16, K=K, io=io, seed=seed)
    rng = np.random.default_rng(seed + 1)
    dy = SI.to_storage(rng.standard_normal((Bt, L, d)).astype(np.float32), io)
    h0 = rng.standard_normal((Bt, d, 16)).astype(np.float32)
    return inp, dy, h0


def _oracle_fwd(inp, conv, zoh, h0, upto=None):
    sl = slice(None) if upto is None else slice(0, upto)
    kw = dict(z=inp["z"][:, sl], dt_bias=inp["dt_bias"], zoh=zoh, h_init=h0)
    if conv:
        kw.update(conv_w=inp["conv_w"], conv_b=inp["conv_b"])
    return O.scan(inp["x"][:, sl], inp["dt"][:, sl], inp["A_log"], inp["B"][:, sl], inp["C"][:, sl], inp["D"], **kw)


def _train_fwd(S, t, conv, zoh, h0d):
    if conv:
        return S.s6_conv_scan_fwd_ckpt(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"],
                                       t["D"], z=t["z"], dt_bias=t["dt_bias"], zoh_mode=int(zoh), h_init=h0d)
    return S.s6_scan_fwd_ckpt(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], z=t["z"], dt_bias=t["dt_bias"],
                              zoh_mode=int(zoh), h_init=h0d)


def _check_forward(io, inp, conv, zoh, h0, y, h, ck, ks):
    ry, rh = _oracle_fwd(inp, conv, zoh, h0)
    err_y = rel_err(y.float().cpu().numpy(), ry)
    err_h = rel_err(h.cpu().numpy(), rh)
    note(f"train fwd y ({io})", err_y)
    assert err_y <= TOL[io], err_y
    assert err_h <= 1e-4, err_h
    ckn = ck.cpu().numpy()
    L = inp["x"].shape[1]
    assert ckn.shape[1] == (L + EVERY - 1) // EVERY
    for k in ks:
        ref = h0.astype(np.float64) if k == 0 else _oracle_fwd(inp, conv, zoh, h0, upto=EVERY * k)[1]
        err = rel_err(ckn[:, k], ref)
        note(f"train fwd checkpoint ({io})", err)
        assert err <= 1e-4, (k, err)


def _check_grads(io, got, ref, keys, what):
    for k in keys:
        g = got[k].cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(g)), k
        err = rel_err(g, ref[k])
        note(f"train grad {k} ({io})", err)
        assert err <= GTOL, f"{what} {k}: max|g-ref|/(1+|ref|) = {err:.3e}"


def _train_case(io, zoh, conv, Bt, L, d, seed):
    """Forward with checkpoints, then the backward from them: y, h_final, every
    kept state and every gradient against the oracle (with a start state)."""
    import torch
    import selective_state_space_19_b200 as S
    inp, dy, h0 = _inputs(io, Bt, L, d, seed=seed)
    t = dev_inputs(inp)
    y, h, ck = _train_fwd(S, t, conv, zoh, to_dev(h0))
    torch.cuda.synchronize()
    _check_forward(io, inp, conv, zoh, h0, y, h, ck, ks=range((L + EVERY - 1) // EVERY))
    if conv:
        got = S.s6_conv_scan_bwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                                 to_dev(dy), z=t["z"], dt_bias=t["dt_bias"], zoh_mode=int(zoh), ckpt=ck,
                                 want_dh_init=True)
        ref = O.conv_scan_bwd(inp["x"], inp["conv_w"], inp["conv_b"], inp["dt"], inp["A_log"], inp["B"], inp["C"],
                              inp["D"], dy, z=inp["z"], dt_bias=inp["dt_bias"], zoh=zoh, h_init=h0)
        keys = ("dx", "dconv_w", "dconv_b", "ddt", "dz", "dB", "dC", "dA_log", "dD", "ddt_bias", "dh_init")
    else:
        got = S.s6_scan_bwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], to_dev(dy), z=t["z"],
                            dt_bias=t["dt_bias"], zoh_mode=int(zoh), ckpt=ck, want_dh_init=True)
        ref = O.scan_bwd(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], dy, z=inp["z"],
                         dt_bias=inp["dt_bias"], zoh=zoh, h_init=h0)
        keys = ("du", "ddt", "dz", "dB", "dC", "dA_log", "dD", "ddt_bias", "dh_init")
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    _check_grads(io, got, ref, keys, f"io={io} zoh={zoh} conv={conv} Bt={Bt} L={L} d={d}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("conv", [False, True])
def test_train_step_matches_oracle(io, zoh, conv):
    """Bt 2, L 150 (the last group of 16 tokens holds 6), 64 channels."""
    _train_case(io, zoh, conv, Bt=2, L=150, d=64, seed=170 + 2 * int(zoh) + int(conv))


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [dict(Bt=3, L=17, d=40, zoh=True, conv=True),     # a tile of 40 channels
                                   dict(Bt=1, L=1, d=72, zoh=False, conv=False),     # one token, a ragged tile
                                   dict(Bt=2, L=16, d=136, zoh=False, conv=True)])   # exactly one group
def test_train_step_ragged_shapes(io, shape):
    sh = dict(shape)
    _train_case(io, sh.pop("zoh"), sh.pop("conv"), seed=200 + sh["L"] + sh["d"], **sh)


def test_train_forward_empty_sequence():
    """L = 0: no checkpoints, h_final is the start state."""
    import torch
    import selective_state_space_19_b200 as S
    inp, _, h0 = _inputs("f32", 2, 0, 64, seed=5)
    t = dev_inputs(inp)
    y, h, ck = _train_fwd(S, t, True, False, to_dev(h0))
    torch.cuda.synchronize()
    assert tuple(ck.shape) == (2, 0, 64, 16) and y.numel() == 0
    assert np.array_equal(h.cpu().numpy(), h0)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_train_step_associative_split(io):
    """One 4096-token sequence of 128 channels: two chains, so the training
    forward takes the associative split (segments scanned from zero, then run
    again from their folded start states, the checkpoints kept on that second
    pass); the backward from those checkpoints cuts the chains into segments."""
    import torch
    import selective_state_space_19_b200 as S
    Bt, L, d = 1, 4096, 128
    inp, dy, h0 = _inputs(io, Bt, L, d, seed=181)
    t = dev_inputs(inp)
    y, h, ck = _train_fwd(S, t, True, False, to_dev(h0))
    torch.cuda.synchronize()
    n = (L + EVERY - 1) // EVERY
    _check_forward(io, inp, True, False, h0, y, h, ck, ks=[0, 1, 37, n // 2, n - 1])
    got = S.s6_conv_scan_bwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                             to_dev(dy), z=t["z"], dt_bias=t["dt_bias"], ckpt=ck, want_dh_init=True)
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    ref = O.conv_scan_bwd(inp["x"], inp["conv_w"], inp["conv_b"], inp["dt"], inp["A_log"], inp["B"], inp["C"],
                          inp["D"], dy, z=inp["z"], dt_bias=inp["dt_bias"], h_init=h0)
    _check_grads(io, got, ref, ("dx", "dconv_w", "dconv_b", "ddt", "dz", "dB", "dC", "dA_log", "dD", "ddt_bias",
                                "dh_init"), f"assoc io={io}")


def test_train_backward_equals_recomputing_backward():
    """The backward from a training forward's checkpoints gives what the
    backward that runs its own forward gives (float32 I/O, where both forwards
    evaluate the SiLUs alike): same values up to the order of float32 sums."""
    import torch
    import selective_state_space_19_b200 as S
    Bt, L, d = 3, 333, 128
    inp, dy, _ = _inputs("f32", Bt, L, d, seed=190)
    t = dev_inputs(inp)
    _, _, ck = _train_fwd(S, t, True, False, None)
    a = S.s6_conv_scan_bwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                           to_dev(dy), z=t["z"], dt_bias=t["dt_bias"], ckpt=ck)
    b = S.s6_conv_scan_bwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                           to_dev(dy), z=t["z"], dt_bias=t["dt_bias"])
    torch.cuda.synchronize()
    for k in ("dx", "ddt", "dz", "dB", "dC", "dA_log", "dD", "dconv_w"):
        err = rel_err(a[k].cpu().numpy(), b[k].cpu().numpy())
        assert err <= 1e-5, (k, err)


def test_train_calls_refuse_what_they_cannot_do():
    """N != 16, and a start state passed to the backward alongside checkpoints."""
    import torch
    import selective_state_space_19_b200 as S
    inp = SI.scan_inputs("mamba_mini", Bt=1, L=32, d=64, N=8, io="f32", seed=3)
    t = dev_inputs(inp)
    with pytest.raises(S.S6Error) as e:
        S.s6_scan_fwd_ckpt(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"])
    assert e.value.status == S.S6_ERR_UNSUPPORTED
    inp, dy, h0 = _inputs("f32", 1, 32, 64, seed=4)
    t = dev_inputs(inp)
    _, _, ck = _train_fwd(S, t, False, False, None)
    with pytest.raises(ValueError):
        S.s6_scan_bwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], to_dev(dy), ckpt=ck,
                      h_init=torch.zeros(1, 64, 16, device="cuda"))
