"""GPU parity of s6_scan_bwd against the float64 oracle's backward pass.

Every gradient output is compared element by element with oracle.scan_bwd on
the same (rounded) inputs, in both write modes and both I/O types, with and
without the gate and a start state.  Shapes span several 64-token checkpoint
chunks with a ragged last chunk, channel counts whose warps straddle two
sequences (per-lane atomics) or not (warp sums), and N = 3, 8, 16.

Tolerance for these float32 gradients: max |g - ref| / (1 + |ref|) <= 2e-3.
The kernel evaluates in float32 with the hardware 2^x (relative error about
2^-22) and sums up to Bt*L (dA_log, dD, ddt_bias) or d (dB, dC) terms with
atomics in arbitrary order; the oracle is exact float64.
"""
import numpy as np
import pytest

from oracle import s6_oracle as O
import s6_inputs as SI
from s6_testutil import dev_inputs, note, rel_err, to_dev

pytestmark = pytest.mark.gpu

GTOL = 2e-3


def _case(io, zoh, gate, with_h, Bt, L, d, N, seed):
    import torch
    import selective_state_space_19_b200 as S
    inp = SI.scan_inputs("mamba_mini", Bt=Bt, L=L, d=d, N=N, io=io, seed=seed)
    rng = np.random.default_rng(seed + 1)
    dy = SI.to_storage(rng.standard_normal((Bt, L, d)).astype(np.float32), io)
    h0 = rng.standard_normal((Bt, d, N)).astype(np.float32) if with_h else None
    ref = O.scan_bwd(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], dy,
                     z=inp["z"] if gate else None, dt_bias=inp["dt_bias"], zoh=zoh, h_init=h0)
    t = dev_inputs(inp)
    got = S.s6_scan_bwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], to_dev(dy),
                        z=t["z"] if gate else None, dt_bias=t["dt_bias"], zoh_mode=int(zoh),
                        h_init=to_dev(h0) if with_h else None, want_dh_init=True)
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    keys = ["du", "ddt", "dB", "dC", "dA_log", "dD", "ddt_bias", "dh_init"] + (["dz"] if gate else [])
    for k in keys:
        g = got[k].cpu().numpy().astype(np.float64)
        err = rel_err(g, ref[k])
        note(f"grad {k} ({io})", err)
        assert np.all(np.isfinite(g)), k
        assert err <= GTOL, f"{k}: max|g-ref|/(1+|ref|) = {err:.3e} (io={io}, zoh={zoh}, gate={gate})"
    if not gate:
        assert got["dz"] is None


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("gate", [True, False])
def test_bwd_matches_oracle(io, zoh, gate):
    _case(io, zoh, gate, with_h=False, Bt=2, L=150, d=64, N=16, seed=11)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [dict(Bt=3, L=70, d=40, N=16),    # warps straddle sequences
                                   dict(Bt=2, L=65, d=96, N=8),
                                   dict(Bt=2, L=33, d=37, N=3),
                                   dict(Bt=1, L=1, d=32, N=16)])
def test_bwd_shapes_from_state(io, shape):
    _case(io, True, True, with_h=True, seed=shape["L"] + shape["d"], **shape)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("shape", [dict(Bt=2, L=150, d=64, N=16, K=4),
                                   dict(Bt=3, L=70, d=40, N=8, K=3),
                                   dict(Bt=2, L=33, d=24, N=3, K=2)])
def test_fused_bwd_matches_oracle(io, zoh, shape):
    """s6_conv_scan_bwd against the oracle's backward of the fused path, with
    the gate and a start state: dx, dconv_w, dconv_b and every scan gradient."""
    import torch
    import selective_state_space_19_b200 as S
    Bt, L, d, N, K = (shape[k] for k in ("Bt", "L", "d", "N", "K"))
    seed = 40 + L + d
    inp = SI.scan_inputs("mamba_mini", io=io, seed=seed, **shape)
    rng = np.random.default_rng(seed + 1)
    dy = SI.to_storage(rng.standard_normal((Bt, L, d)).astype(np.float32), io)
    h0 = rng.standard_normal((Bt, d, N)).astype(np.float32)
    ref = O.conv_scan_bwd(inp["x"], inp["conv_w"], inp["conv_b"], inp["dt"], inp["A_log"], inp["B"], inp["C"],
                          inp["D"], dy, z=inp["z"], dt_bias=inp["dt_bias"], zoh=zoh, h_init=h0)
    t = dev_inputs(inp)
    got = S.s6_conv_scan_bwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                             to_dev(dy), z=t["z"], dt_bias=t["dt_bias"], zoh_mode=int(zoh), h_init=to_dev(h0),
                             want_dh_init=True)
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    for k in ("dx", "dconv_w", "dconv_b", "ddt", "dz", "dB", "dC", "dA_log", "dD", "ddt_bias", "dh_init"):
        g = got[k].cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(g)), k
        err = rel_err(g, ref[k])
        note(f"grad fused {k} ({io})", err)
        assert err <= GTOL, f"{k}: max|g-ref|/(1+|ref|) = {err:.3e} (io={io}, zoh={zoh}, {shape})"


# ------------------------------------------------ the pipelined path (N = 16)
# At N = 16 with rows the tensor unit can move, the backward runs the forward
# kernel with state checkpoints, the reverse kernel over (segment, chain)
# units, and a reduction of the per-tile dB / dC rows.  These shapes cut the
# chains into segments (dLoss/dh and the conv's dpre window handed from one
# segment to the one before it) and take the associative split in the
# checkpointing forward.
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("zoh", [False, True])
def test_bwd_segmented_chains(io, zoh):
    _case(io, zoh, True, with_h=True, Bt=1, L=2000, d=128, N=16, seed=91)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("zoh", [False, True])
def test_fused_bwd_segmented_chains(io, zoh):
    import torch
    import selective_state_space_19_b200 as S
    Bt, L, d, N, K = 2, 1500, 64, 16, 4
    inp = SI.scan_inputs("mamba_mini", Bt=Bt, L=L, d=d, N=N, K=K, io=io, seed=92)
    rng = np.random.default_rng(93)
    dy = SI.to_storage(rng.standard_normal((Bt, L, d)).astype(np.float32), io)
    ref = O.conv_scan_bwd(inp["x"], inp["conv_w"], inp["conv_b"], inp["dt"], inp["A_log"], inp["B"], inp["C"],
                          inp["D"], dy, z=inp["z"], dt_bias=inp["dt_bias"], zoh=zoh)
    t = dev_inputs(inp)
    got = S.s6_conv_scan_bwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                             to_dev(dy), z=t["z"], dt_bias=t["dt_bias"], zoh_mode=int(zoh), want_dh_init=True)
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    for k in ("dx", "dconv_w", "dconv_b", "ddt", "dz", "dB", "dC", "dA_log", "dD", "ddt_bias", "dh_init"):
        g = got[k].cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(g)), k
        err = rel_err(g, ref[k])
        note(f"grad fused {k} ({io})", err)
        assert err <= GTOL, f"{k}: max|g-ref|/(1+|ref|) = {err:.3e} (io={io}, zoh={zoh})"


def test_bwd_unaligned_rows_take_the_simple_kernel():
    """Rows that are not 16-byte aligned (an offset view) take the plain
    backward kernel; the gradients still match the oracle."""
    import torch
    import selective_state_space_19_b200 as S
    Bt, L, d, N = 2, 90, 64, 16
    inp = SI.scan_inputs("mamba_mini", Bt=Bt, L=L, d=d, N=N, io="f32", seed=94)
    rng = np.random.default_rng(95)
    dy = rng.standard_normal((Bt, L, d)).astype(np.float32)
    ref = O.scan_bwd(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], dy, z=inp["z"],
                     dt_bias=inp["dt_bias"])
    t = dev_inputs(inp)
    buf = torch.empty(Bt * L * d + 1, device="cuda")
    u_off = buf[1:].view(Bt, L, d)  # 4 bytes past a 16-byte boundary
    u_off.copy_(t["x"])
    got = S.s6_scan_bwd(u_off, t["dt"], t["A_log"], t["B"], t["C"], t["D"], to_dev(dy), z=t["z"],
                        dt_bias=t["dt_bias"])
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    for k in ("du", "ddt", "dz", "dB", "dC", "dA_log", "dD", "ddt_bias"):
        err = rel_err(got[k].cpu().numpy().astype(np.float64), ref[k])
        assert err <= GTOL, f"{k}: {err:.3e}"


def test_bwd_full_long_seq_workload():
    """The backward at the long-sequence workload's full size (Bt16 L8192 d1536
    N16, bf16 inputs, gate, simplified write), in one launch sequence as the
    bench times it, against the oracle sequence by sequence: every element of
    du, ddt, dz, dB and dC, and the sums over all sequences dA_log, dD and
    ddt_bias."""
    import torch
    import selective_state_space_19_b200 as S
    cfg = SI.CONFIGS["long_seq"]
    inp = SI.scan_inputs("long_seq")
    Bt, L, d = cfg["Bt"], cfg["L"], cfg["d"]
    dy = SI.to_storage(np.random.default_rng(41).standard_normal((Bt, L, d)).astype(np.float32), "bf16")
    t = dev_inputs(inp)
    got = S.s6_scan_bwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], to_dev(dy), z=t["z"],
                        dt_bias=t["dt_bias"])
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    sums = {k: 0.0 for k in ("dA_log", "dD", "ddt_bias")}
    worst = {}
    for b in range(Bt):
        sl = slice(b, b + 1)
        ref = O.scan_bwd(inp["x"][sl], inp["dt"][sl], inp["A_log"], inp["B"][sl], inp["C"][sl], inp["D"], dy[sl],
                         z=inp["z"][sl], dt_bias=inp["dt_bias"])
        for k in ("du", "ddt", "dz", "dB", "dC"):
            err = rel_err(got[k][b].cpu().numpy().astype(np.float64), ref[k][0])
            worst[k] = max(worst.get(k, 0.0), err)
        for k in sums:
            sums[k] = sums[k] + ref[k]
    for k in sums:
        worst[k] = rel_err(got[k].cpu().numpy().astype(np.float64), sums[k])
    for k, err in worst.items():
        note(f"grad full long-seq {k} (bf16)", err)
        assert err <= GTOL, f"{k}: max|g-ref|/(1+|ref|) = {err:.3e}"


def test_conv_bwd_full_long_seq_workload():
    """The fused backward (conv + SiLU + scan) at the long-sequence workload's
    full size, against the oracle sequence by sequence: every element of dx,
    ddt, dz, dB and dC, and the sums over all sequences dconv_w, dconv_b,
    dA_log, dD and ddt_bias."""
    import torch
    import selective_state_space_19_b200 as S
    cfg = SI.CONFIGS["long_seq"]
    inp = SI.scan_inputs("long_seq")
    Bt, L, d = cfg["Bt"], cfg["L"], cfg["d"]
    dy = SI.to_storage(np.random.default_rng(43).standard_normal((Bt, L, d)).astype(np.float32), "bf16")
    t = dev_inputs(inp)
    got = S.s6_conv_scan_bwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                             to_dev(dy), z=t["z"], dt_bias=t["dt_bias"])
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    sums = {k: 0.0 for k in ("dconv_w", "dconv_b", "dA_log", "dD", "ddt_bias")}
    worst = {}
    for b in range(Bt):
        sl = slice(b, b + 1)
        ref = O.conv_scan_bwd(inp["x"][sl], inp["conv_w"], inp["conv_b"], inp["dt"][sl], inp["A_log"], inp["B"][sl],
                              inp["C"][sl], inp["D"], dy[sl], z=inp["z"][sl], dt_bias=inp["dt_bias"])
        for k in ("dx", "ddt", "dz", "dB", "dC"):
            err = rel_err(got[k][b].cpu().numpy().astype(np.float64), ref[k][0])
            worst[k] = max(worst.get(k, 0.0), err)
        for k in sums:
            sums[k] = sums[k] + ref[k]
    for k in sums:
        worst[k] = rel_err(got[k].cpu().numpy().astype(np.float64), sums[k])
    for k, err in worst.items():
        note(f"grad fused full long-seq {k} (bf16)", err)
        assert err <= GTOL, f"{k}: max|g-ref|/(1+|ref|) = {err:.3e}"
