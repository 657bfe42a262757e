"""GPU parity of causal_conv1d_silu_fwd and s6_step against the float64 oracle,
plus the streaming checks of the TinyMamba example on the GPU path: token
streaming equals the full forward, and a scan resumed by the step equals the
longer scan."""
import numpy as np
import pytest

from oracle import s6_oracle as O
import s6_inputs as SI
from s6_testutil import as_f64, assert_close, dev_inputs, from_dev, sample_channels, to_dev

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------ standalone conv
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("Bt,L,d,K", [(1, 6, 8, 3), (2, 300, 1536, 4), (3, 257, 40, 2), (1, 1, 64, 4),
                                      (2, 1000, 264, 3)])
def test_conv_silu(io, Bt, L, d, K):
    import selective_state_space_19_b200 as S
    import torch
    inp = SI.scan_inputs("mamba_mini", Bt=Bt, L=L, d=d, K=K, io=io, seed=L + d)
    t = dev_inputs(inp)
    out = S.causal_conv1d_silu_fwd(t["x"], t["conv_w"], t["conv_b"])
    torch.cuda.synchronize()
    ref = O.conv_silu(inp["x"], inp["conv_w"], inp["conv_b"])
    assert_close(as_f64(from_dev(out)), ref, io, "xc")


def test_conv_silu_no_bias_full_long_seq_rows():
    """Full-width rows of the long-sequence workload (bf16, d=1536, K=4), no bias."""
    import selective_state_space_19_b200 as S
    import torch
    inp = SI.scan_inputs("long_seq", Bt=2, L=2048)
    t = dev_inputs(inp)
    out = S.causal_conv1d_silu_fwd(t["x"], t["conv_w"], None)
    torch.cuda.synchronize()
    ref = O.conv_silu(inp["x"], inp["conv_w"], None)
    assert_close(as_f64(from_dev(out)), ref, "bf16", "xc")


def test_conv_silu_full_long_seq_workload():
    """The standalone conv at the bench row's configuration: the long-sequence
    workload's x in full (Bt16 L8192 d1536 bf16, K=4, with bias), every
    element, the oracle sequence by sequence."""
    import selective_state_space_19_b200 as S
    import torch
    inp = SI.scan_inputs("long_seq")
    t = dev_inputs(inp)
    out = S.causal_conv1d_silu_fwd(t["x"], t["conv_w"], t["conv_b"])
    torch.cuda.synchronize()
    got = from_dev(out)
    for b in range(inp["Bt"]):
        ref = O.conv_silu(inp["x"][b:b + 1], inp["conv_w"], inp["conv_b"])
        assert_close(as_f64(got[b:b + 1]), ref, "bf16", "xc full long-seq")


# ------------------------------------------------------------ streaming step
def _step_gpu(S, t, tok, h, cs, zoh):
    return S.s6_step(tok["x"], tok["dt"], tok["B"], tok["C"], t["A_log"], t["D"], t["conv_w"], h, cs, z_t=tok["z"],
                     dt_bias=t["dt_bias"], conv_b=t["conv_b"], zoh_mode=int(zoh))


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("cfg", [dict(Bt=1, L=6, d=8, N=3, K=3), dict(Bt=4, L=40, d=200, N=16, K=4),
                                 dict(Bt=3, L=25, d=72, N=5, K=2), dict(Bt=2, L=30, d=64, N=8, K=4)])
def test_streaming_equals_full_forward(io, zoh, cfg):
    """The streaming check of "Carry context through a selective state" (Verified
    by the local recipe): L single-token steps on the GPU reproduce the oracle's
    full-sequence outputs and final state."""
    import selective_state_space_19_b200 as S
    import torch
    inp = SI.scan_inputs("mamba_mini", io=io, seed=31 + cfg["L"], **cfg)
    Bt, L, d, N, K = (cfg[k] for k in ("Bt", "L", "d", "N", "K"))
    ry, rh, rhist = O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"],
                           dt_bias=inp["dt_bias"], zoh=zoh, conv_w=inp["conv_w"], conv_b=inp["conv_b"],
                           return_state=True)
    t = dev_inputs(inp)
    h = torch.zeros(Bt, d, N, device="cuda")
    cs = torch.zeros(Bt, d, K - 1, device="cuda", dtype=t["x"].dtype)
    ys = []
    for s in range(L):
        tok = {k: t[k][:, s].contiguous() for k in ("x", "dt", "z", "B", "C")}
        ys.append(from_dev(_step_gpu(S, t, tok, h, cs, zoh)))
    torch.cuda.synchronize()
    y = np.stack([as_f64(v) for v in ys], axis=1)
    assert_close(y, ry, io, "y")
    assert_close(h.cpu().numpy(), rh, io, "h_ssm")
    # the conv history holds the last K-1 inputs exactly
    np.testing.assert_array_equal(as_f64(from_dev(cs)), rhist)


def _shifted(tensor, shift):
    """A copy of `tensor` placed `shift` elements into a larger buffer: aligned to
    its element size but not to 16 bytes."""
    import torch
    flat = torch.empty(tensor.numel() + shift, dtype=tensor.dtype, device=tensor.device)
    view = flat[shift:].view(tensor.shape)
    view.copy_(tensor)
    return view


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("case", ["n4_bulk_rows", "rows_not_16B_multiple", "rows_misaligned_k2", "n8_k3_ragged"])
def test_step_row_paths(io, zoh, case):
    """The step's ways of moving a tile's per-token rows, against the oracle's full
    forward: N = 4 with bulk-copied rows; d * sizeof(io) not a multiple of 16
    (rows read with plain loads, results written directly); rows and conv history
    at element-aligned but not 16-byte-aligned addresses, K = 2 (plain loads
    again); N = 8, K = 3 with a ragged last channel tile."""
    import selective_state_space_19_b200 as S
    import torch
    cfg = {"n4_bulk_rows": dict(Bt=3, L=12, d=136, N=4, K=4),
           "rows_not_16B_multiple": dict(Bt=2, L=10, d=202, N=16, K=3),
           "rows_misaligned_k2": dict(Bt=2, L=10, d=160, N=16, K=2),
           "n8_k3_ragged": dict(Bt=5, L=9, d=300, N=8, K=3)}[case]
    shift = 1 if case == "rows_misaligned_k2" else 0
    inp = SI.scan_inputs("mamba_mini", io=io, seed=71 + cfg["d"], **cfg)
    Bt, L, d, N, K = (cfg[k] for k in ("Bt", "L", "d", "N", "K"))
    ry, rh, rhist = O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"],
                           dt_bias=inp["dt_bias"], zoh=zoh, conv_w=inp["conv_w"], conv_b=inp["conv_b"],
                           return_state=True)
    t = dev_inputs(inp)
    h = torch.zeros(Bt, d, N, device="cuda")
    cs = torch.zeros(Bt, d, K - 1, device="cuda", dtype=t["x"].dtype)
    if shift:
        cs = _shifted(cs, shift)
    ys = []
    for s in range(L):
        tok = {k: t[k][:, s].contiguous() for k in ("x", "dt", "z", "B", "C")}
        if shift:
            tok = {k: _shifted(v, shift) for k, v in tok.items()}
        ys.append(from_dev(_step_gpu(S, t, tok, h, cs, zoh)))
    torch.cuda.synchronize()
    assert S.s6_device_status() == 0
    y = np.stack([as_f64(v) for v in ys], axis=1)
    assert_close(y, ry, io, "y")
    assert_close(h.cpu().numpy(), rh, io, "h_ssm")
    np.testing.assert_array_equal(as_f64(from_dev(cs)), rhist)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_scan_then_step_resume(io):
    """Checkpoint/resume: scan tokens [0, L1) with h_final, then continue with the
    step from (h_final, last K-1 inputs); equals the oracle's scan over [0, L)."""
    import selective_state_space_19_b200 as S
    import torch
    Bt, L, L1, d, N, K = 2, 60, 41, 136, 16, 4
    inp = SI.scan_inputs("mamba_mini", Bt=Bt, L=L, d=d, N=N, K=K, io=io, seed=44)
    ry, rh = O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"],
                    dt_bias=inp["dt_bias"], conv_w=inp["conv_w"], conv_b=inp["conv_b"])
    t = dev_inputs(inp)
    pre = {k: t[k][:, :L1].contiguous() for k in ("x", "dt", "z", "B", "C")}
    y1, h = S.s6_conv_scan_fwd(pre["x"], t["conv_w"], t["conv_b"], pre["dt"], t["A_log"], pre["B"], pre["C"],
                               t["D"], z=pre["z"], dt_bias=t["dt_bias"])
    cs = t["x"][:, L1 - (K - 1):L1].transpose(1, 2).contiguous()  # [Bt, d, K-1], oldest first
    ys = [from_dev(y1)]
    for s in range(L1, L):
        tok = {k: t[k][:, s].contiguous() for k in ("x", "dt", "z", "B", "C")}
        ys.append(from_dev(_step_gpu(S, t, tok, h, cs, False))[:, None, :])
    torch.cuda.synchronize()
    y = np.concatenate([as_f64(v) for v in ys], axis=1)
    assert_close(y, ry, io, "y")
    assert_close(h.cpu().numpy(), rh, io, "h")


def test_decode_workload_sampled():
    """Streaming-decode workload shape: 256 sequences x d1536 x N16, K4, fp32 state,
    for two of the six blocks over 24 steps, against the oracle on 48 sampled
    (sequence, channel) pairs; plus a step from a non-zero state."""
    import selective_state_space_19_b200 as S
    import torch
    Bt, d, N, K, steps = 256, 1536, 16, 4, 24
    rng = np.random.default_rng(5)
    pick_b = rng.integers(0, Bt, 48)
    pick_d = rng.integers(0, d, 48)
    for block in (0, 5):
        p = SI.decode_params(block)
        pt = {k: to_dev(v) for k, v in p.items()}
        h = torch.zeros(Bt, d, N, device="cuda")
        cs = torch.zeros(Bt, d, K - 1, device="cuda")
        toks = [SI.decode_tokens(s, block) for s in range(steps)]
        ys = []
        for tok in toks:
            tt = {k: to_dev(v) for k, v in tok.items()}
            ys.append(from_dev(S.s6_step(tt["x"], tt["dt"], tt["B"], tt["C"], pt["A_log"], pt["D"], pt["conv_w"], h,
                                         cs, z_t=tt["z"], dt_bias=pt["dt_bias"], conv_b=pt["conv_b"])))
        torch.cuda.synchronize()
        # oracle: the sampled channels over the same token sequence
        xs = np.stack([tok["x"] for tok in toks], axis=1)  # [Bt, steps, d]
        seq = {k: np.stack([tok[k] for tok in toks], axis=1) for k in ("x", "dt", "z", "B", "C")}
        ch = np.stack([pick_b, pick_d], axis=1)
        ry, rh = O.scan(seq["x"], seq["dt"], p["A_log"], seq["B"], seq["C"], p["D"], z=seq["z"],
                        dt_bias=p["dt_bias"], conv_w=p["conv_w"], conv_b=p["conv_b"], channels=ch)
        y = np.stack(ys, axis=1)
        assert xs.shape == (Bt, steps, d)
        assert_close(np.stack([y[b, :, dd] for b, dd in ch]), ry, "f32", "y")
        hg = h.cpu().numpy()
        assert_close(np.stack([hg[b, dd] for b, dd in ch]), rh, "f32", "h_ssm")


def test_decode_workload_full_length():
    """The streaming-decode workload at its stated length: 1024 single-token steps
    through each of the 6 blocks (d1536, N16, K4, float32 state), on a stated
    subset of 16 sequences (the workload's per-(step, block) seeding with a
    16-sequence batch), against the oracle's scan of the same token sequence:
    y at every step on 96 sampled channels per block, the final h_ssm on those
    channels, and the final conv history of every channel (exact)."""
    import selective_state_space_19_b200 as S
    import torch
    Bt, d, N, K, steps, blocks = 16, 1536, 16, 4, 1024, 6
    ch = sample_channels(Bt, d, 92, seed=9)
    for block in range(blocks):
        p = SI.decode_params(block)
        pt = {k: to_dev(v) for k, v in p.items()}
        toks = [SI.decode_tokens(s, block, Bt=Bt) for s in range(steps)]
        seq = {k: np.stack([tok[k] for tok in toks], axis=0) for k in ("x", "dt", "z", "B", "C")}  # [steps, Bt, .]
        td = {k: to_dev(v) for k, v in seq.items()}
        h = torch.zeros(Bt, d, N, device="cuda")
        cs = torch.zeros(Bt, d, K - 1, device="cuda")
        ys = torch.empty(steps, Bt, d, device="cuda")
        for s in range(steps):
            S.s6_step(td["x"][s], td["dt"][s], td["B"][s], td["C"][s], pt["A_log"], pt["D"], pt["conv_w"], h, cs,
                      z_t=td["z"][s], dt_bias=pt["dt_bias"], conv_b=pt["conv_b"], y_t=ys[s])
        torch.cuda.synchronize()
        assert S.s6_device_status() == 0
        ref_in = {k: np.ascontiguousarray(np.transpose(v, (1, 0, 2))) for k, v in seq.items()}  # [Bt, steps, .]
        ry, rh = O.scan(ref_in["x"], ref_in["dt"], p["A_log"], ref_in["B"], ref_in["C"], p["D"], z=ref_in["z"],
                        dt_bias=p["dt_bias"], conv_w=p["conv_w"], conv_b=p["conv_b"], channels=ch)
        y = ys.cpu().numpy()  # [steps, Bt, d]
        assert_close(np.stack([y[:, b, dd] for b, dd in ch]), ry, "f32", "decode 1024-step y")
        hg = h.cpu().numpy()
        assert_close(np.stack([hg[b, dd] for b, dd in ch]), rh, "f32", "decode 1024-step h_ssm")
        # the history holds the last K-1 inputs exactly, oldest first
        np.testing.assert_array_equal(cs.cpu().numpy(), np.transpose(seq["x"][-(K - 1):], (1, 2, 0)))


def test_step_rejects_bad_arguments():
    import selective_state_space_19_b200 as S
    import torch
    p = {k: to_dev(v) for k, v in SI.decode_params(0, d=64, N=16, K=4).items()}
    tok = {k: to_dev(v) for k, v in SI.decode_tokens(0, 0, Bt=2, d=64, N=16).items()}
    h = torch.zeros(2, 64, 16, device="cuda")
    cs = torch.zeros(2, 64, 3, device="cuda")
    with pytest.raises(S.S6Error) as e:
        S.s6_step(tok["x"], tok["dt"], tok["B"], tok["C"], p["A_log"], p["D"], p["conv_w"], h, cs, zoh_mode=5)
    assert e.value.status == S.S6_ERR_INVALID_ARG
    w5 = torch.zeros(64, 5, device="cuda")
    cs4 = torch.zeros(2, 64, 4, device="cuda")
    with pytest.raises(S.S6Error) as e:
        S.s6_step(tok["x"], tok["dt"], tok["B"], tok["C"], p["A_log"], p["D"], w5, h, cs4)
    assert e.value.status == S.S6_ERR_UNSUPPORTED


def test_calls_capture_into_a_cuda_graph():
    """The step and the fused scan can be captured in a CUDA graph and replayed;
    replays equal eager calls."""
    import selective_state_space_19_b200 as S
    import torch
    p = {k: to_dev(v) for k, v in SI.decode_params(1, d=256).items()}
    toks = [{k: to_dev(v) for k, v in SI.decode_tokens(s, 1, Bt=8, d=256).items()} for s in range(3)]
    inp = SI.scan_inputs("long_seq", Bt=1, L=300, d=256)
    t = dev_inputs(inp)
    stream = torch.cuda.Stream()

    def run(h, cs, ys, y):
        for i, tok in enumerate(toks):
            S.s6_step(tok["x"], tok["dt"], tok["B"], tok["C"], p["A_log"], p["D"], p["conv_w"], h, cs, z_t=tok["z"],
                      dt_bias=p["dt_bias"], conv_b=p["conv_b"], y_t=ys[i], stream=stream)
        S.s6_conv_scan_fwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], z=t["z"],
                           dt_bias=t["dt_bias"], y=y, h_final=hf, stream=stream)

    def fresh():
        return (torch.zeros(8, 256, 16, device="cuda"), torch.zeros(8, 256, 3, device="cuda"),
                [torch.empty(8, 256, device="cuda") for _ in toks], torch.empty_like(t["x"]))

    hf = torch.empty(1, 256, 16, device="cuda")
    with torch.cuda.stream(stream):
        h0, c0, ys0, y0 = fresh()
        run(h0, c0, ys0, y0)
        torch.cuda.synchronize()
        ref = [v.clone() for v in ys0] + [h0.clone(), y0.clone(), hf.clone()]
        h1, c1, ys1, y1 = fresh()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            run(h1, c1, ys1, y1)
        g.replay()
        torch.cuda.synchronize()
    got = ys1 + [h1, y1, hf]
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    assert S.s6_device_status() == 0
