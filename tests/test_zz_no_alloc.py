"""s6_conv_scan_fwd_noalloc: the fused scan for callers that cannot allocate.

Some callers own all of their device memory through their own allocator (a
framework's caching pool that has reserved the GPU) or run under a fixed memory
plan, so a library call must not cudaMalloc on their behalf.  The no-allocation
entry point keeps its segment carries in a fixed array inside the library.
These tests call it through the C ABI on shapes that do need the carries, twice
in a row on the same device (the array keeps the previous call's contents), and
compare with s6_conv_scan_fwd within the parity tolerance, and with the float64
oracle on sampled channels.  The file is
collected last and also passes when run alone in a fresh process.
"""
import numpy as np
import pytest

from oracle import s6_oracle as O
import s6_inputs as SI
from s6_testutil import TOL, as_f64, assert_close, dev_inputs, from_dev, sample_channels

pytestmark = pytest.mark.gpu


def _run(fn, t, zoh, y, h):
    return fn(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], z=t["z"],
              dt_bias=t["dt_bias"], zoh_mode=int(zoh), y=y, h_final=h)


@pytest.mark.parametrize("io,zoh", [("bf16", False), ("f32", True)])
def test_noalloc_matches_allocating_entry_point_twice(io, zoh):
    import torch
    import selective_state_space_19_b200 as S
    # few (sequence, channel-tile) pairs and a long sequence: the scan is split
    # into segments whose end states pass through the scratch array
    inp = SI.scan_inputs("long_seq", Bt=2, L=3000, d=256, io=io, seed=77)
    t = dev_inputs(inp)
    y_ref = torch.empty_like(t["x"])
    h_ref = torch.empty(2, 256, 16, device="cuda")
    _run(S.s6_conv_scan_fwd, t, zoh, y_ref, h_ref)
    for _ in range(2):
        y = torch.full_like(t["x"], 7.0)
        h = torch.full((2, 256, 16), 7.0, device="cuda")
        _run(S.s6_conv_scan_fwd_noalloc, t, zoh, y, h)
        torch.cuda.synchronize()
        assert S.s6_device_status() == 0
        assert_close(as_f64(from_dev(y)), as_f64(from_dev(y_ref)), io, "y")
        assert_close(h.cpu().numpy(), h_ref.cpu().numpy(), io, "h_final")
    # and, standing on its own, against the float64 oracle on sampled channels
    ch = sample_channels(2, 256, 30, seed=76)
    ry, rh = O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"],
                    dt_bias=inp["dt_bias"], zoh=zoh, conv_w=inp["conv_w"], conv_b=inp["conv_b"], channels=ch)
    yg, hg = as_f64(from_dev(y)), h.cpu().numpy()
    assert_close(np.stack([yg[b, :, c] for b, c in ch]), ry, io, "noalloc y vs oracle")
    assert_close(np.stack([hg[b, c] for b, c in ch]), rh, io, "noalloc h_final vs oracle")


def test_noalloc_other_shape_after_a_larger_one():
    """A smaller problem right after a larger one: nothing left in the array from
    the previous call leaks into the result."""
    import torch
    import selective_state_space_19_b200 as S
    for (Bt, L, d, seed) in ((3, 2500, 512, 78), (1, 1700, 64, 79)):
        inp = SI.scan_inputs("long_seq", Bt=Bt, L=L, d=d, seed=seed)
        t = dev_inputs(inp)
        y_ref, h_ref = _run(S.s6_conv_scan_fwd, t, False, None, None)
        y, h = _run(S.s6_conv_scan_fwd_noalloc, t, False, None, None)
        torch.cuda.synchronize()
        assert S.s6_device_status() == 0
        assert_close(as_f64(from_dev(y)), as_f64(from_dev(y_ref)), "bf16", "y")
        assert_close(h.cpu().numpy(), h_ref.cpu().numpy(), "bf16", "h_final")


def test_noalloc_rejects_problems_beyond_the_array():
    """A segmented schedule whose carries exceed the fixed array is refused with
    S6_ERR_SCRATCH_LIMIT before anything is enqueued."""
    import torch
    import selective_state_space_19_b200 as S
    # 1024 (sequence, 64-channel tile) chains, each long enough to be split into
    # segments: ~4.2 MB of carries
    Bt, L, d, N = 16, 1024, 4096, 16
    x = torch.zeros(Bt, L, d, dtype=torch.bfloat16, device="cuda")
    Bm = torch.zeros(Bt, L, N, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(d, 4, device="cuda")
    A = torch.zeros(d, N, device="cuda")
    Dv = torch.zeros(d, device="cuda")
    with pytest.raises(S.S6Error) as e:
        S.s6_conv_scan_fwd_noalloc(x, w, None, x, A, Bm, Bm, Dv)
    assert e.value.status == S.S6_ERR_SCRATCH_LIMIT
    assert "4 MiB" in S.s6_status_string(S.S6_ERR_SCRATCH_LIMIT)
    assert S.s6_device_status() == 0
    assert TOL["bf16"] == 1e-2
