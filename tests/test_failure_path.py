"""The failure path of the bounded device-side waits, exercised without a GPU fault.

A segmented scan hands a segment's end state (or, in the associative split, a
segment's pieces) to the unit that continues the sequence; that unit waits for
a published flag, with a limit.  The test-only knob s6_debug_carry_fault makes
one unit skip its publication and shortens the limit, so the successor's wait
runs out: the kernel records the timeout in the device error word and exits
normally, s6_device_status reports S6_ERR_TIMEOUT, and the context stays
usable -- the next scan, with the knob off, matches the oracle again.
"""
import numpy as np
import pytest

from oracle import s6_oracle as O
import s6_inputs as SI
from s6_testutil import as_f64, assert_close, dev_inputs, from_dev, sample_channels

pytestmark = pytest.mark.gpu


def _scan(S, t):
    return S.s6_conv_scan_fwd(t["x"], t["conv_w"], t["conv_b"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                              z=t["z"], dt_bias=t["dt_bias"])


@pytest.mark.parametrize("shape,schedule", [
    # 256 (sequence, 64-channel tile) chains: the serial chain of segments
    (dict(Bt=16, L=2048, d=1024), "serial"),
    # 2 chains: the associative split
    (dict(Bt=1, L=3000, d=128), "associative"),
])
def test_skipped_carry_times_out_and_recovers(shape, schedule):
    import selective_state_space_19_b200 as S
    import torch
    inp = SI.scan_inputs("long_seq", seed=61, **shape)
    t = dev_inputs(inp)
    assert S.s6_device_status() == S.S6_OK
    try:
        # unit 0 (the first segment of the first chain) publishes nothing; waits
        # for it give up after 2048 polls
        S.s6_debug_carry_fault(0, 2048)
        _scan(S, t)
        torch.cuda.synchronize()
        assert S.s6_device_status() == S.S6_ERR_TIMEOUT
    finally:
        S.s6_debug_carry_fault()
    # the error word was cleared by the read, and the context is usable
    assert S.s6_device_status() == S.S6_OK
    y, h = _scan(S, t)
    torch.cuda.synchronize()
    assert S.s6_device_status() == S.S6_OK
    ch = sample_channels(shape["Bt"], shape["d"], 20, seed=62)
    ry, rh = O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"],
                    dt_bias=inp["dt_bias"], conv_w=inp["conv_w"], conv_b=inp["conv_b"], channels=ch)
    yg, hg = as_f64(from_dev(y)), h.cpu().numpy()
    assert_close(np.stack([yg[b, :, c] for b, c in ch]), ry, "bf16", "y after recovery")
    assert_close(np.stack([hg[b, c] for b, c in ch]), rh, "bf16", "h_final after recovery")


def test_knob_off_by_default_and_reset():
    """With no injection, a segmented scan reports no error."""
    import selective_state_space_19_b200 as S
    import torch
    S.s6_debug_carry_fault()
    inp = SI.scan_inputs("long_seq", Bt=16, L=1024, d=1024, seed=63)
    _scan(S, dev_inputs(inp))
    torch.cuda.synchronize()
    assert S.s6_device_status() == S.S6_OK
