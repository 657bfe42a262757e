"""Pins for the float64 oracle: what the pages and the mathematics fix.

Nothing here compares the oracle with itself.  Each test checks one of:
  * values the TinyMamba example prints ("Carry context through a selective
    state", model manifest `experiment.cases`, stored in
    tests/golden/tinymamba_recorded.json);
  * the four checks that page lists under "Verified by the local recipe";
  * closed forms (geometric series, the exact zero-order-hold solution of
    dh/dt = A h + B u for a held input);
  * an independent brute-force decayed sum, written from the sum formula;
  * special values and identities of softplus / SiLU against the C library;
  * the state sizes printed by "mamba, live" and the TinyMamba example.
test_mutations.py then shows these pins fail when a plausible mistake is
planted in a copy of the oracle.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import s6_oracle as O
import s6_inputs as SI

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tinymamba_recorded.json")


def golden():
    with open(GOLDEN) as f:
        return {c["id"]: c for c in json.load(f)["cases"]}


def a_log_teaching(n):
    # TinyMamba keeps A_log as a float32 parameter initialised to log(n+1)
    return float(np.float32(math.log(n + 1)))


# ---------------------------------------------------------------- recorded values
def test_recorded_decays_exact():
    """Printed Delta (channel 0) and A_log = f32(log(n+1)) give the printed decays."""
    g = golden()
    for cid in ("first", "middle", "last", "changed"):
        c = g[cid]
        delta0 = c["delta"][0]
        for n in range(3):
            assert O.decay(delta0, a_log_teaching(n)) == pytest.approx(c["channel0_decay"][n], rel=1e-15, abs=0)


def test_recorded_decays_in_unit_interval():
    g = golden()
    for c in g.values():
        for ch in range(8):
            for n in range(3):
                a = O.decay(c["delta"][ch], a_log_teaching(n))
                assert 0.0 < a < 1.0


def test_recorded_first_state_equals_first_write():
    """Zero initial state: after token 0 the state is exactly the write."""
    c = golden()["first"]
    for n in range(3):
        h0 = O.update(0.0, c["channel0_decay"][n], c["channel0_write"][n])
        assert h0 == c["channel0_state_history"][0][n]
        assert h0 == c["full_state"][0][n]


def test_recorded_update_rule_exact():
    """h_t = A_bar_t * h_{t-1} + write_t reproduces the printed states bit for bit."""
    g = golden()
    mid, last, chg = g["middle"], g["last"], g["changed"]
    for n in range(3):
        # token 2 from token 1
        h2 = O.update(mid["channel0_state_history"][1][n], mid["channel0_decay"][n], mid["channel0_write"][n])
        assert h2 == pytest.approx(mid["channel0_state_history"][2][n], rel=1e-15, abs=1e-18)
        # token 5 from token 4, both the original and the changed sequence
        for c in (last, chg):
            h5 = O.update(c["channel0_state_history"][4][n], c["channel0_decay"][n], c["channel0_write"][n])
            assert h5 == pytest.approx(c["channel0_state_history"][5][n], rel=1e-15, abs=1e-18)


def test_recorded_changed_token_carries_through_decay_only():
    """Changing token 2: tokens 0-1 unchanged; at token 5 (outside a width-3 conv
    window of token 2) Delta, decays and write are unchanged, so the state
    difference is the decayed previous difference."""
    g = golden()
    last, chg = g["last"], g["changed"]
    assert chg["channel0_state_history"][:2] == last["channel0_state_history"][:2]
    assert chg["channel0_state_history"][2] != last["channel0_state_history"][2]
    assert chg["delta"] == last["delta"]
    assert chg["channel0_write"] == last["channel0_write"]
    for n in range(3):
        d4 = chg["channel0_state_history"][4][n] - last["channel0_state_history"][4][n]
        d5 = chg["channel0_state_history"][5][n] - last["channel0_state_history"][5][n]
        a5 = O.decay(last["delta"][0], a_log_teaching(n))
        assert d5 == pytest.approx(a5 * d4, rel=1e-9, abs=1e-18)


def test_state_sizes():
    g = golden()["first"]
    # TinyMamba: 8 channels x 3 states; conv width 3 -> 2 past inputs x 8 channels
    assert O.ssm_state_values(8, 3) == 24 == g["ssm_state_values"]
    assert O.conv_history_values(8, 3) == 16 == g["conv_history_values"]
    # Mamba-mini ("mamba, live"): 1,536 channels x 16 states x 6 blocks
    assert O.ssm_state_values(1536, 16, 6) == 147456


# ------------------------------------------------------------ special functions
@pytest.mark.parametrize("v", [-60.0, -20.0, -7.0, -1.0, -1e-3, 0.0, 1e-3, 0.5, 3.0, 19.0, 21.0, 60.0])
def test_softplus_against_libm(v):
    ref = math.log1p(math.exp(v)) if v < 30 else v + math.log1p(math.exp(-v))
    assert O.softplus(v) == pytest.approx(ref, rel=1e-14, abs=0)
    assert O.softplus(v) > 0
    # softplus(v) - softplus(-v) = v
    assert O.softplus(v) - O.softplus(-v) == pytest.approx(v, rel=1e-12, abs=1e-15)


def test_softplus_zero_is_ln2():
    assert O.softplus(0.0) == math.log(2.0)


@pytest.mark.parametrize("v", [-80.0, -10.0, -1.0, -1e-4, 0.0, 1e-4, 0.7, 5.0, 40.0])
def test_silu_against_libm(v):
    ref = v / (1.0 + math.exp(-v))
    assert O.silu(v) == pytest.approx(ref, rel=1e-14, abs=1e-300)
    # SiLU(v) - SiLU(-v) = v
    assert O.silu(v) - O.silu(-v) == pytest.approx(v, rel=1e-12, abs=1e-15)


def test_A_is_negative_exp():
    for al in (-2.0, 0.0, math.log(2.0), 3.0):
        assert O.A_of(al) == -math.exp(al)


def test_zoh_gain_tends_to_delta():
    """expm1(Delta*A)/A -> Delta as Delta -> 0: the exact ZOH reduces to the simplified term."""
    for al in (0.0, math.log(16.0)):
        A = math.exp(al)
        for delta in (1e-9, 1e-6, 1e-3):
            g = O.write_gain(delta, al, True)
            assert abs(g / delta - 1.0) <= A * delta  # |1 - (1-e^-x)/x| <= x/2
            assert O.write_gain(delta, al, False) == delta


# --------------------------------------------------------------- closed forms
def _mk(L, N, *, zoh, seed=0, K=0, gate=False, const=False):
    rng = np.random.default_rng(seed)
    Bt, d = 1, 3
    if const:
        x = np.full((Bt, L, d), 0.8)
        dtr = np.full((Bt, L, d), -0.3)
        Bm = np.full((Bt, L, N), 1.3)
        Cm = np.full((Bt, L, N), 0.7)
    else:
        x = rng.standard_normal((Bt, L, d))
        dtr = rng.standard_normal((Bt, L, d))
        Bm = rng.standard_normal((Bt, L, N))
        Cm = rng.standard_normal((Bt, L, N))
    z = rng.standard_normal((Bt, L, d)) if gate else None
    A_log = np.log(rng.uniform(0.5, 4.0, (d, N)))
    D = rng.uniform(0.5, 1.5, d)
    dt_bias = rng.uniform(-1, 1, d)
    cw = rng.uniform(-0.5, 0.5, (d, K)) if K else None
    cb = rng.uniform(-0.5, 0.5, d) if K else None
    return dict(x=x, dt_raw=dtr, B=Bm, C=Cm, z=z, A_log=A_log, D=D, dt_bias=dt_bias, conv_w=cw, conv_b=cb)


def _run(p, zoh, **kw):
    return O.scan(p["x"], p["dt_raw"], p["A_log"], p["B"], p["C"], p["D"], z=p["z"], dt_bias=p["dt_bias"],
                  zoh=zoh, conv_w=p["conv_w"], conv_b=p["conv_b"], **kw)


def test_geometric_series_simplified():
    """Held input, one state: h_t = w (1 - a^(t+1)) / (1 - a), a first-order IIR filter."""
    L, N = 40, 1
    p = _mk(L, N, zoh=False, const=True)
    y, h = _run(p, False)
    for ch in range(3):
        delta = math.log1p(math.exp(-0.3 + p["dt_bias"][ch]))
        A = -math.exp(p["A_log"][ch, 0])
        a = math.exp(delta * A)
        w = delta * 1.3 * 0.8
        for t in (0, 1, 7, L - 1):
            ht = w * (1 - a ** (t + 1)) / (1 - a)
            assert y[0, t, ch] == pytest.approx(ht * 0.7 + p["D"][ch] * 0.8, rel=1e-12)
        assert h[0, ch, 0] == pytest.approx(w * (1 - a ** L) / (1 - a), rel=1e-12)


def test_zoh_matches_continuous_time_solution():
    """Exact ZOH: for a held input u and B, stepping with Delta_1..Delta_T must equal the
    exact solution of dh/dt = A h + B u over the total time T = sum Delta_t:
    h(T) = (exp(A T) - 1)/A * B u.  The simplified term does not satisfy this."""
    L, N = 25, 4
    rng = np.random.default_rng(5)
    x = np.full((1, L, 2), 0.9)
    dtr = rng.standard_normal((1, L, 2))
    Bm = np.full((1, L, N), -1.1)
    Cm = rng.standard_normal((1, L, N))
    A_log = np.log(rng.uniform(0.3, 3.0, (2, N)))
    D = np.zeros(2)
    _, h = O.scan(x, dtr, A_log, Bm, Cm, D, dt_bias=np.zeros(2), zoh=True)
    _, h_s = O.scan(x, dtr, A_log, Bm, Cm, D, dt_bias=np.zeros(2), zoh=False)
    for ch in range(2):
        T = sum(math.log1p(math.exp(v)) for v in dtr[0, :, ch])
        for n in range(N):
            A = -math.exp(A_log[ch, n])
            exact = math.expm1(A * T) / A * (-1.1) * 0.9
            assert h[0, ch, n] == pytest.approx(exact, rel=1e-12)
            assert abs(h_s[0, ch, n] - exact) > 1e-6 * abs(exact)


@pytest.mark.parametrize("zoh", [False, True])
def test_bruteforce_decayed_sum(zoh):
    """'The recurrent state matches an independent sum of decayed past writes':
    h_t = sum_{s<=t} (prod_{s<r<=t} A_bar_r) * write_s, with y_t = <h_t, C_t> + D u_t."""
    L, N = 9, 3
    p = _mk(L, N, zoh=zoh, seed=11, gate=True)
    y, h = _run(p, zoh)
    for ch in range(3):
        delta = np.logaddexp(0.0, p["dt_raw"][0, :, ch] + p["dt_bias"][ch])
        A = -np.exp(p["A_log"][ch])
        u = p["x"][0, :, ch]
        abar = np.exp(delta[:, None] * A[None, :])
        gain = (np.expm1(delta[:, None] * A[None, :]) / A[None, :]) if zoh else delta[:, None]
        write = gain * p["B"][0] * u[:, None]
        for t in range(L):
            hs = np.zeros(N)
            for s in range(t + 1):
                hs += np.prod(abar[s + 1:t + 1], axis=0) * write[s]
            gate = p["z"][0, t, ch] / (1 + np.exp(-p["z"][0, t, ch]))
            yt = (hs @ p["C"][0, t] + p["D"][ch] * u[t]) * gate
            assert y[0, t, ch] == pytest.approx(yt, rel=1e-11, abs=1e-14)
        assert h[0, ch] == pytest.approx(hs, rel=1e-11, abs=1e-14)


def test_readout_uses_updated_state():
    """'C reads the updated state': one token from zero state gives y = <write, C> + D u."""
    p = _mk(1, 1, zoh=False)
    p["D"] = np.zeros(3)
    y, _ = _run(p, False)
    for ch in range(3):
        delta = math.log1p(math.exp(p["dt_raw"][0, 0, ch] + p["dt_bias"][ch]))
        w = delta * p["B"][0, 0, 0] * p["x"][0, 0, ch]
        assert y[0, 0, ch] == pytest.approx(w * p["C"][0, 0, 0], rel=1e-13)
        assert y[0, 0, ch] != 0.0


# ---------------------------------------------------------------- conv / D / gate
def test_conv_onehot_taps_shift():
    """A one-hot tap k picks the input K-1-k tokens back (zero before the start)."""
    rng = np.random.default_rng(3)
    Bt, L, d, K = 2, 11, 4, 4
    x = rng.standard_normal((Bt, L, d))
    for k in range(K):
        w = np.zeros((d, K))
        w[:, k] = 1.0
        xc = O.conv_silu(x, w, np.zeros(d))
        lag = K - 1 - k
        for t in range(L):
            src = x[:, t - lag, :] if t - lag >= 0 else np.zeros((Bt, d))
            np.testing.assert_allclose(xc[:, t, :], src / (1 + np.exp(-src)), rtol=1e-14, atol=0)


def test_conv_against_numpy_convolve():
    rng = np.random.default_rng(4)
    Bt, L, d, K = 2, 17, 5, 3
    x = rng.standard_normal((Bt, L, d))
    w = rng.standard_normal((d, K))
    b = rng.standard_normal(d)
    xc = O.conv_silu(x, w, b)
    for bb in range(Bt):
        for ch in range(d):
            # causal correlation: pre[t] = b + sum_k w[k] x[t-K+1+k]
            pre = np.convolve(x[bb, :, ch], w[ch, ::-1])[:L] + b[ch]
            np.testing.assert_allclose(xc[bb, :, ch], pre / (1 + np.exp(-pre)), rtol=1e-12, atol=1e-15)


def test_D_multiplies_conv_output_and_gate():
    """With C = 0 the output is D * SiLU(conv(x)) * SiLU(z): D acts on the conv output."""
    L, N, K = 7, 2, 4
    p = _mk(L, N, zoh=False, K=K, gate=True, seed=9)
    p["C"] = np.zeros_like(p["C"])
    y, _ = _run(p, False)
    xc = O.conv_silu(p["x"], p["conv_w"], p["conv_b"])
    z = p["z"]
    np.testing.assert_allclose(y, p["D"][None, None, :] * xc * z / (1 + np.exp(-z)), rtol=1e-13, atol=1e-16)


# ------------------------------------------------------ the page's checklist
def test_future_changes_leave_past_unchanged():
    L, N, K = 12, 3, 3
    p = _mk(L, N, zoh=True, K=K, gate=True, seed=21)
    y0, _ = _run(p, True)
    q = {k: (None if v is None else np.array(v, copy=True)) for k, v in p.items()}
    t0 = 5
    for key in ("x", "dt_raw", "z"):
        q[key][:, t0:, :] += 1.0
    for key in ("B", "C"):
        q[key][:, t0:, :] -= 0.5
    y1, _ = _run(q, True)
    np.testing.assert_array_equal(y0[:, :t0], y1[:, :t0])
    assert np.all(np.abs(y0[:, t0:] - y1[:, t0:]) > 0)


def test_conv_window_width3():
    """Changing token 2 changes conv outputs at tokens 2..4 only (width-3 window)."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((1, 6, 8))
    w = rng.uniform(0.2, 0.6, (8, 3))
    b = np.zeros(8)
    a = O.conv_silu(x, w, b)
    x2 = x.copy()
    x2[0, 2] += 1.0
    c = O.conv_silu(x2, w, b)
    np.testing.assert_array_equal(a[0, [0, 1, 5]], c[0, [0, 1, 5]])
    assert np.all(a[0, 2:5] != c[0, 2:5])


@pytest.mark.parametrize("zoh", [False, True])
def test_streaming_equals_full_forward(zoh):
    """Token streaming with the carried state (SSM state + K-1 conv inputs) equals the
    full forward, output by output and for the final state."""
    inp = SI.scan_inputs("teaching")
    kw = dict(A_log=inp["A_log"], D=inp["D"], dt_bias=inp["dt_bias"], conv_w=inp["conv_w"],
              conv_b=inp["conv_b"])
    y, h, hist = O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"],
                        dt_bias=inp["dt_bias"], zoh=zoh, conv_w=inp["conv_w"], conv_b=inp["conv_b"],
                        return_state=True)
    Bt, L, d = inp["x"].shape
    hs = np.zeros((Bt, d, inp["N"]))
    cs = np.zeros((Bt, d, inp["K"] - 1))
    assert hs.size == 24 and cs.size == 16
    for t in range(L):
        yt, hs, cs = O.step(inp["x"][:, t], inp["dt"][:, t], inp["B"][:, t], inp["C"][:, t], h=hs,
                            conv_state=cs, z_t=inp["z"][:, t], zoh=zoh, **kw)
        np.testing.assert_allclose(yt, y[:, t], rtol=1e-15, atol=0)
    np.testing.assert_allclose(hs, h, rtol=1e-15, atol=0)
    np.testing.assert_allclose(cs, hist, rtol=0, atol=0)
    np.testing.assert_array_equal(cs[0, :, -1], inp["x"][0, -1].astype(np.float64))


def test_resume_from_state_equals_full_scan():
    inp = SI.scan_inputs("mamba_mini", Bt=2, L=50, d=16)
    args = (inp["A_log"], )
    full_y, full_h = O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"],
                            dt_bias=inp["dt_bias"], conv_w=inp["conv_w"], conv_b=inp["conv_b"])
    L1 = 23
    sl = lambda a: a[:, :L1]
    sr = lambda a: a[:, L1:]
    y1, h1, hist1 = O.scan(sl(inp["x"]), sl(inp["dt"]), inp["A_log"], sl(inp["B"]), sl(inp["C"]), inp["D"],
                           z=sl(inp["z"]), dt_bias=inp["dt_bias"], conv_w=inp["conv_w"], conv_b=inp["conv_b"],
                           return_state=True)
    y2, h2 = O.scan(sr(inp["x"]), sr(inp["dt"]), inp["A_log"], sr(inp["B"]), sr(inp["C"]), inp["D"],
                    z=sr(inp["z"]), dt_bias=inp["dt_bias"], conv_w=inp["conv_w"], conv_b=inp["conv_b"],
                    h_init=h1, conv_hist=hist1)
    assert args
    np.testing.assert_allclose(np.concatenate([y1, y2], axis=1), full_y, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(h2, full_h, rtol=1e-13, atol=1e-15)


def test_channel_subset_equals_full():
    inp = SI.scan_inputs("mamba_mini", Bt=3, L=20, d=32)
    y, h = O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"],
                  dt_bias=inp["dt_bias"], conv_w=inp["conv_w"], conv_b=inp["conv_b"], threads=3)
    ch = np.array([[0, 5], [2, 31], [1, 0]])
    ys, hs = O.scan(inp["x"], inp["dt"], inp["A_log"], inp["B"], inp["C"], inp["D"], z=inp["z"],
                    dt_bias=inp["dt_bias"], conv_w=inp["conv_w"], conv_b=inp["conv_b"], channels=ch)
    for i, (b, dd) in enumerate(ch):
        np.testing.assert_array_equal(ys[i], y[b, :, dd])
        np.testing.assert_array_equal(hs[i], h[b, dd])
