"""Pins of the oracle's backward pass (oracle.scan_bwd) -- CPU only.

The gradients are fixed by the forward oracle alone: for the loss
sum(dy * y), every partial derivative must equal the central difference of
the forward scan with respect to that one input element.  This checks every
gradient output (u, dt_raw, z, B, C, A_log, D, dt_bias and the start state)
element by element, in both write modes, with and without the gate.
"""
import numpy as np
import pytest

from oracle import s6_oracle as O


def _problem(seed, Bt=2, L=6, d=3, N=4):
    rng = np.random.default_rng(seed)
    p = {
        "u": rng.standard_normal((Bt, L, d)),
        "dt": 0.5 * rng.standard_normal((Bt, L, d)) - 1.0,
        "z": rng.standard_normal((Bt, L, d)),
        "B": rng.standard_normal((Bt, L, N)),
        "C": rng.standard_normal((Bt, L, N)),
        "A_log": np.log(rng.uniform(0.5, 4.0, (d, N))),
        "D": rng.uniform(0.5, 1.5, d),
        "dt_bias": rng.uniform(-0.5, 0.5, d),
        "h_init": rng.standard_normal((Bt, d, N)),
    }
    dy = rng.standard_normal((Bt, L, d))
    return p, dy


def _loss(p, dy, zoh, gate):
    y, _ = O.scan(p["u"], p["dt"], p["A_log"], p["B"], p["C"], p["D"], z=p["z"] if gate else None,
                  dt_bias=p["dt_bias"], zoh=zoh, h_init=p["h_init"], threads=1)
    return float(np.sum(y * dy))


def _analytic(p, dy, zoh, gate):
    g = O.scan_bwd(p["u"], p["dt"], p["A_log"], p["B"], p["C"], p["D"], dy, z=p["z"] if gate else None,
                   dt_bias=p["dt_bias"], zoh=zoh, h_init=p["h_init"], threads=1)
    return {"u": g["du"], "dt": g["ddt"], "z": g["dz"], "B": g["dB"], "C": g["dC"], "A_log": g["dA_log"],
            "D": g["dD"], "dt_bias": g["ddt_bias"], "h_init": g["dh_init"]}


def check_gradients_by_central_differences(zoh, gate, seed=3):
    p, dy = _problem(seed)
    an = _analytic(p, dy, zoh, gate)
    names = ["u", "dt", "B", "C", "A_log", "D", "dt_bias", "h_init"] + (["z"] if gate else [])
    for name in names:
        base = p[name]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            eps = 1e-6 * max(1.0, abs(base[idx]))
            q = dict(p)
            q[name] = base.copy()
            q[name][idx] = base[idx] + eps
            lp = _loss(q, dy, zoh, gate)
            q[name][idx] = base[idx] - eps
            lm = _loss(q, dy, zoh, gate)
            fd[idx] = (lp - lm) / (2 * eps)
        err = np.max(np.abs(fd - an[name]) / (1.0 + np.abs(fd)))
        assert err < 1e-6, f"{name} (zoh={zoh}, gate={gate}): max rel diff {err:.2e}"
    if not gate:
        assert _analytic(p, dy, zoh, gate)["z"] is None


@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("gate", [True, False])
def test_gradients_equal_central_differences(zoh, gate):
    check_gradients_by_central_differences(zoh, gate)


def test_sigmoid_and_dsilu_closed_forms():
    assert O.sigmoid(0.0) == 0.5
    assert O.dsilu(0.0) == 0.5
    for v in (-30.0, -2.5, -0.1, 0.3, 4.0, 30.0):
        h = 1e-6
        # sigmoid is the derivative of softplus, dsilu the derivative of SiLU
        assert abs(O.sigmoid(v) - (O.softplus(v + h) - O.softplus(v - h)) / (2 * h)) < 1e-8
        assert abs(O.dsilu(v) - (O.silu(v + h) - O.silu(v - h)) / (2 * h)) < 1e-8
        assert abs(O.sigmoid(v) + O.sigmoid(-v) - 1.0) < 1e-15


def test_gradient_of_linear_readout_is_state():
    """dC is sum_d (dy * gate) * h: with D = 0, no gate and one channel it is
    exactly dy_t * h_t, whose h_t the forward oracle gives."""
    p, dy = _problem(5, Bt=1, L=4, d=1, N=3)
    p["D"] = np.zeros(1)
    g = O.scan_bwd(p["u"], p["dt"], p["A_log"], p["B"], p["C"], p["D"], dy, dt_bias=p["dt_bias"],
                   h_init=p["h_init"], threads=1)
    for t in range(4):
        _, h_t = O.scan(p["u"][:, :t + 1], p["dt"][:, :t + 1], p["A_log"], p["B"][:, :t + 1], p["C"][:, :t + 1],
                        p["D"], dt_bias=p["dt_bias"], h_init=p["h_init"], threads=1)
        np.testing.assert_allclose(g["dC"][0, t], dy[0, t, 0] * h_t[0, 0], rtol=1e-14, atol=1e-15)


def check_fused_gradients_by_central_differences(zoh, seed=4):
    """The fused path (conv + SiLU, then the scan): every gradient, including
    those of x, conv_w and conv_b, equals the central difference of the fused
    forward oracle."""
    p, dy = _problem(seed, Bt=2, L=6, d=2, N=3)
    rng = np.random.default_rng(seed + 9)
    K = 3
    p["x"] = p.pop("u")
    p["conv_w"] = rng.uniform(-0.8, 0.8, (2, K))
    p["conv_b"] = rng.uniform(-0.3, 0.3, 2)

    def loss(q):
        y, _ = O.scan(q["x"], q["dt"], q["A_log"], q["B"], q["C"], q["D"], z=q["z"], dt_bias=q["dt_bias"], zoh=zoh,
                      conv_w=q["conv_w"], conv_b=q["conv_b"], h_init=q["h_init"], threads=1)
        return float(np.sum(y * dy))

    g = O.conv_scan_bwd(p["x"], p["conv_w"], p["conv_b"], p["dt"], p["A_log"], p["B"], p["C"], p["D"], dy,
                        z=p["z"], dt_bias=p["dt_bias"], zoh=zoh, h_init=p["h_init"], threads=1)
    an = {"x": g["dx"], "conv_w": g["dconv_w"], "conv_b": g["dconv_b"], "dt": g["ddt"], "z": g["dz"], "B": g["dB"],
          "C": g["dC"], "A_log": g["dA_log"], "D": g["dD"], "dt_bias": g["ddt_bias"], "h_init": g["dh_init"]}
    for name, ref in an.items():
        base = p[name]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            eps = 1e-6 * max(1.0, abs(base[idx]))
            q = dict(p)
            q[name] = base.copy()
            q[name][idx] = base[idx] + eps
            lp = loss(q)
            q[name][idx] = base[idx] - eps
            lm = loss(q)
            fd[idx] = (lp - lm) / (2 * eps)
        err = np.max(np.abs(fd - ref) / (1.0 + np.abs(fd)))
        assert err < 1e-6, f"{name} (zoh={zoh}): max rel diff {err:.2e}"


@pytest.mark.parametrize("zoh", [False, True])
def test_fused_gradients_equal_central_differences(zoh):
    check_fused_gradients_by_central_differences(zoh)
