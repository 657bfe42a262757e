"""Pins of the oracle's constant-decay diagonal recurrence (CPU only).

"the s6 cell", *one cell, two architectures*: both recurrences reduce to
h <- a*h + b*u with a = 2^(negative); in the constant-decay cell a is a
per-(channel, state) constant 2^w (*the difference that no engineering
removes*: the decay can be precomputed once), the write is B_t * u_t, and the
readout is the S6 cell's, <h, C_t> + D*u, optionally gated by SiLU(z).

Each pin fixes the oracle by something other than itself: a brute-force
decayed sum written out independently, the geometric series of a held input,
the identity with the selective (live-decay) scan at a step size of exactly
one, and the streaming property (a scan continued from its own final state).
"""
import math

import numpy as np

from oracle import s6_oracle as O


def _inputs(Bt=2, L=7, d=3, N=4, seed=0, gate=True):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((Bt, L, d))
    z = rng.standard_normal((Bt, L, d)) if gate else None
    B = rng.standard_normal((Bt, L, N))
    C = rng.standard_normal((Bt, L, N))
    w = -rng.uniform(0.05, 3.0, size=(d, N))  # log2 of the decays, < 0
    D = rng.uniform(0.5, 1.5, size=d)
    return u, z, B, C, w, D


def test_diag_bruteforce_decayed_sum():
    """h_t[n] = sum_{s<=t} a[n]^(t-s) B_s[n] u_s, y_t = (<h_t, C_t> + D u_t) SiLU(z_t)."""
    u, z, B, C, w, D = _inputs()
    Bt, L, d = u.shape
    N = B.shape[2]
    y, h = O.diag_const(u, w, B, C, D, z=z)
    for b in range(Bt):
        for c in range(d):
            a = 2.0 ** w[c]
            for t in range(L):
                ht = np.zeros(N)
                for s in range(t + 1):
                    ht += a ** (t - s) * B[b, s] * u[b, s, c]
                gate = z[b, t, c] / (1.0 + math.exp(-z[b, t, c]))
                ref = (ht @ C[b, t] + D[c] * u[b, t, c]) * gate
                assert abs(y[b, t, c] - ref) <= 1e-12 * (1 + abs(ref))
            np.testing.assert_allclose(h[b, c], ht, rtol=1e-12, atol=1e-12)


def test_diag_geometric_series():
    """A held input through one state: h_t = b (1 - a^(t+1)) / (1 - a)."""
    L, a, b = 40, 0.8, 0.3
    u = np.ones((1, L, 1))
    B = np.full((1, L, 1), b)
    C = np.ones((1, L, 1))
    y, h = O.diag_const(u, np.array([[math.log2(a)]]), B, C, np.zeros(1))
    t = np.arange(L)
    np.testing.assert_allclose(y[0, :, 0], b * (1 - a ** (t + 1)) / (1 - a), rtol=1e-13)
    assert abs(h[0, 0, 0] - b * (1 - a ** L) / (1 - a)) < 1e-13


def test_diag_equals_selective_scan_at_unit_step():
    """With Delta = softplus(log(e - 1)) = 1 the selective scan's decay is
    exp(A) = 2^(A log2 e) and its write B*u: the constant cell with
    w = -exp(A_log) log2 e gives the same outputs."""
    u, z, B, C, _, D = _inputs(seed=3)
    Bt, L, d = u.shape
    N = B.shape[2]
    rng = np.random.default_rng(4)
    A_log = np.log(rng.uniform(0.5, 16.0, size=(d, N)))
    dt_raw = np.full((Bt, L, d), math.log(math.e - 1.0))
    ys, hs = O.scan(u, dt_raw, A_log, B, C, D, z=z, zoh=False)
    yd, hd = O.diag_const(u, -np.exp(A_log) * math.log2(math.e), B, C, D, z=z)
    np.testing.assert_allclose(yd, ys, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hd, hs, rtol=1e-12, atol=1e-12)


def test_diag_decays_in_unit_interval_and_state_bounded():
    """a = 2^w lies in (0, 1) for w < 0, so |h| <= max|B u| / (1 - max a)."""
    u, _, B, C, w, D = _inputs(Bt=1, L=300, d=2, N=3, seed=5, gate=False)
    a = 2.0 ** w
    assert np.all((a > 0) & (a < 1))
    y, h = O.diag_const(u, w, B, C, D)
    bound = np.max(np.abs(B[0][:, None, :] * u[0][:, :, None])) / (1 - a.max())
    assert np.all(np.abs(h) <= bound)
    assert np.all(np.isfinite(y))


def test_diag_streaming_continues_from_state():
    """Scanning [0, L1) then [L1, L) from the first part's final state equals one scan."""
    u, z, B, C, w, D = _inputs(L=11, seed=6)
    y, h = O.diag_const(u, w, B, C, D, z=z)
    y1, h1 = O.diag_const(u[:, :5], w, B[:, :5], C[:, :5], D, z=z[:, :5])
    y2, h2 = O.diag_const(u[:, 5:], w, B[:, 5:], C[:, 5:], D, z=z[:, 5:], h_init=h1)
    np.testing.assert_allclose(np.concatenate([y1, y2], axis=1), y, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(h2, h, rtol=1e-13, atol=1e-13)


def test_diag_channel_list_matches_full():
    u, z, B, C, w, D = _inputs(seed=7)
    y, h = O.diag_const(u, w, B, C, D, z=z)
    ch = np.array([[1, 2], [0, 0]])
    yc, hc = O.diag_const(u, w, B, C, D, z=z, channels=ch)
    np.testing.assert_array_equal(yc, np.stack([y[1, :, 2], y[0, :, 0]]))
    np.testing.assert_array_equal(hc, np.stack([h[1, 2], h[0, 0]]))
