"""Pins of the oracle's decode block (CPU only).

"mamba, live", section *what is actually running*: one token through a block
is LayerNorm -> in_proj (-> xin, z) -> conv + SiLU -> x_proj (-> dt, B, C) ->
dt_proj + softplus -> the recurrence -> readout -> gate -> out_proj -> residual
add, with weights stored as per-row symmetric int8 times a float32 scale
(*Weights*).  The pins: a worked example small enough to follow by hand, the
block over a sequence rebuilt from independent pieces (numpy's mean, variance
and matrix products around the already pinned scan and conv oracles), and the
int8 linear and LayerNorm against numpy.
"""
import math

import numpy as np

from oracle import s6_oracle as O
import s6_inputs as SI


def _tiny():
    """dm 2, di 1, N 1, dt rank 1, conv width 2 -- every number chosen by hand."""
    return dict(ln_w=np.array([1.0, 1.0]), ln_b=np.array([0.0, 0.0]),
                in_q=np.array([[1, 2], [0, 1]], np.int8), in_s=np.array([0.5, 1.0]),
                conv_w=np.array([[0.5, 2.0]]), conv_b=np.array([0.0]),
                xp_q=np.array([[2], [4], [-1]], np.int8), xp_s=np.array([0.25, 0.5, 1.0]),
                dt_q=np.array([[1]], np.int8), dt_s=np.array([1.0]), dt_bias=np.array([0.1]),
                A_log=np.array([[0.0]]), D=np.array([1.0]),
                out_q=np.array([[1], [-2]], np.int8), out_s=np.array([1.0, 0.5]))


def test_block_worked_example():
    """x = (1, 3): LayerNorm (eps 0) gives (-1, 1); in_proj rows (1, 2)*0.5 and
    (0, 1)*1 give xin = 0.5, z = 1; the conv (taps 0.5, 2; history 0.4) gives
    pre = 0.2 + 1.0 = 1.2 and xc = SiLU(1.2); x_proj gives dt = xc/2, B = 2 xc,
    C = -xc; Delta = softplus(xc/2 + 0.1); A = -1; from h = 0.3 the state is
    e^-Delta * 0.3 + Delta * B * xc; y = h C + xc; the gate multiplies by
    SiLU(1); out_proj rows 1 and -2*0.5 add (g, -g) to x."""
    xc = 1.2 / (1.0 + math.exp(-1.2))                       # 0.92223...
    delta = math.log1p(math.exp(0.5 * xc + 0.1))           # softplus(0.56111...)
    h = math.exp(-delta) * 0.3 + delta * (2.0 * xc) * xc
    y = h * (-xc) + 1.0 * xc
    g = y * (1.0 / (1.0 + math.exp(-1.0)))
    x1, cs1, h1 = O.block_step(np.array([[1.0, 3.0]]), np.array([[[0.4]]]), np.array([[[0.3]]]), _tiny(), eps=0.0)
    assert abs(xc - 0.922230) < 1e-6
    np.testing.assert_allclose(x1[0], [1.0 + g, 3.0 - g], rtol=1e-14)
    np.testing.assert_allclose(h1[0, 0, 0], h, rtol=1e-14)
    assert cs1[0, 0, 0] == 0.5  # the history now holds xin


def _sequence_form(xs, w, eps=1e-5):
    """The block applied to a whole sequence of residual inputs xs [Bt, L, dm]
    from zero states, from independent pieces: numpy for the LayerNorm and the
    int8 linears, the pinned conv and scan oracles for the rest."""
    f = lambda a: np.asarray(a, dtype=np.float64)
    deq = lambda q, s: f(q) * f(s)[:, None]
    di, N = np.asarray(w["A_log"]).shape
    R = np.asarray(w["dt_q"]).shape[1]
    mu = xs.mean(axis=-1, keepdims=True)
    var = ((xs - mu) ** 2).mean(axis=-1, keepdims=True)
    hn = (xs - mu) / np.sqrt(var + eps) * f(w["ln_w"]) + f(w["ln_b"])
    xz = hn @ deq(w["in_q"], w["in_s"]).T
    xin, z = xz[..., :di], xz[..., di:]
    xc = O.conv_silu(xin, w["conv_w"], w["conv_b"])
    dbc = xc @ deq(w["xp_q"], w["xp_s"]).T
    dtr = dbc[..., :R] @ deq(w["dt_q"], w["dt_s"]).T
    Bm, Cm = dbc[..., R:R + N], dbc[..., R + N:]
    g, h = O.scan(xc, dtr, w["A_log"], Bm, Cm, w["D"], z=z, dt_bias=w["dt_bias"])
    return xs + g @ deq(w["out_q"], w["out_s"]).T, h


def test_block_streaming_equals_sequence_form():
    Bt, L = 2, 6
    w = SI.block_weights(3, dm=8, di=16, N=4, R=2, K=4)
    xs = np.stack([SI.block_tokens(t, Bt=Bt, dm=8) for t in range(L)], axis=1).astype(np.float64)
    ref_x, ref_h = _sequence_form(xs, w)
    cs = np.zeros((Bt, 16, 3))
    h = np.zeros((Bt, 16, 4))
    out = []
    for t in range(L):
        x1, cs, h = O.block_step(xs[:, t], cs, h, w)
        out.append(x1)
    np.testing.assert_allclose(np.stack(out, axis=1), ref_x, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(h, ref_h, rtol=1e-11, atol=1e-11)
    # the history holds the last K-1 xin values
    assert cs.shape == (Bt, 16, 3)


def test_linear_q8_against_numpy():
    rng = np.random.default_rng(1)
    q = rng.integers(-127, 128, size=(7, 5)).astype(np.int8)
    s = rng.uniform(0.01, 0.1, size=7)
    x = rng.standard_normal((3, 5))
    np.testing.assert_allclose(O.linear_q8(q, s, x), x @ (q.astype(np.float64) * s[:, None]).T, rtol=1e-13)


def test_layernorm_against_numpy():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((4, 384)) * 3 + 1
    y = O.layernorm(x, np.ones(384), np.zeros(384), eps=0.0)
    np.testing.assert_allclose(y.mean(axis=-1), 0.0, atol=1e-13)
    np.testing.assert_allclose(y.var(axis=-1), 1.0, rtol=1e-12)
    w, b = rng.standard_normal(384), rng.standard_normal(384)
    np.testing.assert_allclose(O.layernorm(x, w, b, eps=1e-5),
                               (x - x.mean(-1, keepdims=True)) / np.sqrt(x.var(-1, keepdims=True) + 1e-5) * w + b,
                               rtol=1e-12, atol=1e-12)


def test_block_weights_are_int8_rows_with_scales():
    w = SI.block_weights(0)
    for k, shape in (("in_q", (3072, 384)), ("xp_q", (56, 1536)), ("dt_q", (1536, 24)), ("out_q", (384, 1536))):
        assert w[k].dtype == np.int8 and w[k].shape == shape
        assert w[k.replace("_q", "_s")].shape == (shape[0],)
    assert w["A_log"].dtype == np.float32 and w["A_log"].shape == (1536, 16)
