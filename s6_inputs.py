"""Seeded synthetic inputs for the S6 selective scan -- shared by the tests,
the benchmark and the smoke check.

This module holds no step of the method: it only draws numbers (numpy PCG64)
and rounds them to the storage type.  Both the CUDA path and the CPU oracle
read exactly the arrays produced here.  The one non-trivial expression, the
inverse softplus ``log(expm1(y))``, belongs to the input *recipe* (step sizes
drawn uniformly in [0.001, 0.1] after the softplus), not to the method.

Storage convention: ``io="f32"`` arrays are float32; ``io="bf16"`` arrays are
uint16 bfloat16 bit patterns (round-to-nearest-even from the float32 draw).
Parameters (A_log, D, dt_bias, conv weights) are always float32.

Workloads (shapes and value distributions follow the pages' two model sizes:
the TinyMamba teaching block of "Carry context through a selective state" and
the Mamba-mini block of "mamba, live" / "two recurrences"):

  teaching   Bt1 L6 d8 N3 K3, fp32, seed 0
  mamba_mini Bt8 L256 d1536 N16 K4, fp32, seed 2
  decode     256 sequences x 6 blocks x d1536 x N16, K4, fp32 state, seed 3
  long_seq   Bt16 L8192 d1536 N16 K4, bf16 I/O, seed 4
  wide       Bt4 L2048 d5120 N16 K4, bf16 I/O, exact ZOH, seed 5

The constant-decay cell ("the s6 cell", one cell, two architectures) reads the
same u, z, B, C draws plus a per-(channel, state) constant decay drawn by
``diag_log2_decay``.
"""
from __future__ import annotations

import numpy as np

CONFIGS = {
    "teaching": dict(Bt=1, L=6, d=8, N=3, K=3, io="f32", zoh=None, gate=True, dist="teaching", seed=0),
    "mamba_mini": dict(Bt=8, L=256, d=1536, N=16, K=4, io="f32", zoh=None, gate=True, dist="mamba_mini",
                       seed=2),
    "decode": dict(Bt=256, blocks=6, steps=1024, d=1536, N=16, K=4, io="f32", zoh=False, gate=True,
                   dist="mamba_mini", seed=3),
    "long_seq": dict(Bt=16, L=8192, d=1536, N=16, K=4, io="bf16", zoh=False, gate=True, dist="mamba_mini",
                     seed=4),
    "wide": dict(Bt=4, L=2048, d=5120, N=16, K=4, io="bf16", zoh=True, gate=True, dist="wide", seed=5),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even (NaN not expected)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_storage(a: np.ndarray, io: str) -> np.ndarray:
    if io == "f32":
        return np.ascontiguousarray(a, dtype=np.float32)
    if io == "bf16":
        return f32_to_bf16_bits(np.asarray(a, dtype=np.float32))
    raise ValueError(io)


def as_float(a: np.ndarray) -> np.ndarray:
    """Storage array -> float32 values (exact)."""
    a = np.asarray(a)
    return bf16_bits_to_f32(a) if a.dtype == np.uint16 else a.astype(np.float32)


def _normal(rng, shape, scale=1.0):
    out = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        out *= np.float32(scale)
    return out


def _inv_softplus(y):
    y = np.asarray(y, dtype=np.float64)
    return np.log(np.expm1(y))


def params(rng, d, N, K, dist, random_A=False):
    """Per-channel parameters: A_log [d,N], D [d], dt_bias [d], conv_w [d,K], conv_b [d]."""
    if random_A:
        A_log = np.log(rng.uniform(0.5, 16.0, size=(d, N))).astype(np.float32)
    else:
        A_log = np.tile(np.log(np.arange(1, N + 1, dtype=np.float64)), (d, 1)).astype(np.float32)
    if dist == "teaching":
        D = np.ones(d, np.float32)
        dt_bias = np.zeros(d, np.float32)
    elif dist == "mamba_mini":
        D = rng.uniform(0.5, 1.5, size=d).astype(np.float32)
        dt_bias = _inv_softplus(rng.uniform(0.001, 0.1, size=d)).astype(np.float32)
    elif dist == "wide":
        D = rng.uniform(0.5, 1.5, size=d).astype(np.float32)
        dt_bias = np.zeros(d, np.float32)
    else:
        raise ValueError(dist)
    bound = 1.0 / np.sqrt(K) if K > 0 else 1.0
    conv_w = rng.uniform(-bound, bound, size=(d, K)).astype(np.float32)
    conv_b = rng.uniform(-bound, bound, size=d).astype(np.float32)
    return dict(A_log=A_log, D=D, dt_bias=dt_bias, conv_w=conv_w, conv_b=conv_b)


def scan_inputs(name: str = None, *, seed=None, random_A=False, **over):
    """Inputs of a full-sequence workload: x, z, B, C, dt ([Bt,L,d] / [Bt,L,N]) + params.

    Any of Bt, L, d, N, K, io, dist may be overridden (smaller or ragged cases keep
    the named workload's value distributions).  Draw order: x, z, B, C, dt, params.
    """
    cfg = dict(CONFIGS[name]) if name else {}
    cfg.update(over)
    Bt, L, d, N, K, io, dist = (cfg[k] for k in ("Bt", "L", "d", "N", "K", "io", "dist"))
    rng = np.random.default_rng(cfg["seed"] if seed is None else seed)
    x = _normal(rng, (Bt, L, d))
    z = _normal(rng, (Bt, L, d))
    Bm = _normal(rng, (Bt, L, N))
    Cm = _normal(rng, (Bt, L, N))
    if dist == "teaching":
        dt = _normal(rng, (Bt, L, d))
    elif dist == "mamba_mini":
        dt = _normal(rng, (Bt, L, d), 0.5)
    else:  # wide: Delta = softplus(dt_raw) lands in [0.001, 0.1]
        dt = _inv_softplus(rng.uniform(0.001, 0.1, size=(Bt, L, d))).astype(np.float32)
    p = params(rng, d, N, K, dist, random_A=random_A)
    out = dict(x=to_storage(x, io), z=to_storage(z, io), B=to_storage(Bm, io), C=to_storage(Cm, io),
               dt=to_storage(dt, io), io=io, Bt=Bt, L=L, d=d, N=N, K=K)
    out.update(p)
    return out


def decode_params(block: int, *, d=1536, N=16, K=4, seed=3, random_A=False):
    """Parameters of one block of the streaming-decode workload."""
    rng = np.random.default_rng([seed, 1000 + block])
    return params(rng, d, N, K, "mamba_mini", random_A=random_A)


def decode_tokens(step: int, block: int, *, Bt=256, d=1536, N=16, seed=3, io="f32"):
    """Per-token inputs of one (step, block): x_t, z_t, dt_t [Bt,d]; B_t, C_t [Bt,N]."""
    rng = np.random.default_rng([seed, step, block])
    x = _normal(rng, (Bt, d))
    z = _normal(rng, (Bt, d))
    Bm = _normal(rng, (Bt, N))
    Cm = _normal(rng, (Bt, N))
    dt = _normal(rng, (Bt, d), 0.5)
    return dict(x=to_storage(x, io), z=to_storage(z, io), B=to_storage(Bm, io), C=to_storage(Cm, io),
                dt=to_storage(dt, io))


def diag_log2_decay(d: int, N: int, seed: int = 6) -> np.ndarray:
    """log2 of constant decays a[d, n] ~ U[0.2, 0.999] (float32 [d, N], <= 0)."""
    rng = np.random.default_rng([seed, d, N])
    return np.log2(rng.uniform(0.2, 0.999, size=(d, N))).astype(np.float32)


# ------------------------------------------------------------ the decode block
# Mamba-mini ("mamba, live", what is actually running): d_model 384, d_inner
# 1536, N 16, dt rank 24, conv width 4, 6 blocks.  Weights are synthetic (no
# trained ones exist here), stored as that page's Weights paragraph says:
# per-row symmetric int8 with one float32 scale per output row; the scales
# give unit-variance inputs unit-variance outputs.
MAMBA_MINI_BLOCK = dict(dm=384, di=1536, N=16, R=24, K=4, blocks=6, eps=1e-5)


def _q8_rows(rng, n_out, n_in, gain=1.0):
    q = rng.integers(-127, 128, size=(n_out, n_in)).astype(np.int8)
    # std of U{-127..127} is about 73.6; scale so that Var(w) = gain^2 / n_in
    scale = (gain / (73.6 * np.sqrt(n_in)) * rng.uniform(0.8, 1.25, size=n_out)).astype(np.float32)
    return q, scale


def block_weights(block: int, *, dm=384, di=1536, N=16, R=24, K=4, seed=7):
    """Synthetic weights of one decode block (int8 rows x float32 scales)."""
    rng = np.random.default_rng([seed, block])
    in_q, in_s = _q8_rows(rng, 2 * di, dm)
    xp_q, xp_s = _q8_rows(rng, R + 2 * N, di)
    dt_q, dt_s = _q8_rows(rng, di, R, gain=0.5)
    out_q, out_s = _q8_rows(rng, dm, di, gain=0.5)
    p = params(rng, di, N, K, "mamba_mini")
    return dict(ln_w=(1.0 + 0.1 * rng.standard_normal(dm)).astype(np.float32),
                ln_b=(0.1 * rng.standard_normal(dm)).astype(np.float32),
                in_q=in_q, in_s=in_s, conv_w=p["conv_w"], conv_b=p["conv_b"], xp_q=xp_q, xp_s=xp_s,
                dt_q=dt_q, dt_s=dt_s, dt_bias=p["dt_bias"], A_log=p["A_log"], D=p["D"], out_q=out_q, out_s=out_s)


def block_tokens(step: int, *, Bt=256, dm=384, seed=8):
    """Residual-stream input of one decode step: x [Bt, dm] ~ N(0, 1) (float32)."""
    rng = np.random.default_rng([seed, step])
    return rng.standard_normal((Bt, dm)).astype(np.float32)
