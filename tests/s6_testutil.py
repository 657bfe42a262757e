"""Helpers shared by the GPU parity tests: move seeded inputs to the device,
call the CUDA path, call the oracle on the same values, compare."""
from __future__ import annotations

import numpy as np

import s6_inputs as SI

# max |y - y_ref| <= TOL * (1 + |y_ref|), per element, for outputs and h_final
TOL = {"f32": 1e-4, "bf16": 1e-2}


def to_dev(a, device="cuda"):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


def from_dev(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def as_f64(a) -> np.ndarray:
    return SI.as_float(a).astype(np.float64)


def dev_inputs(inp: dict, device="cuda") -> dict:
    keys = ("x", "z", "B", "C", "dt", "A_log", "D", "dt_bias", "conv_w", "conv_b")
    return {k: to_dev(inp[k], device) for k in keys}


def rel_err(got, ref) -> float:
    """max |got - ref| / (1 + |ref|)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(got - ref) / (1.0 + np.abs(ref))))


# largest error seen per quantity in this session (printed in the terminal summary)
OBSERVED = {}


def note(key, err):
    OBSERVED[key] = max(OBSERVED.get(key, 0.0), float(err))


def assert_close(got, ref, io, what=""):
    err = rel_err(got, ref)
    note(f"{what} ({io})", err)
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), f"{what}: non-finite values"
    assert err <= TOL[io], f"{what}: max|got-ref|/(1+|ref|) = {err:.3e} > {TOL[io]:.0e}"
    return err


def sample_channels(Bt, d, n, seed=0, include_edges=True):
    rng = np.random.default_rng(seed)
    ch = np.stack([rng.integers(0, Bt, n), rng.integers(0, d, n)], axis=1)
    if include_edges:
        edges = np.array([[0, 0], [Bt - 1, d - 1], [0, d - 1], [Bt - 1, 0]])
        ch = np.concatenate([edges, ch])
    return ch
