"""GPU parity of s6_block_step against the float64 oracle's decode block.

One token through a Mamba-mini block ("mamba, live", what is actually
running; per-row int8 weights as its Weights paragraph says) for a batch of
sequences, stepped token by token through several blocks, compared element by
element with oracle.block_step on the same stored weights and inputs: the
residual stream x after every block and step, and the final h_ssm and conv
history.  Bound: max |got - ref| / (1 + |ref|) <= 1e-4 (float32 activations
and state; the projections sum up to 1536 float32 products).
"""
import numpy as np
import pytest

from oracle import s6_oracle as O
import s6_inputs as SI
from s6_testutil import assert_close, to_dev

pytestmark = pytest.mark.gpu


def _dev_weights(w):
    return {k: to_dev(np.ascontiguousarray(v)) for k, v in w.items()}


def _run(Bt, dm, di, N, R, K, blocks, steps, seed, tol_key="f32"):
    import selective_state_space_19_b200 as S
    import torch
    ws = [SI.block_weights(b, dm=dm, di=di, N=N, R=R, K=K, seed=seed) for b in range(blocks)]
    wd = [_dev_weights(w) for w in ws]
    cs = [torch.zeros(Bt, di, K - 1, device="cuda") for _ in range(blocks)]
    hs = [torch.zeros(Bt, di, N, device="cuda") for _ in range(blocks)]
    rcs = [np.zeros((Bt, di, K - 1)) for _ in range(blocks)]
    rhs = [np.zeros((Bt, di, N)) for _ in range(blocks)]
    for t in range(steps):
        x0 = SI.block_tokens(t, Bt=Bt, dm=dm, seed=seed + 1)
        x = to_dev(x0)
        rx = x0.astype(np.float64)
        for b in range(blocks):
            S.s6_block_step(x, cs[b], hs[b], wd[b])
            rx, rcs[b], rhs[b] = O.block_step(rx, rcs[b], rhs[b], ws[b])
            torch.cuda.synchronize()
            assert_close(x.cpu().numpy(), rx, tol_key, "block x")
    assert S.s6_device_status() == 0
    for b in range(blocks):
        assert_close(hs[b].cpu().numpy(), rhs[b], tol_key, "block h_ssm")
        assert_close(cs[b].cpu().numpy(), rcs[b], tol_key, "block conv_state")


def test_block_small_dims():
    _run(Bt=5, dm=64, di=256, N=16, R=8, K=4, blocks=3, steps=4, seed=11)


def test_block_ragged_dims():
    """di not a multiple of the tiles, more than one 64-row tile of sequences,
    N = 8, conv width 3, an odd dt rank."""
    _run(Bt=70, dm=96, di=200, N=8, R=5, K=3, blocks=2, steps=3, seed=12)


def test_block_single_sequence_and_tile_edges():
    """One sequence (a single, mostly empty row tile of the products), then 65
    sequences (one row past a tile); d_model 48 and d_inner 80 leave the
    tensor-core products' K (48, 80) a multiple of 16 with N (160, 48) not a
    multiple of the 64-wide output tile."""
    _run(Bt=1, dm=48, di=80, N=16, R=4, K=4, blocks=2, steps=3, seed=15)
    _run(Bt=65, dm=48, di=80, N=16, R=4, K=2, blocks=2, steps=2, seed=16)


def test_block_xproj_row_paths():
    """d_inner 1600 (x_proj rows longer than the 12 x 128 channels a lane
    holds in registers) and 90 (rows not a multiple of 4 channels): the x_proj
    loops that stream a row from the L2, in front of the fused recurrence."""
    _run(Bt=3, dm=40, di=1600, N=16, R=6, K=4, blocks=1, steps=2, seed=17)
    _run(Bt=3, dm=40, di=90, N=16, R=6, K=4, blocks=1, steps=2, seed=18)


def test_block_product_epilogue_paths():
    """The tensor-core product's split-reduction adds: 8-byte atomics on rows
    of an even length (every test above), and single floats where d_model 45
    makes out_proj's rows (the residual stream, K = d_inner 96 on the tensor
    cores) only 4-byte aligned."""
    _run(Bt=5, dm=45, di=96, N=16, R=4, K=4, blocks=2, steps=2, seed=19)
    _run(Bt=70, dm=40, di=128, N=16, R=8, K=4, blocks=1, steps=2, seed=20)


def test_block_mamba_mini_dims():
    """The Mamba-mini block (d_model 384, d_inner 1536, N 16, dt rank 24, conv 4)
    through all 6 blocks for 6 tokens, on a 16-sequence batch."""
    _run(Bt=16, dm=384, di=1536, N=16, R=24, K=4, blocks=6, steps=6, seed=13)


def test_block_decode_batch_one_step():
    """The decode workload's batch (256 sequences) through the 6 blocks, one
    token from zero states, every output element."""
    _run(Bt=256, dm=384, di=1536, N=16, R=24, K=4, blocks=6, steps=1, seed=14)


def test_block_rejects_bad_arguments():
    import selective_state_space_19_b200 as S
    import torch
    w = _dev_weights(SI.block_weights(0, dm=32, di=64, N=16, R=4, K=4))
    x = torch.zeros(2, 32, device="cuda")
    cs = torch.zeros(2, 64, 3, device="cuda")
    h = torch.zeros(2, 64, 16, device="cuda")
    with pytest.raises(S.S6Error) as e:
        S.s6_block_step(x, cs, h, w, eps=-1.0)
    assert e.value.status == S.S6_ERR_INVALID_ARG
    w2 = dict(w)
    w2.pop("_abi", None)
    w2["xp_q"] = None
    with pytest.raises(S.S6Error) as e:
        S.s6_block_step(x, cs, h, w2)
    assert e.value.status == S.S6_ERR_INVALID_ARG
