"""Pins of the oracle's weight-clipping search (mudrobot.github.io AWQ notes,
"searching the optimal scale": weight clipping applied to minimise the
quantisation MSE).  Reading: per (group, column) and clip ratio c, the group
maximum m becomes fl32(c m) before delta = m / qmax, codes are clamped to
+-qmax, and the objective is the squared error of that group's share of the
layer output.

The pins check the oracle against what the quantiser's definition and exact
algebra fix, not against itself: the identity at c = 1, a group worked by
hand, the clamp of the group maximum, an independent numpy evaluation of the
losses from the returned codes, the single-group identity with the search
loss, and the argmin rule.
"""
import numpy as np
import pytest
import torch

import oracle
from post_weight_only_b200 import synth


def _layer(N, D_in, D_out, seed):
    return synth.layer_inputs(synth.small_layer(N, D_in, D_out, seed=seed))


def test_clip_grid_endpoints():
    g = synth.clip_grid(20).numpy()
    assert g.shape == (21,) and g[0] == 1.0 and g[-1] == 0.5
    assert np.all(np.diff(g) < 0)


def test_clip_one_is_the_unclipped_quantiser():
    X, W = _layer(8, 256, 40, seed=1)
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.6)
    q0, d0 = oracle.quantize(W, s, 4, 128)
    q1, d1 = oracle.quantize(W, s, 4, 128, clip=np.ones((2, 40), np.float32))
    assert np.array_equal(q0, q1) and np.array_equal(d0, d1)


def test_hand_worked_group():
    """w' = [7, 1, ..., 1] (s = 1), 4 bits (qmax = 7), one token of ones:
    c = 1:    delta = 1,    q = [7, 1, ...],  error 0,                 loss 0
    c = 0.5:  delta = 0.5,  q_0 = clamp(14) = 7 -> 3.5 (error -3.5),
              others 1 / 0.5 = 2 -> 1 exactly,                          loss 12.25
    c = 0.75: delta = 0.75, q_0 = clamp(rne(9.33)) = 7 -> 5.25 (-1.75),
              others rne(1.33) = 1 -> 0.75 (-0.25 each, 31 of them),
              y = -1.75 - 7.75 = -9.5,                                   loss 90.25"""
    W = np.ones((32, 1), np.float32)
    W[0, 0] = 7.0
    X = torch.ones(1, 32, dtype=torch.bfloat16)
    grid = np.array([1.0, 0.5, 0.75], np.float32)
    best, loss = oracle.clip_search(X, W, None, grid, 4, 32, want_loss=True)
    assert loss[:, 0, 0].tolist() == [0.0, 12.25, 90.25]
    assert best[0, 0] == 0
    q, d = oracle.quantize(W, None, 4, 32, clip=np.full((1, 1), 0.5, np.float32))
    assert d[0, 0] == 0.5 and q[0, 0] == 7 and np.all(q[1:, 0] == 2)


def test_group_maximum_codes_to_qmax_and_codes_bounded():
    X, W = _layer(4, 256, 64, seed=2)
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.5)
    wp = s[:, None].astype(np.float32) * W.numpy()
    for bits in (4, 3):
        qmax = 2 ** (bits - 1) - 1
        for c in synth.clip_grid(20).numpy():
            q, d = oracle.quantize(W, s, bits, 64, clip=np.full((4, 64), c, np.float32))
            assert np.abs(q).max() <= qmax
            for g in range(4):
                blk = wp[g * 64:(g + 1) * 64]
                k = np.abs(blk).argmax(axis=0)
                cols = np.arange(64)
                assert np.array_equal(q[g * 64 + k, cols], np.sign(blk[k, cols]).astype(np.int8) * qmax)


@pytest.mark.parametrize("bits,group", [(4, 128), (3, 64), (4, 32)])
def test_losses_against_numpy_from_codes(bits, group):
    """Each group's loss re-evaluated with numpy (fp64 matmul) from the codes
    and deltas of the clipped quantiser."""
    N, D_in, D_out = 24, 256, 12
    X, W = _layer(N, D_in, D_out, seed=3 + group)
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.45)
    grid = synth.clip_grid(10).numpy()
    best, loss = oracle.clip_search(X, W, s, grid, bits, group, want_loss=True)
    G = D_in // group
    x = X.float().numpy().astype(np.float64)
    w = W.numpy().astype(np.float64)
    for i, c in enumerate(grid):
        q, d = oracle.quantize(W, s, bits, group, clip=np.full((G, D_out), c, np.float32))
        e = q.astype(np.float64) * np.repeat(d, group, axis=0).astype(np.float64) / s.astype(np.float64)[:, None] - w
        for g in range(G):
            sl = slice(g * group, (g + 1) * group)
            ref = ((x[:, sl] @ e[sl]) ** 2).sum(axis=0)
            assert np.allclose(loss[i, g], ref, rtol=1e-12, atol=1e-300)
    # the argmin rule: the smallest loss, the lowest grid index among equals
    for g in range(G):
        for n in range(D_out):
            col = loss[:, g, n]
            assert best[g, n] == int(np.flatnonzero(col == col.min())[0])


def test_single_group_matches_the_search_loss():
    """With one group per column the group's output error is the column's
    whole loss, so c = 1 reproduces the search oracle's column loss."""
    X, W = _layer(40, 128, 16, seed=5)
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.3)
    _, loss = oracle.clip_search(X, W, s, np.array([1.0], np.float32), 4, 128, want_loss=True)
    assert np.allclose(loss[0, 0], oracle.loss_cols(X, W, s, 4, 128), rtol=1e-12)


def test_columns_subset():
    X, W = _layer(16, 256, 20, seed=6)
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.5)
    grid = synth.clip_grid(20).numpy()
    b_all, l_all = oracle.clip_search(X, W, s, grid, 4, 128, want_loss=True)
    cols = np.array([0, 7, 19])
    b_sub, l_sub = oracle.clip_search(X, W, s, grid, 4, 128, cols=cols, want_loss=True)
    assert np.array_equal(b_sub, b_all[:, cols]) and np.array_equal(l_sub, l_all[:, :, cols])
