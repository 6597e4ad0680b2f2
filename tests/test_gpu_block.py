"""A block's linears in one go (compassingai.com concept page, "full
scale-optimisation flow", final note: every linear searched independently):
`awq.quantize_block` (device buffers, one batched statistic and one batched
search) and `awq.quantize_block_host` (pinned host buffers in, host results
out, copies overlapped with compute and the layers run in an order of their
own) give bit for bit the results of the single-layer calls, in the layers'
given order; the host form reuses its state across calls; and one layer's
L(alpha) and alpha* are checked against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_bounds import check_alpha
from post_weight_only_b200 import synth

pytestmark = pytest.mark.gpu

GRID = [k / 20 for k in range(21)]


@pytest.fixture(scope="module")
def awq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from post_weight_only_b200 import awq as mod
    return mod


def _block(seed):
    """Two inputs and four linears of different widths, layer 1 the smallest and
    layer 3 the second smallest W (so the host form runs them first and last)."""
    x0, _ = synth.layer_inputs(synth.small_layer(300, 256, 8, seed=seed))
    x1, _ = synth.layer_inputs(synth.small_layer(300, 512, 8, seed=seed + 1))
    shapes = [(0, 256, 320), (0, 256, 64), (1, 512, 256), (0, 256, 132)]
    layers = []
    for i, (xi, d_in, d_out) in enumerate(shapes):
        _, w = synth.layer_inputs(synth.small_layer(8, d_in, d_out, seed=seed + 10 + i))
        layers.append((xi, w))
    return [x0, x1], layers


def _single(awq, xs, layers):
    out = []
    for xi, w in layers:
        x, wd = xs[xi].cuda(), w.cuda()
        a = awq.act_stats(x)
        r = awq.search(x, wd, a, GRID, 4, 128)
        s_star = awq.scales(a, r.alpha_star)
        packed, sc = awq.quantize_pack(wd, s_star, 4, 128)
        out.append((r.L.cpu(), r.alpha_star.cpu(), packed.cpu(), sc.cpu()))
    return out


def test_quantize_block_equals_single_layers(awq):
    xs, layers = _block(3)
    ref = _single(awq, xs, layers)
    res = awq.quantize_block([x.cuda() for x in xs], [(xi, w.cuda()) for xi, w in layers], GRID, 4, 128)
    torch.cuda.synchronize()
    for r, (L, a_star, packed, sc) in zip(res, ref):
        awq.check_device_status(r.search.status)
        assert torch.equal(r.search.L.cpu(), L)
        assert torch.equal(r.search.alpha_star.cpu(), a_star)
        assert torch.equal(r.packed.cpu(), packed)
        assert torch.equal(r.scales.cpu(), sc)


def test_quantize_block_host_equals_single_layers_and_reuses_state(awq):
    state = awq.BlockHostState()
    ws = awq.Workspace()
    for seed in (5, 6):                                   # the second call reuses buffers and streams
        xs, layers = _block(seed)
        ref = _single(awq, xs, layers)
        res = awq.quantize_block_host([x.pin_memory() for x in xs], [(xi, w.pin_memory()) for xi, w in layers],
                                      GRID, 4, 128, workspace=ws, state=state)
        assert len(res) == len(layers)
        for host, (L, a_star, packed, sc) in zip(res, ref):
            assert int(host["status"][0]) == 0
            assert torch.equal(host["L"], L)
            assert torch.equal(host["alpha_star"], a_star)
            assert torch.equal(host["packed"], packed)
            assert torch.equal(host["scales"], sc)


def test_quantize_block_host_layer_against_oracle(awq):
    xs, layers = _block(7)
    res = awq.quantize_block_host([x.pin_memory() for x in xs], [(xi, w.pin_memory()) for xi, w in layers],
                                  GRID, 4, 128)
    xi, w = layers[2]
    a = oracle.act_stats(xs[xi], oracle.STAT_MEAN).astype(np.float32)
    L_or, best_or = oracle.search(xs[xi], w, a, np.array(GRID, dtype=np.float32), 4, 128)
    L = res[2]["L"].numpy()
    assert np.allclose(L, L_or, rtol=1e-2, atol=0)
    check_alpha(L_or, best_or, int(np.argmin(L)))
    assert float(res[2]["alpha_star"][0]) == np.float32(GRID[int(np.argmin(L))])


def test_quantize_block_host_prefetch_chain(awq):
    """Blocks in a row, each call queueing the next block's upload
    (``prefetch``): every block's results equal the single-layer calls; a
    call whose inputs are not the prefetched ones uploads its own."""
    blocks = [_block(20 + 3 * i) for i in range(3)] + [_block(40)]
    pinned = [([x.pin_memory() for x in xs], [(xi, w.pin_memory()) for xi, w in layers]) for xs, layers in blocks]
    state, ws = awq.BlockHostState(), awq.Workspace()
    # 0 -> 1 -> 2 with prefetch, then 3, whose upload was not queued (2 queued block 0 again)
    plan = [(0, 1), (1, 2), (2, 0), (3, None)]
    for cur, nxt in plan:
        xs_h, layers_h = pinned[cur]
        res = awq.quantize_block_host(xs_h, layers_h, GRID, 4, 128, workspace=ws, state=state,
                                      prefetch=None if nxt is None else pinned[nxt])
        got = [{k: v.clone() for k, v in r.items()} for r in res]
        ref = _single(awq, *blocks[cur])
        for host, (L, a_star, packed, sc) in zip(got, ref):
            assert int(host["status"][0]) == 0
            assert torch.equal(host["L"], L)
            assert torch.equal(host["alpha_star"], a_star)
            assert torch.equal(host["packed"], packed)
            assert torch.equal(host["scales"], sc)
