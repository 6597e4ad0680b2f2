"""The column-sharded search on the GPU (robocikowo.com AWQ page,
"parallelism": parallel within a layer; the loss is a sum over output columns,
concept page flow step 4c).

* A column slice of a wider W, searched in place through its row stride
  (awq_search_ex with ldw), gives bit for bit the losses of the same slice
  copied out contiguously.
* Two gloo ranks, each a process on cuda:0 searching its own slice through
  parallel.cuda_shard_loss, combined by one all-reduce: every rank holds the
  whole layer's L(alpha) (equal to the one-GPU search of the whole layer up to
  the order of the fp64 sums) and the same alpha*, which matches the oracle.
  The ranks' kernels never wait on each other; only the host all-reduce
  joins them.
"""
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from gpu_bounds import check_alpha
from post_weight_only_b200 import synth

pytestmark = pytest.mark.gpu

WORLD = 2


@pytest.fixture(scope="module")
def awq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from post_weight_only_b200 import awq as mod
    return mod


@pytest.mark.parametrize("form", [0, 1])
@pytest.mark.parametrize("c0,c1", [(256, 768), (0, 256), (768, 1000), (512, 516)])
def test_strided_slice_matches_contiguous_copy(awq, form, c0, c1):
    X, W = synth.layer_inputs(synth.small_layer(300, 512, 1000, seed=4))
    Xd, Wd = X.cuda(), W.cuda()
    a = awq.act_stats(Xd)
    grid = synth.alpha_grid(20).tolist()
    view = Wd[:, c0:c1]
    assert not view.is_contiguous() or c1 - c0 == 1000
    r_view = awq.search(Xd, view, a, grid, 4, 128, want_cols=True, loss_form=form)
    r_copy = awq.search(Xd, view.contiguous(), a, grid, 4, 128, want_cols=True, loss_form=form)
    assert torch.equal(r_view.L, r_copy.L)
    assert torch.equal(r_view.L_col, r_copy.L_col)
    assert int(r_view.alpha_idx.item()) == int(r_copy.alpha_idx.item())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer():
    return synth.layer_inputs(synth.small_layer(48, 256, 600, seed=3))


def _worker(rank, port, out_q):
    import torch.distributed as dist
    from post_weight_only_b200 import awq, parallel
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=WORLD)
    try:
        torch.cuda.set_device(0)
        X, W = _layer()
        Xd, Wd = X.cuda(), W.cuda()
        a = awq.act_stats(Xd)
        alphas = synth.alpha_grid(10).tolist()
        fn = parallel.cuda_shard_loss(Xd, Wd, a, alphas)
        L, best = parallel.column_sharded_search(fn, W.shape[1], align=256, device=torch.device("cpu"))
        torch.cuda.synchronize()
        out_q.put((rank, L.numpy(), best, a.cpu().numpy()))
    finally:
        dist.destroy_process_group()


def test_column_sharded_search_two_ranks_on_gpu(awq):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    outs = sorted([q.get(timeout=300) for _ in range(WORLD)], key=lambda o: o[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    X, W = _layer()
    alphas = synth.alpha_grid(10)
    a = outs[0][3]
    assert np.array_equal(outs[0][1], outs[1][1]) and outs[0][2] == outs[1][2]   # every rank holds the same result
    # the one-GPU search of the whole layer: the same sum in another order
    full = awq.search(X.cuda(), W.cuda(), torch.from_numpy(a).cuda(), alphas.tolist(), 4, 128)
    assert np.allclose(outs[0][1], full.L.cpu().numpy(), rtol=1e-12, atol=0)
    # the oracle on the same statistic
    L_or, best_or = oracle.search(X, W, a, alphas.numpy(), 4, 128)
    assert np.allclose(outs[0][1], L_or, rtol=1e-2, atol=0)
    check_alpha(L_or, best_or, outs[0][2])
