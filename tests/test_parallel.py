"""Multi-rank host logic of the sharded search, on the CPU with gloo
(world size 2).  The per-shard search is the oracle (test code), so these
tests check the orchestration: column slices that tile the layer, one
all-reduce giving every rank the whole layer's L(alpha) and the same alpha*,
and layer sharding collecting every layer's result on every rank."""
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from post_weight_only_b200 import parallel, synth

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer():
    return synth.layer_inputs(synth.small_layer(48, 256, 600, seed=3))


def _worker(rank, port, kind, out_q):
    import oracle
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=WORLD)
    try:
        alphas = synth.alpha_grid(10).numpy()
        if kind == "columns":
            X, W = _layer()
            a = oracle.act_stats(X).astype(np.float32)

            def shard_loss(c0, c1):
                if c1 <= c0:
                    return torch.zeros(len(alphas), dtype=torch.float64)
                L, _ = oracle.search(X, W[:, c0:c1].contiguous(), a, alphas, 4, 128)
                return torch.from_numpy(L)

            L, best = parallel.column_sharded_search(shard_loss, W.shape[1], align=256)
            out_q.put((rank, L.numpy(), best))
        else:
            layers = [synth.layer_inputs(synth.small_layer(24, 128, 32 + 8 * i, seed=i)) for i in range(3)]

            def layer_search(i):
                X, W = layers[i]
                a = oracle.act_stats(X).astype(np.float32)
                L, best = oracle.search(X, W, a, alphas, 4, 128)
                return torch.from_numpy(L), best

            res = parallel.layer_sharded_search(3, layer_search, len(alphas))
            out_q.put((rank, [r[0].numpy() for r in res], [r[1] for r in res]))
    finally:
        dist.destroy_process_group()


def _run(kind):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, kind, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    outs = [q.get(timeout=240) for _ in range(WORLD)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(outs, key=lambda o: o[0])


def test_shard_ranges_tile_the_columns():
    for D_out in (4, 256, 600, 4096, 11008):
        for world in (1, 2, 3, 8):
            spans = [parallel.column_shard(D_out, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == D_out
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            # each slice starts on a column tile, or is empty at the end
            assert all(s[0] % 256 == 0 or s[0] == s[1] == D_out for s in spans)


def test_argmin_lowest_index_on_ties():
    assert parallel.argmin_lowest(torch.tensor([3.0, 1.0, 1.0, 2.0])) == 1


def test_column_sharded_search_gloo():
    import oracle
    outs = _run("columns")
    X, W = _layer()
    a = oracle.act_stats(X).astype(np.float32)
    alphas = synth.alpha_grid(10).numpy()
    L_full, best_full = oracle.search(X, W, a, alphas, 4, 128)
    for rank, L, best in outs:
        assert np.allclose(L, L_full, rtol=1e-12)       # the shards tile the layer
        assert best == best_full
    assert np.array_equal(outs[0][1], outs[1][1])        # every rank holds the same L


def test_layer_sharded_search_gloo():
    import oracle
    outs = _run("layers")
    alphas = synth.alpha_grid(10).numpy()
    for i in range(3):
        X, W = synth.layer_inputs(synth.small_layer(24, 128, 32 + 8 * i, seed=i))
        a = oracle.act_stats(X).astype(np.float32)
        L, best = oracle.search(X, W, a, alphas, 4, 128)
        for rank, Ls, bests in outs:
            assert np.array_equal(Ls[i], L)
            assert bests[i] == best
