"""Parity at the full sizes of the five workloads: their shapes, value
distributions, quantiser settings and alpha grids, through the calls a user
makes and the benchmark times -- awq.quantize_layer (statistic -> search ->
s* = a^alpha* -> quantise + pack) for single layers, awq.search_batched for
the seven linears of the 70B-shaped block in one call.

At these sizes the oracle cannot evaluate every output column, so
  * the statistic, s* and the packed codes and group scales at s* are
    compared in full (max bit-exact, mean within relative 1e-5; s*, codes,
    scales bit-exact);
  * L(alpha) is compared column by column on a sample of output columns (the
    first and last, tile edges, seeded random ones) against the oracle, each
    within the arithmetic's own bound, and their sum within relative 1e-2;
  * alpha*: the full L equals the sum of the per-column losses, alpha* is its
    argmin, and on the sampled columns the GPU's and the oracle's argmins
    agree (identical, or the oracle's loss at the GPU's choice within 1% of
    the oracle's minimum).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from gpu_bounds import activations64, check_alpha, rounding_bound
from post_weight_only_b200 import synth

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

L_RTOL = 1e-2


@pytest.fixture(scope="module")
def awq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from post_weight_only_b200 import awq as mod
    return mod


def _sample_cols(D_out, n_random, seed):
    fixed = [0, 1, 127, 128, 255, 256, D_out // 2, D_out - 1]
    rng = np.random.default_rng(seed)
    cols = set(c for c in fixed if c < D_out)
    cols.update(int(c) for c in rng.choice(D_out, size=min(n_random, D_out), replace=False))
    return np.array(sorted(cols), dtype=np.int64)


def _check_columns(X, W, a_or, alphas, bits, group, L_gpu, Lc_gpu, idx_gpu, cols, form):
    L_or, best_or, Lc_or = oracle.search(X, W, a_or, alphas, bits, group, cols=cols, want_cols=True)
    # the full loss is the sum of the per-column losses; alpha* is its argmin
    assert np.allclose(Lc_gpu.sum(axis=1), L_gpu, rtol=1e-9)
    assert idx_gpu == int(np.argmin(L_gpu))
    samp_gpu = Lc_gpu[:, cols]
    x64 = activations64(X)
    for i, al in enumerate(alphas):
        bound = rounding_bound(X, W, a_or, al, bits, group, form, cols=cols, x64=x64)
        err = np.abs(samp_gpu[i] - Lc_or[i])
        assert np.all(err <= bound), (al, samp_gpu[i], Lc_or[i], bound)
        # relative 1e-2 on the sampled loss; the reference form (two rounded
        # products subtracted) is held to its own bound where that is wider
        rtol = L_RTOL if form == "error" else max(L_RTOL, bound.sum() / L_or[i])
        assert abs(samp_gpu[i].sum() - L_or[i]) <= rtol * L_or[i], (al, samp_gpu[i].sum(), L_or[i])
    check_alpha(L_or, best_or, int(np.argmin(samp_gpu.sum(axis=1))))


def _check_layer_path(awq, X, W, alphas, bits, group, form, cols):
    Xd, Wd = X.cuda(), W.cuda()
    fid = awq.LOSS_ERROR if form == "error" else awq.LOSS_REFERENCE
    r = awq.quantize_layer(Xd, Wd, alphas.tolist(), bits, group, want_cols=True, loss_form=fid)
    torch.cuda.synchronize()
    awq.check_device_status(r.search.status)
    a_or = oracle.act_stats(X).astype(np.float32)
    a_gpu = r.a.cpu().numpy()
    assert np.allclose(a_gpu, a_or, rtol=1e-5, atol=0)
    a_gpu = a_gpu.astype(np.float32)
    # everything downstream is checked on the GPU's own statistic
    idx = int(r.search.alpha_idx.item())
    assert float(r.search.alpha_star.item()) == np.float32(alphas[idx])
    _check_columns(X, W, a_gpu, alphas, bits, group, r.search.L.cpu().numpy(), r.search.L_col.cpu().numpy(), idx,
                   cols, form)
    s_or = oracle.scales(a_gpu, float(alphas[idx]))
    assert np.array_equal(r.s_star.cpu().numpy(), s_or)
    q_or, d_or = oracle.quantize(W, s_or, bits, group)
    assert np.array_equal(r.packed.cpu().numpy().view(np.uint32), oracle.pack(q_or, bits))
    assert np.array_equal(r.scales.cpu().numpy(), d_or)


GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("name", ["llama7b_attn_proj", "llama7b_mlp_down"])
def test_full_layer_against_full_oracle(awq, name):
    """Every L(alpha) of the whole layer (all output columns) and alpha*
    against the oracle's full search, stored once by
    tests/golden/make_full_goldens.py (oracle only): relative 1e-2 per alpha,
    alpha* identical or within 1% of the oracle's minimum."""
    from golden.make_full_goldens import input_digest
    g = json.load(open(os.path.join(GOLDEN, f"full_{name}.json")))
    wl = synth.workload(name)
    X, W = synth.layer_inputs(wl.layers[0])
    assert input_digest(X, W) == g["input_sha1"], "the seeded inputs differ from those of the stored oracle run"
    alphas = synth.alpha_grid(wl.n_intervals).numpy()
    assert [float(v) for v in alphas] == g["alphas"]
    bits, group = wl.quant[0]
    r = awq.quantize_layer(X.cuda(), W.cuda(), alphas.tolist(), bits, group)
    torch.cuda.synchronize()
    awq.check_device_status(r.search.status)
    L_or = np.array(g["L"])
    L_gpu = r.search.L.cpu().numpy()
    assert np.all(np.abs(L_gpu - L_or) <= L_RTOL * L_or), np.max(np.abs(L_gpu / L_or - 1))
    idx = int(r.search.alpha_idx.item())
    check_alpha(L_or, g["alpha_idx"], idx)
    assert abs(float(r.a.double().sum().item()) - g["a_sum"]) <= 1e-5 * g["a_sum"]


def test_linear_512_n256_all_columns(awq):
    """The small single-layer workload, every column, both loss forms."""
    wl = synth.workload("linear_512_n256")
    X, W = synth.layer_inputs(wl.layers[0])
    alphas = synth.alpha_grid(wl.n_intervals).numpy()
    for form in ("error", "reference"):
        _check_layer_path(awq, X, W, alphas, 4, 128, form, np.arange(W.shape[1]))


@pytest.mark.parametrize("name", ["llama7b_attn_proj", "llama7b_mlp_down"])
def test_llama7b_layers(awq, name):
    wl = synth.workload(name)
    X, W = synth.layer_inputs(wl.layers[0])
    alphas = synth.alpha_grid(wl.n_intervals).numpy()
    bits, group = wl.quant[0]
    _check_layer_path(awq, X, W, alphas, bits, group, "error", _sample_cols(W.shape[1], 8, seed=1))


def test_llama7b_attn_proj_reference_form(awq):
    wl = synth.workload("llama7b_attn_proj")
    X, W = synth.layer_inputs(wl.layers[0])
    alphas = synth.alpha_grid(wl.n_intervals).numpy()
    _check_layer_path(awq, X, W, alphas, 4, 128, "reference", _sample_cols(W.shape[1], 4, seed=2))


def test_llama70b_block_batched(awq):
    """All seven linears of the 70B-shaped block in one awq_search_batched
    call; sampled columns of every layer against the oracle."""
    wl = synth.workload("llama70b_block")
    alphas = synth.alpha_grid(wl.n_intervals).numpy()
    bits, group = wl.quant[0]
    host, dev, xs = [], [], {}
    for spec in wl.layers:
        key = (spec.x.kind, spec.x.seed, spec.D_in)
        if key not in xs:
            xs[key] = synth.make_x(spec.N, spec.D_in, spec.x)
        X = xs[key]
        W = synth.make_w(spec.D_in, spec.D_out, spec.w_std, spec.w_seed)
        host.append((X, W))
    xdev = {k: v.cuda() for k, v in xs.items()}
    for spec, (X, W) in zip(wl.layers, host):
        Xd = xdev[(spec.x.kind, spec.x.seed, spec.D_in)]
        dev.append((Xd, W.cuda(), awq.act_stats(Xd)))
    res = awq.search_batched(dev, alphas.tolist(), bits, group, want_cols=True)
    torch.cuda.synchronize()
    for li, ((X, W), (_, _, a_d), r) in enumerate(zip(host, dev, res)):
        a = a_d.cpu().numpy().astype(np.float32)
        cols = _sample_cols(W.shape[1], 2, seed=10 + li)
        _check_columns(X, W, a, alphas, bits, group, r.L.cpu().numpy(), r.L_col.cpu().numpy(),
                       int(r.alpha_idx.item()), cols, "error")


@pytest.mark.parametrize("bits,group", [(4, 128), (4, 64), (3, 128)])
def test_sweep_4096x11008_n16k(awq, bits, group):
    """Bit-width / group sweep, 41-point grid, both outlier densities."""
    wl = synth.workload("sweep_4096x11008_n16k")
    alphas = synth.alpha_grid(wl.n_intervals).numpy()
    W = synth.make_w(wl.layers[0].D_in, wl.layers[0].D_out, wl.layers[0].w_std, wl.layers[0].w_seed)
    for li, spec in enumerate(wl.layers):
        X = synth.make_x(spec.N, spec.D_in, spec.x)
        _check_layer_path(awq, X, W, alphas, bits, group, "error", _sample_cols(W.shape[1], 2, seed=20 + li))


def test_llama70b_qkv_joint(awq):
    """q/k/v of the 70B-shaped block share one input, hence one scale vector:
    the joint loss is the sum of the layers' losses, each of which matches a
    separate search of that layer."""
    wl = synth.workload("llama70b_block")
    alphas = synth.alpha_grid(wl.n_intervals).tolist()
    bits, group = wl.quant[0]
    specs = wl.layers[:3]
    X = synth.make_x(specs[0].N, specs[0].D_in, specs[0].x).cuda()
    Ws = [synth.make_w(s.D_in, s.D_out, s.w_std, s.w_seed).cuda() for s in specs]
    a = awq.act_stats(X)
    r = awq.search_joint(X, Ws, a, alphas, bits, group)
    L, per = r.L.cpu().numpy(), r.L_layers.cpu().numpy()
    assert np.allclose(per.sum(axis=0), L, rtol=1e-12)
    assert int(r.alpha_idx.item()) == int(np.argmin(L))
    for l, W in enumerate(Ws):
        single = awq.search(X, W, a, alphas, bits, group).L.cpu().numpy()
        assert np.allclose(per[l], single, rtol=1e-6)
