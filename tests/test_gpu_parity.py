"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on
the same seeded inputs.

Acceptance, per the contract of the search:
  * act_stats: max bit-exact; mean within relative 1e-5 (fp32 sums vs fp64)
  * scales: bit-exact (both sides round an fp64 power once to fp32)
  * quantize_pack: codes, packed words and scales bit-exact for the same s
  * search: L(alpha) within relative 1e-2 of the oracle for every alpha
    (bf16 operands, fp32 accumulation); alpha* identical, or the oracle's loss
    at the GPU's alpha* within 1% of the oracle's minimum
Sizes span several tiles (128 output columns x 256 tokens x 64 k) and ragged
tails in every dimension.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from gpu_bounds import check_alpha, rounding_bound
from post_weight_only_b200 import synth

pytestmark = pytest.mark.gpu

L_RTOL = 1e-2


@pytest.fixture(scope="module")
def awq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from post_weight_only_b200 import awq as mod
    return mod


def _layer(N, D_in, D_out, seed=0, **kw):
    return synth.layer_inputs(synth.small_layer(N, D_in, D_out, seed=seed, **kw))


def _oracle_a(X):
    return oracle.act_stats(X).astype(np.float32)


FORMS = ("error", "reference")
_rounding_bound = rounding_bound


def _form_id(form, awq):
    return awq.LOSS_ERROR if form == "error" else awq.LOSS_REFERENCE


_check_alpha = check_alpha


# ------------------------------------------------------------------ statistic
@pytest.mark.parametrize("N,D", [
    (1, 8), (7, 264), (300, 520), (4096, 4096), (1000, 11008),
    (1, 4096),                                    # one row: the second CTA of each pair has none
    (3, 262144), (2, 524288), (1, 1048576),       # one row lane per chunk; one, two, four rounds
    (64, 65536), (40, 151552),                    # slabs wider than the CTA's threads, with several row lanes
])
def test_act_stats(awq, N, D):
    X, _ = _layer(N, D, 8, seed=N)
    Xd = X.cuda()
    a_mean = awq.act_stats(Xd, awq.STAT_MEAN).cpu().numpy()
    a_max = awq.act_stats(Xd, awq.STAT_MAX).cpu().numpy()
    torch.cuda.synchronize()
    ref_mean = oracle.act_stats(X, oracle.STAT_MEAN)
    ref_max = oracle.act_stats(X, oracle.STAT_MAX)
    assert np.array_equal(a_max.astype(np.float64), ref_max)
    assert np.allclose(a_mean, ref_mean, rtol=1e-5, atol=0)


def test_act_stats_hand_worked(awq):
    """The worked 4 x 8 example (golden file): every mean is an exact binary
    fraction, so the fp32 statistic equals it exactly."""
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "act_stats_hand.json")))
    X = torch.tensor(g["X_rows"], dtype=torch.float32).to(torch.bfloat16).cuda()
    assert awq.act_stats(X, awq.STAT_MEAN).cpu().tolist() == g["mean_abs"]
    assert awq.act_stats(X, awq.STAT_MAX).cpu().tolist() == g["max_abs"]


def test_weight_mean_hand_worked(awq):
    """The worked 4 x 5 example of the balanced scale's weight statistic."""
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "weight_mean_hand.json")))
    W = torch.tensor(g["W_rows"], dtype=torch.float32).cuda()
    got = awq.weight_mean(W).cpu().numpy()
    assert got.tolist() == [float(np.float32(v)) for v in g["mean_abs_rows_fp32"]]


def test_act_stats_batched(awq):
    """Several inputs of different shapes in one launch: each statistic as the
    oracle's (max exact, mean within relative 1e-5)."""
    shapes = [(4096, 8192), (300, 264), (1, 4096), (2048, 28672), (17, 8)]
    Xs = [_layer(N, D, 8, seed=N + D)[0] for N, D in shapes]
    for stat in (awq.STAT_MEAN, awq.STAT_MAX):
        got = awq.act_stats_batched([X.cuda() for X in Xs], stat)
        for X, a in zip(Xs, got):
            ref = oracle.act_stats(X, oracle.STAT_MEAN if stat == awq.STAT_MEAN else oracle.STAT_MAX)
            a = a.cpu().numpy().astype(np.float64)
            if stat == awq.STAT_MAX:
                assert np.array_equal(a, ref)
            else:
                assert np.allclose(a, ref, rtol=1e-5, atol=0)


def test_act_stats_reproducible(awq):
    X, _ = _layer(3000, 1024, 8, seed=3)
    Xd = X.cuda()
    a1 = awq.act_stats(Xd)
    a2 = awq.act_stats(Xd)
    assert torch.equal(a1, a2)


# ------------------------------------------------------------------ scales
@pytest.mark.parametrize("alpha", [0.0, 0.05, 0.35, 0.5, 1.0])
def test_scales_bit_exact(awq, alpha):
    X, _ = _layer(64, 1024, 8, seed=1)
    a = _oracle_a(X)
    a[5] = 0.0                                           # a dead channel exercises the floor
    s_gpu = awq.scales(torch.from_numpy(a).cuda(), alpha).cpu().numpy()
    assert np.array_equal(s_gpu, oracle.scales(a, alpha))


def test_scales_from_device_alpha(awq):
    a = np.abs(np.random.default_rng(0).standard_normal(256)).astype(np.float32) + 0.1
    al = torch.tensor([0.45], dtype=torch.float32, device="cuda")
    s_gpu = awq.scales(torch.from_numpy(a).cuda(), al).cpu().numpy()
    assert np.array_equal(s_gpu, oracle.scales(a, np.float32(0.45)))


# ------------------------------------------------------------------ quantise + pack
@pytest.mark.parametrize("bits,group", [(4, 128), (4, 64), (3, 128), (2, 32), (3, 32), (4, 256)])
@pytest.mark.parametrize("D_in,D_out", [(256, 200), (1024, 4096)])
def test_quantize_pack_bit_exact(awq, bits, group, D_in, D_out):
    X, W = _layer(32, D_in, D_out, seed=D_out + bits)
    a = _oracle_a(X)
    s = oracle.scales(a, 0.55)
    packed, sc = awq.quantize_pack(W.cuda(), torch.from_numpy(s).cuda(), bits, group)
    q_or, d_or = oracle.quantize(W, s, bits, group)
    p_or = oracle.pack(q_or, bits)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_or)
    assert np.array_equal(sc.cpu().numpy(), d_or)


@pytest.mark.parametrize("bits,group,D_in,D_out", [
    (4, 128, 256, 203),    # D_out % 4 != 0: the untiled kernel
    (4, 128, 128, 1),      # one column (untiled)
    (4, 32, 96, 200),      # the last 128-row tile reaches past D_in
    (3, 64, 192, 132),     # same, two groups per tile
    (4, 64, 320, 4100),    # ragged last column tile
    (4, 256, 768, 132),    # group 256: the untiled kernel, 64 rows per thread
    (3, 256, 256, 7),
])
def test_quantize_pack_ragged(awq, bits, group, D_in, D_out):
    X, W = _layer(16, D_in, D_out, seed=D_in + D_out)
    s = oracle.scales(_oracle_a(X), 0.4)
    packed, sc = awq.quantize_pack(W.cuda(), torch.from_numpy(s).cuda(), bits, group)
    q_or, d_or = oracle.quantize(W, s, bits, group)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack(q_or, bits))
    assert np.array_equal(sc.cpu().numpy(), d_or)


def test_quantize_pack_hand_group(awq):
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_group_b4_g128.json")))
    W = np.zeros((128, 4), dtype=np.float32)
    W[:7, 0] = np.array(g["w_rows_0_to_6"], dtype=np.float32)
    W[:7, 2] = -W[:7, 0]
    packed, sc = awq.quantize_pack(torch.from_numpy(W).cuda(), torch.ones(128, device="cuda"), 4, 128)
    p = packed.cpu().numpy().view(np.uint32)
    assert int(p[0, 0]) == int(g["packed_word_0"], 16)
    assert all(int(v) == 0x88888888 for v in p[1:, 0])
    assert float(sc[0, 0]) == g["delta"]
    assert (p[:, 1] == 0x88888888).all() and float(sc[0, 1]) == 0.0   # all-zero group
    q_or, _ = oracle.quantize(W, None, 4, 128)
    assert np.array_equal(p, oracle.pack(q_or, 4))


def test_quantize_pack_near_ties(awq):
    """Weights placed exactly on and next to half-integer multiples of delta,
    where the reciprocal shortcut must defer to the exact IEEE quotient."""
    rng = np.random.default_rng(7)
    D_in, D_out = 128, 256
    W = np.zeros((D_in, D_out), dtype=np.float32)
    W[0, :] = 7.0                                      # delta = 1 at 4 bits
    base = rng.integers(-6, 6, size=(D_in - 1, D_out)).astype(np.float32) + np.float32(0.5)
    nudge = rng.integers(-2, 3, size=base.shape).astype(np.float32)
    W[1:, :] = np.nextafter(base, base + nudge * np.float32(1e9))    # on, above or below the tie
    s = (np.float32(1.0) + rng.random(D_in).astype(np.float32) * np.float32(2.0 ** -20)).astype(np.float32)
    s[0] = 1.0
    packed, sc = awq.quantize_pack(torch.from_numpy(W).cuda(), torch.from_numpy(s).cuda(), 4, 128)
    q_or, d_or = oracle.quantize(W, s, 4, 128)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack(q_or, 4))
    assert np.array_equal(sc.cpu().numpy(), d_or)


# ------------------------------------------------------------------ reference output (the X.W term)
@pytest.mark.parametrize("N,D_in,D_out", [(1, 64, 128), (300, 512, 200), (256, 96, 132), (1000, 1024, 1024)])
def test_layer_output(awq, N, D_in, D_out):
    X, W = _layer(N, D_in, D_out, seed=5)
    Y = awq.layer_output(X.cuda(), W.cuda()).cpu().double()
    ref = X.double() @ W.to(torch.bfloat16).double()
    scale = ref.abs().max().item() + 1e-30
    err = (Y - ref).abs().max().item() / scale
    assert err < 1e-5, err


# ------------------------------------------------------------------ search
def _search_both(awq, X, W, bits, group, alphas, cols=None, form="error"):
    a = _oracle_a(X)
    res = awq.search(X.cuda(), W.cuda(), torch.from_numpy(a).cuda(), alphas.tolist(), bits, group, want_cols=True,
                     loss_form=_form_id(form, awq))
    L_gpu = res.L.cpu().numpy()
    idx = int(res.alpha_idx.item())
    Lc_gpu = res.L_col.cpu().numpy()
    if cols is None:
        L_or, best_or = oracle.search(X, W, a, alphas, bits, group)
        return L_gpu, idx, Lc_gpu, L_or, best_or, float(res.alpha_star.item())
    L_or, best_or, Lc_or = oracle.search(X, W, a, alphas, bits, group, cols=cols, want_cols=True)
    return L_gpu, idx, Lc_gpu, (L_or, Lc_or), best_or, float(res.alpha_star.item())


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("N,D_in,D_out,bits,group,n_int", [
    (300, 512, 200, 4, 128, 20),     # ragged tokens and columns, split alpha tail
    (256, 512, 512, 4, 128, 20),     # the 512 x 512 / 256-token layer
    (64, 256, 128, 3, 128, 20),
    (130, 256, 64, 4, 64, 10),
    (97, 96, 132, 2, 32, 8),         # D_in not a multiple of 64; two groups per stage
    (1, 512, 1024, 4, 128, 20),      # a single token
    (700, 384, 4, 4, 128, 20),       # four output columns (one ragged tile)
    (300, 768, 200, 4, 256, 20),     # group 256 (16 threads per column in the pre-pass)
])
def test_search_small(awq, form, N, D_in, D_out, bits, group, n_int):
    """Every alpha within the arithmetic's own bound; within relative 1e-2 of
    the oracle wherever that bound allows it (always, for the error form)."""
    X, W = _layer(N, D_in, D_out, seed=N + D_in)
    alphas = synth.alpha_grid(n_int).numpy()
    L_gpu, idx, Lc_gpu, L_or, best_or, astar = _search_both(awq, X, W, bits, group, alphas, form=form)
    a = _oracle_a(X)
    for i, al in enumerate(alphas):
        bound = _rounding_bound(X, W, a, al, bits, group, form).sum()
        err = abs(L_gpu[i] - L_or[i])
        assert err <= bound, (al, L_gpu[i], L_or[i], bound)
        assert err <= max(L_RTOL, bound / L_or[i]) * L_or[i], (al, err / L_or[i])
        if form == "error":
            assert err <= L_RTOL * L_or[i], (al, err / L_or[i])
    assert np.allclose(Lc_gpu.sum(axis=1), L_gpu, rtol=1e-9)
    _check_alpha(L_or, best_or, idx)
    assert astar == alphas[idx]


@pytest.mark.parametrize("form", FORMS)
def test_search_degenerate_one_token_four_columns(awq, form):
    """One token and four output columns: L is a sum of four squares, so the
    operand noise does not average out; each column is held to the
    arithmetic's own bound."""
    X, W = _layer(1, 128, 4, seed=129)
    alphas = synth.alpha_grid(20).numpy()
    L_gpu, idx, Lc_gpu, L_or, best_or, _ = _search_both(awq, X, W, 4, 128, alphas, form=form)
    a = _oracle_a(X)
    for i, al in enumerate(alphas):
        bound = _rounding_bound(X, W, a, al, 4, 128, form)
        assert np.all(np.abs(Lc_gpu[i] - oracle.loss_cols(X, W, oracle.scales(a, al), 4, 128)) <= bound)


@pytest.mark.parametrize("form", FORMS)
def test_search_many_units_sampled_columns(awq, form):
    """More units than SMs (a full wave plus a split tail): every sampled
    column's per-alpha loss against the oracle within the arithmetic's bound
    (a single column's loss can be dominated by one or two outlier channels,
    so it is compared column by column with its own bound)."""
    N, D_in, D_out = 2560, 256, 2048
    X, W = _layer(N, D_in, D_out, seed=11)
    alphas = synth.alpha_grid(10).numpy()
    cols = np.array([0, 1, 127, 128, 1000, 2047], dtype=np.int64)
    L_gpu, idx, Lc_gpu, (L_or, Lc_or), best_or, _ = _search_both(awq, X, W, 4, 128, alphas, cols=cols, form=form)
    a = _oracle_a(X)
    for i, al in enumerate(alphas):
        bound = _rounding_bound(X, W, a, al, 4, 128, form, cols=cols)
        assert np.all(np.abs(Lc_gpu[i, cols] - Lc_or[i]) <= bound), (al, Lc_gpu[i, cols], Lc_or[i], bound)


@pytest.mark.parametrize("form", FORMS)
def test_search_reproducible(awq, form):
    X, W = _layer(700, 512, 384, seed=2)
    a = torch.from_numpy(_oracle_a(X)).cuda()
    Xd, Wd = X.cuda(), W.cuda()
    grid = synth.alpha_grid(20).tolist()
    r1 = awq.search(Xd, Wd, a, grid, 4, 128, loss_form=_form_id(form, awq))
    r2 = awq.search(Xd, Wd, a, grid, 4, 128, loss_form=_form_id(form, awq))
    assert torch.equal(r1.L, r2.L) and int(r1.alpha_idx) == int(r2.alpha_idx)


def test_search_then_pack_pipeline(awq):
    """alpha* -> s* on the device -> bit-exact codes for that s*."""
    X, W = _layer(256, 512, 256, seed=4)
    Xd, Wd = X.cuda(), W.cuda()
    a = awq.act_stats(Xd)
    grid = synth.alpha_grid(20).tolist()
    res = awq.search(Xd, Wd, a, grid, 4, 128)
    s_star = awq.scales(a, res.alpha_star)
    packed, sc = awq.quantize_pack(Wd, s_star, 4, 128)
    s_np = s_star.cpu().numpy()
    assert np.array_equal(s_np, oracle.scales(a.cpu().numpy(), float(res.alpha_star.item())))
    q_or, d_or = oracle.quantize(W, s_np, 4, 128)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack(q_or, 4))
    assert np.array_equal(sc.cpu().numpy(), d_or)


@pytest.mark.parametrize("form", FORMS)
def test_batched_matches_single(awq, form):
    layers = []
    for i, (N, D_in, D_out) in enumerate([(300, 256, 128), (300, 256, 64), (512, 512, 256)]):
        X, W = _layer(N, D_in, D_out, seed=20 + i)
        layers.append((X.cuda(), W.cuda(), awq.act_stats(X.cuda())))
    grid = synth.alpha_grid(20).tolist()
    batched = awq.search_batched(layers, grid, 4, 128, loss_form=_form_id(form, awq))
    for (X, W, a), rb in zip(layers, batched):
        rs = awq.search(X, W, a, grid, 4, 128, loss_form=_form_id(form, awq))
        assert torch.equal(rb.L, rs.L)
        assert int(rb.alpha_idx) == int(rs.alpha_idx)


def _batched_layers(awq, shapes, seed):
    layers = []
    for i, (N, D_in, D_out) in enumerate(shapes):
        X, W = _layer(N, D_in, D_out, seed=seed + i)
        layers.append((X.cuda(), W.cuda(), awq.act_stats(X.cuda())))
    return layers


def test_batched_overlap_varied_inputs(awq):
    """Layers whose D_in and D_out shrink and grow (so every workspace region
    changes its layout from one layer to the next, ragged token and column
    tails included) give bit for bit the single-layer L, per-column L and
    alpha* when searched in one batched call."""
    shapes = [(300, 512, 128), (300, 256, 64), (257, 1024, 256), (300, 256, 132), (64, 512, 68)]
    layers = _batched_layers(awq, shapes, 40)
    grid = synth.alpha_grid(20).tolist()
    batched = awq.search_batched(layers, grid, 4, 128, want_cols=True)
    for (X, W, a), rb in zip(layers, batched):
        rs = awq.search(X, W, a, grid, 4, 128, want_cols=True)
        assert torch.equal(rb.L, rs.L)
        assert torch.equal(rb.L_col, rs.L_col)
        assert int(rb.alpha_idx) == int(rs.alpha_idx)


def test_concurrent_searches_on_two_streams(awq):
    """Two searches in flight at once on two streams, each with its own
    workspace.  Each grid has a full wave of units (16 token tiles x 5 weight
    tiles on 74 CTA pairs), so its producers meet at every pass boundary; a
    grid whose CTAs wait for SMs that the other grid holds must stop waiting
    rather than stall.  The results equal those of the same searches run one
    after the other."""
    grid = synth.alpha_grid(20).tolist()
    layers = []
    for i in range(2):
        X, W = _layer(4096, 512, 1280, seed=80 + i)
        X, W = X.cuda(), W.cuda()
        layers.append((X, W, awq.act_stats(X)))
    ref = [awq.search(X, W, a, grid, 4, 128, want_cols=True) for X, W, a in layers]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    out = []
    for (X, W, a), st in zip(layers, streams):
        st.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(st):
            out.append(awq.search(X, W, a, grid, 4, 128, want_cols=True, workspace=awq.Workspace(),
                                  check_status=False))
    torch.cuda.synchronize()
    for r, rr in zip(out, ref):
        awq.check_device_status(r.status)
        assert torch.equal(r.L, rr.L)
        assert torch.equal(r.L_col, rr.L_col)
        assert int(r.alpha_idx) == int(rr.alpha_idx)


# ------------------------------------------------------------------ quantiser arithmetic
@pytest.mark.parametrize("divisor", [1, 3, 7, 15, 31, 127, 255])
def test_constant_divisor_matches_ieee_on_every_float(awq, divisor):
    """delta = fl(m / d) by Markstein's FMA correction equals __fdiv_rn for
    every non-negative finite float, and the fast reciprocal of the quotient
    shortcut stays within one ulp of the correctly rounded one."""
    bad_div, bad_rcp = awq.selftest_divide(divisor)
    assert bad_div == 0
    assert bad_rcp == 0


# ------------------------------------------------------------------ failure detection
def test_bounded_wait_gives_up_with_status(awq):
    """A wait on a barrier nothing arrives at returns AWQ_ETIMEOUT in the device
    status word; the context stays usable afterwards."""
    st = awq.selftest_wait_timeout(2_000_000)
    assert st & 0xFF == awq.AWQ_ETIMEOUT
    assert st >> 8 > 0
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0
