"""GPU parity of the quantiser and scale variants of the search
against the CPU oracle, through the C ABI.

  * the power-of-two delta (mudrobot.github.io AWQ notes, "analysing the
    quantisation error": delta = max|w| / 2^(b-1), codes clamped to b bits):
    the final pack bit-exact (codes, packed words, deltas) on both pack
    kernels, alone and with clip ratios and FP16 deltas; the search's losses
    within the arithmetic's bound and relative 1e-2, alpha* by the contract's
    rule;
  * the balanced scale (laojiahuo2003.github.io GPTQ/AWQ/SmoothQuant notes, section 4.4, the
    per-channel scale s_j = mean|X_j|^alpha / mean|W_j|^(1-alpha)): the weight
    statistic within relative 1e-6 (fp64 sums in another order), the scales
    within one fp32 ulp (fp64 powers from two math libraries), the search as
    above with the GPU's weight statistic given to both sides;
  * the asymmetric quantiser (compassingai.com AWQ concept page, "the AWQ
    mechanism": MinMax with a zero point): the zero-point pack bit-exact
    (codes, packed words in both layouts, deltas, zero points) on both pack
    kernels, including one-sided, all-zero and clamped groups; the search as
    above.
"""
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


def _layer(N, D_in, D_out, seed=0):
    return synth.layer_inputs(synth.small_layer(N, D_in, D_out, seed=seed))


def _ulps(x, y):
    xi = x.astype(np.float32).view(np.int32).astype(np.int64)
    yi = y.astype(np.float32).view(np.int32).astype(np.int64)
    return np.abs(xi - yi)


# ---------------------------------------------------------------- power-of-two delta
@pytest.mark.parametrize("bits,group,D_in,D_out,delta16,clip", [
    (4, 128, 512, 256, False, False),     # tiled pack kernel
    (3, 64, 384, 200, False, False),
    (2, 32, 96, 36, False, False),
    (4, 128, 256, 203, False, False),     # D_out % 4 != 0: the untiled kernel
    (4, 64, 256, 128, True, False),       # with FP16 deltas
    (4, 128, 256, 131, True, True),       # FP16 deltas and clip ratios, untiled
    (4, 128, 512, 128, False, True),      # clip ratios, tiled
    (4, 256, 512, 96, True, False),       # group 256 (untiled) with FP16 deltas
])
def test_pack_pow2_bit_exact(awq, bits, group, D_in, D_out, delta16, clip):
    X, W = _layer(16, D_in, D_out, seed=D_in + D_out)
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.4)
    c = None
    if clip:
        rng = np.random.default_rng(D_out)
        c = synth.clip_grid(20).numpy()[rng.integers(0, 21, size=(D_in // group, D_out))]
    packed, sc = awq.quantize_pack_ex(W.cuda(), torch.from_numpy(s).cuda(), bits, group,
                                      clip=None if c is None else torch.from_numpy(c).cuda(),
                                      delta_fp16=delta16, delta_pow2=True)
    q, d = oracle.quantize(W, s, bits, group, clip=c, delta16=delta16, qmode=oracle.QMODE_POW2)
    assert q.min() >= -(1 << (bits - 1)) and q.max() <= (1 << (bits - 1)) - 1
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack(q, bits))
    got = sc.cpu().numpy()
    assert np.array_equal(got.astype(np.float32) if delta16 else got, d)


def test_pack_pow2_codes_reach_both_ends(awq):
    """The largest magnitude of a group sits at code 2^(b-1) - 1 when
    positive and at -2^(b-1) when negative."""
    W = torch.zeros(128, 8)
    W[3, :4] = 1.0
    W[5, 4:] = -1.0
    W[7, :] = 0.3
    s = torch.ones(128)
    packed, sc = awq.quantize_pack_ex(W.cuda(), s.cuda(), 4, 128, delta_pow2=True)
    q, d = oracle.quantize(W, s.numpy(), 4, 128, qmode=oracle.QMODE_POW2)
    assert q[3, :4].tolist() == [7] * 4 and q[5, 4:].tolist() == [-8] * 4
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack(q, 4))


@pytest.mark.parametrize("form", ("error", "reference"))
@pytest.mark.parametrize("N,D_in,D_out,bits,group", [
    (300, 512, 200, 4, 128),
    (97, 96, 132, 2, 32),
    (64, 256, 128, 3, 64),
])
def test_search_pow2_against_oracle(awq, form, N, D_in, D_out, bits, group):
    X, W = _layer(N, D_in, D_out, seed=N + D_out)
    a = oracle.act_stats(X).astype(np.float32)
    alphas = synth.alpha_grid(20).numpy()
    lf = awq.LOSS_ERROR if form == "error" else awq.LOSS_REFERENCE
    res = awq.search(X.cuda(), W.cuda(), torch.from_numpy(a).cuda(), alphas.tolist(), bits, group, loss_form=lf,
                     quantizer=awq.QUANT_DELTA_POW2)
    L_gpu = res.L.cpu().numpy()
    L_or, best = oracle.search(X, W, a, alphas, bits, group, qmode=oracle.QMODE_POW2)
    for i, al in enumerate(alphas):
        bound = rounding_bound(X, W, a, al, bits, group, form, qmode=oracle.QMODE_POW2).sum()
        err = abs(L_gpu[i] - L_or[i])
        assert err <= bound, (al, L_gpu[i], L_or[i], bound)
        if form == "error":
            assert err <= L_RTOL * L_or[i], (al, err / L_or[i])
    check_alpha(L_or, best, int(res.alpha_idx.item()))


# ---------------------------------------------------------------- balanced scale
@pytest.mark.parametrize("D_in,D_out", [(512, 256), (4096, 4096), (96, 36), (1, 8)])
def test_weight_mean(awq, D_in, D_out):
    rng = np.random.default_rng(D_in)
    W = (rng.standard_normal((D_in, D_out)) * np.exp(rng.standard_normal((D_in, 1)))).astype(np.float32)
    b = awq.weight_mean(torch.from_numpy(W).cuda()).cpu().numpy()
    assert np.allclose(b, oracle.weight_mean(W), rtol=1e-6, atol=0)


@pytest.mark.parametrize("alpha", [0.0, 0.3, 0.5, 1.0])
def test_balanced_scales(awq, alpha):
    rng = np.random.default_rng(3)
    a = (rng.random(1000) + 0.01).astype(np.float32)
    b = (rng.random(1000) + 0.01).astype(np.float32)
    a[7] = 0.0
    b[9] = 0.0                                            # both floors
    s_gpu = awq.scales(torch.from_numpy(a).cuda(), alpha, w_mean=torch.from_numpy(b).cuda()).cpu().numpy()
    s_or = oracle.scales(a, alpha, w_mean=b)
    assert np.all(_ulps(s_gpu, s_or) <= 1), np.max(_ulps(s_gpu, s_or))
    assert np.mean(s_gpu == s_or) > 0.999
    # the device-alpha form gives the same values
    s_dev = awq.scales(torch.from_numpy(a).cuda(), torch.tensor([alpha], device="cuda"),
                       w_mean=torch.from_numpy(b).cuda()).cpu().numpy()
    assert np.array_equal(s_dev, s_gpu)


@pytest.mark.parametrize("form", ("error", "reference"))
@pytest.mark.parametrize("N,D_in,D_out,bits,group", [
    (300, 512, 200, 4, 128),
    (130, 256, 64, 4, 64),
])
def test_search_balanced_against_oracle(awq, form, N, D_in, D_out, bits, group):
    X, W = _layer(N, D_in, D_out, seed=N + 3 * D_out)
    a = oracle.act_stats(X).astype(np.float32)
    b_dev = awq.weight_mean(W.cuda())
    b = b_dev.cpu().numpy()
    alphas = synth.alpha_grid(20).numpy()
    lf = awq.LOSS_ERROR if form == "error" else awq.LOSS_REFERENCE
    res = awq.search(X.cuda(), W.cuda(), torch.from_numpy(a).cuda(), alphas.tolist(), bits, group, loss_form=lf,
                     w_mean=b_dev)
    L_gpu = res.L.cpu().numpy()
    L_or, best = oracle.search(X, W, a, alphas, bits, group, w_mean=b)
    for i, al in enumerate(alphas):
        bound = rounding_bound(X, W, a, al, bits, group, form, w_mean=b).sum()
        err = abs(L_gpu[i] - L_or[i])
        assert err <= bound, (al, L_gpu[i], L_or[i], bound)
        if form == "error":
            assert err <= L_RTOL * L_or[i], (al, err / L_or[i])
    check_alpha(L_or, best, int(res.alpha_idx.item()))
    # s* on the device from alpha* and the pack bit-exact for it
    s_star = awq.scales(torch.from_numpy(a).cuda(), res.alpha_star, w_mean=b_dev)
    packed, sc = awq.quantize_pack(W.cuda(), s_star, bits, group)
    q, d = oracle.quantize(W, s_star.cpu().numpy(), bits, group)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack(q, bits))


# ---------------------------------------------------------------- dense 3-bit packing
@pytest.mark.parametrize("group,D_in,D_out,pow2,clip", [
    (128, 512, 256, False, False),     # tiled kernel
    (64, 384, 200, False, False),
    (32, 96, 36, True, False),         # tiled, power-of-two delta (codes reach -4)
    (128, 256, 203, False, False),     # untiled (D_out % 4 != 0), one string per thread
    (256, 512, 131, True, False),      # untiled, group 256: two strings per thread
    (128, 512, 128, False, True),      # clip ratios, tiled
])
def test_pack_dense3_bit_exact(awq, group, D_in, D_out, pow2, clip):
    X, W = _layer(16, D_in, D_out, seed=7 * D_in + D_out)
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.45)
    c = None
    if clip:
        rng = np.random.default_rng(D_in)
        c = synth.clip_grid(20).numpy()[rng.integers(0, 21, size=(D_in // group, D_out))]
    packed, sc = awq.quantize_pack_ex(W.cuda(), torch.from_numpy(s).cuda(), 3, group,
                                      clip=None if c is None else torch.from_numpy(c).cuda(), delta_pow2=pow2,
                                      dense3=True)
    q, d = oracle.quantize(W, s, 3, group, clip=c, qmode=oracle.QMODE_POW2 if pow2 else oracle.QMODE_SYMMETRIC)
    assert packed.shape == (D_in // 32 * 3, D_out)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack3(q))
    assert np.array_equal(sc.cpu().numpy(), d)


def test_pack_dense3_zero_group(awq):
    W = torch.zeros(128, 8)
    W[:, 4:] = torch.linspace(-1, 1, 128)[:, None]
    s = torch.ones(128)
    packed, _ = awq.quantize_pack_ex(W.cuda(), s.cuda(), 3, 128, dense3=True)
    q, _ = oracle.quantize(W, s.numpy(), 3, 128)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack3(q))


def test_pack_dense3_unsupported_combination(awq):
    W = torch.zeros(64, 6, device="cuda")
    s = torch.ones(64, device="cuda")
    with pytest.raises(awq.AwqError):
        awq.quantize_pack_ex(W, s, 3, 32, dense3=True)     # D_out % 4 != 0 with a group below 128
    with pytest.raises(awq.AwqError):
        awq.quantize_pack_ex(torch.zeros(64, 8, device="cuda"), s, 4, 32, dense3=True)   # 4-bit codes


# ---------------------------------------------------------------- asymmetric (MinMax, zero point)
def _check_zp(awq, W, s, bits, group, delta16=False, dense3=False):
    packed, sc, z = awq.quantize_pack_zp(W.cuda(), torch.from_numpy(s).cuda(), bits, group, delta_fp16=delta16,
                                         dense3=dense3)
    q, d, z_or = oracle.quantize_asym(W, s, bits, group, delta16=delta16)
    u = q.astype(np.int16) + np.repeat(z_or, group, axis=0).astype(np.int16)
    assert u.min() >= 0 and u.max() <= (1 << bits) - 1
    want = oracle.pack3((u - 4).astype(np.int8)) if dense3 else oracle.pack_unsigned(u)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), want)
    assert np.array_equal(z.cpu().numpy(), z_or)
    got = sc.cpu().numpy()
    assert np.array_equal(got.astype(np.float32) if delta16 else got, d)
    return q, d, z_or


@pytest.mark.parametrize("bits,group,D_in,D_out,delta16,dense3", [
    (4, 128, 512, 256, False, False),     # tiled pack kernel
    (3, 64, 384, 200, False, False),
    (2, 32, 96, 36, False, False),
    (4, 128, 256, 203, False, False),     # D_out % 4 != 0: the untiled kernel
    (4, 64, 256, 128, True, False),       # FP16 deltas (z formed from the rounded delta)
    (4, 256, 512, 96, True, False),       # group 256 (untiled) with FP16 deltas
    (3, 128, 512, 128, False, True),      # dense 3-bit, tiled
    (3, 32, 128, 64, False, True),        # dense 3-bit, group 32 (one string per group)
    (3, 256, 512, 131, True, True),       # dense 3-bit, untiled, FP16 deltas
])
def test_pack_asym_bit_exact(awq, bits, group, D_in, D_out, delta16, dense3):
    X, W = _layer(16, D_in, D_out, seed=D_in + 7 * D_out)
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.6)
    _check_zp(awq, W, s, bits, group, delta16, dense3)


@pytest.mark.parametrize("dense3", [False, True])
def test_pack_asym_special_groups(awq, dense3):
    """One-sided groups (z = 0 and z = 2^b - 1), an all-zero group (delta = 0,
    z = 0, codes 0), shifted columns, and a group whose top code is clamped:
    lo = -3.5, hi = 11.5 give delta = 1, z = rne(3.5) = 4 and rne(11.5) = 12
    above 2^b - 1 - z = 11 (4 bits)."""
    bits = 3 if dense3 else 4
    rng = np.random.default_rng(5)
    W = rng.standard_normal((256, 64)).astype(np.float32)
    W[:128, 0:8] = np.abs(W[:128, 0:8])          # non-negative groups
    W[:128, 8:16] = -np.abs(W[:128, 8:16])       # non-positive groups
    W[:128, 16:20] = 0.0                         # all-zero groups
    W[:, 20:40] += 3.0                           # mostly positive, lo = 0 in many groups
    W[128:, 40:44] = 0.25
    W[128, 40:44] = -3.5
    W[129, 40:44] = 11.5
    s = np.ones(256, dtype=np.float32)
    q, d, z = _check_zp(awq, torch.from_numpy(W), s, bits, 128, dense3=dense3)
    umax = (1 << bits) - 1
    assert np.all(z[0, 0:8] == 0) and np.all(z[0, 8:16] == umax)
    assert np.all(d[0, 16:20] == 0) and np.all(z[0, 16:20] == 0) and np.all(q[:128, 16:20] == 0)
    if bits == 4:
        assert np.all(d[1, 40:44] == 1.0) and np.all(z[1, 40:44] == 4)
        assert np.all(q[129, 40:44] == 11) and np.all(q[128, 40:44] == -4)


@pytest.mark.parametrize("form", ("error", "reference"))
@pytest.mark.parametrize("N,D_in,D_out,bits,group", [
    (300, 512, 200, 4, 128),
    (97, 96, 132, 2, 32),
    (64, 256, 128, 3, 64),
    (40, 512, 96, 4, 256),
])
def test_search_asym_against_oracle(awq, form, N, D_in, D_out, bits, group):
    X, W = _layer(N, D_in, D_out, seed=N + 5 * D_out)
    a = oracle.act_stats(X).astype(np.float32)
    alphas = synth.alpha_grid(20).numpy()
    lf = awq.LOSS_ERROR if form == "error" else awq.LOSS_REFERENCE
    res = awq.search(X.cuda(), W.cuda(), torch.from_numpy(a).cuda(), alphas.tolist(), bits, group, loss_form=lf,
                     quantizer=awq.QUANT_ASYMMETRIC)
    L_gpu = res.L.cpu().numpy()
    L_or, best = oracle.search(X, W, a, alphas, bits, group, qmode=oracle.QMODE_ASYMMETRIC)
    for i, al in enumerate(alphas):
        bound = rounding_bound(X, W, a, al, bits, group, form, qmode=oracle.QMODE_ASYMMETRIC).sum()
        err = abs(L_gpu[i] - L_or[i])
        assert err <= bound, (al, L_gpu[i], L_or[i], bound)
        if form == "error":
            assert err <= L_RTOL * L_or[i], (al, err / L_or[i])
    check_alpha(L_or, best, int(res.alpha_idx.item()))


def test_search_asym_below_symmetric(awq):
    """On weights with a non-zero mean per column the asymmetric grid fits the
    groups' ranges better: its losses lie below the symmetric ones (a
    property of the two quantisers, checked on the oracle's own losses too)."""
    X, W = _layer(256, 512, 128, seed=9)
    W = W + 0.05
    a = torch.from_numpy(oracle.act_stats(X).astype(np.float32)).cuda()
    grid = synth.alpha_grid(10).tolist()
    L_sym = awq.search(X.cuda(), W.cuda(), a, grid, 4, 128).L.cpu().numpy()
    L_asym = awq.search(X.cuda(), W.cuda(), a, grid, 4, 128, quantizer=awq.QUANT_ASYMMETRIC).L.cpu().numpy()
    assert np.all(L_asym < L_sym)
    Lo_sym, _ = oracle.search(X, W, a.cpu().numpy(), np.asarray(grid, dtype=np.float32), 4, 128)
    Lo_asym, _ = oracle.search(X, W, a.cpu().numpy(), np.asarray(grid, dtype=np.float32), 4, 128,
                               qmode=oracle.QMODE_ASYMMETRIC)
    assert np.all(Lo_asym < Lo_sym)
