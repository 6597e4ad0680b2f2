"""Pins that tie the CPU oracle to what the AWQ pages and plain mathematics
fix, independently of the oracle's own code.

Each test names the passage or the mathematical fact it checks:
hand-worked examples from the pages' quantiser definition (golden files),
special cases that reduce to a textbook routine (alpha = 0 is plain RTN),
exact identities (S^-1 and S cancel without quantisation; power-of-two scale
invariance; sign symmetry), bounds (|q| <= qmax, |error| <= delta / 2), a
library check of the loss (numpy fp64 matmul) and brute force on tiny layers.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from post_weight_only_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def _small(N, D_in, D_out, seed=0, **kw):
    return synth.layer_inputs(synth.small_layer(N, D_in, D_out, seed=seed, **kw))


def _rtn_numpy(W: np.ndarray, bits: int, group: int):
    """Plain round-to-nearest absmax group quantiser written with numpy float32
    primitives (the RTN baseline of the mudrobot.github.io notes, "baselines")."""
    qmax = np.float32(2 ** (bits - 1) - 1)
    D_in, D_out = W.shape
    Wg = W.reshape(D_in // group, group, D_out).astype(np.float32)
    m = np.abs(Wg).max(axis=1)                                   # [G, D_out]
    d = (m / qmax).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (Wg / d[:, None, :]).astype(np.float32)
    q = np.clip(np.round(t), -qmax, qmax)                         # np.round: half to even
    q = np.where(d[:, None, :] == 0, 0, q).astype(np.int8)
    return q.reshape(D_in, D_out), d


# --------------------------------------------------------------------------
# Hand-worked examples (golden files)
# --------------------------------------------------------------------------

def test_hand_group_codes_pack_and_delta():
    g = json.load(open(os.path.join(GOLDEN, "hand_group_b4_g128.json")))
    W = np.zeros((128, 1), dtype=np.float32)
    W[:7, 0] = np.array(g["w_rows_0_to_6"], dtype=np.float32)
    q, d = oracle.quantize(W, None, g["bits"], g["group"])
    assert d[0, 0] == np.float32(g["delta"])
    assert q[:8, 0].tolist() == g["q_rows_0_to_7"]
    assert (q[8:, 0] == 0).all()
    packed = oracle.pack(q, g["bits"])
    assert packed.shape == (16, 1)
    assert int(packed[0, 0]) == int(g["packed_word_0"], 16)
    assert all(int(v) == int(g["packed_words_1_to_15"], 16) for v in packed[1:, 0])
    err = q[:6, 0].astype(np.float64) * float(d[0, 0]) - W[:6, 0].astype(np.float64)
    assert err.tolist() == g["errors_rows_0_to_5"]


def test_hand_group_loss_and_tie_break():
    g = json.load(open(os.path.join(GOLDEN, "hand_group_b4_g128.json")))
    W = np.zeros((128, 1), dtype=np.float32)
    W[:7, 0] = np.array(g["w_rows_0_to_6"], dtype=np.float32)
    X = _bf16(np.ones((1, 128), dtype=np.float32))
    a = oracle.act_stats(X)
    assert (a == 1.0).all()
    alphas = synth.alpha_grid(20).numpy()
    L, best = oracle.search(X, W, a.astype(np.float32), alphas, 4, 128)
    expect = (-0.0625 + 0.125 - float(np.float32(0.1))) ** 2
    assert np.allclose(L, expect, rtol=1e-14, atol=0)
    assert len(set(L.tolist())) == 1          # bit-identical for every alpha
    assert best == g["alpha_star_index"]


def test_scalar_example_page3():
    g = json.load(open(os.path.join(GOLDEN, "scalar_example_page3.json")))
    W = np.zeros((g["group"], 1), dtype=np.float32)
    W[:2, 0] = np.array(g["group_values"], dtype=np.float32)
    q, d = oracle.quantize(W, None, g["bits"], g["group"])
    assert d[0, 0] == np.float32(g["delta"])
    assert q[:2, 0].tolist() == g["q"]
    w_hat = float(q[1, 0]) * float(d[0, 0])
    assert w_hat == g["w_hat_of_1.23"]
    assert abs((w_hat - float(np.float32(1.23))) - g["error_of_1.23"]) < 1e-7


# --------------------------------------------------------------------------
# Special cases and identities
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits,group", [(4, 128), (3, 128), (4, 64), (2, 32)])
def test_alpha_zero_is_plain_rtn(bits, group):
    """alpha = 0 gives s = 1 exactly, i.e. no scaling: the codes degenerate to
    plain RTN (compassingai.com concept page, "scale search": alpha = 0 means
    no scaling, plain uniform quantisation)."""
    X, W = _small(64, 256, 40, seed=3)
    a = oracle.act_stats(X).astype(np.float32)
    s0 = oracle.scales(a, 0.0)
    assert (s0 == 1.0).all()
    q, d = oracle.quantize(W, s0, bits, group)
    q_rtn, d_rtn = _rtn_numpy(W.numpy(), bits, group)
    assert np.array_equal(q, q_rtn)
    assert np.array_equal(d, d_rtn)
    L, _, Lc = oracle.search(X, W, a, np.array([0.0], dtype=np.float32), bits, group, want_cols=True)
    L_plain = oracle.loss_cols(X, W, None, bits, group)
    assert np.array_equal(Lc[0], L_plain)          # column by column, bit for bit
    assert np.isclose(L[0], L_plain.sum(), rtol=1e-13)


def test_cancellation_without_quantisation():
    """With Q replaced by the identity, X S^-1 (S W) = X W: the transform is
    exactly equivalent (compassingai.com concept page, "core mechanism";
    laojiahuo2003.github.io notes, AWQ section: W'x' = Wx).  Only the fp32
    rounding of s*w is left, ~2^-24 relative."""
    X, W = _small(32, 256, 24, seed=5)
    a = oracle.act_stats(X).astype(np.float32)
    Y = X.double() @ W.double()
    ref = float((Y * Y).sum())
    for alpha in (0.0, 0.35, 1.0):
        s = oracle.scales(a, alpha)
        L = oracle.loss_cols(X, W, s, 4, 128, quantize_w=False).sum()
        assert L <= 1e-12 * ref


def test_power_of_two_scale_invariance_and_sign_symmetry():
    """The absmax definition makes the codes invariant to s -> 2^t s (delta
    scales by 2^t, exactly in fp32) and antisymmetric in W -> -W; the loss is
    unchanged in both cases."""
    X, W = _small(32, 256, 24, seed=7)
    a = oracle.act_stats(X).astype(np.float32)
    s = oracle.scales(a, 0.5)
    q, d = oracle.quantize(W, s, 4, 128)
    for t in (-3, 5):
        q2, d2 = oracle.quantize(W, (s * np.float32(2.0 ** t)).astype(np.float32), 4, 128)
        assert np.array_equal(q, q2)
        assert np.array_equal(d2, (d * np.float32(2.0 ** t)).astype(np.float32))
    qn, dn = oracle.quantize(-W, s, 4, 128)
    assert np.array_equal(qn, -q) and np.array_equal(dn, d)
    L1 = oracle.loss_cols(X, W, s, 4, 128).sum()
    L2 = oracle.loss_cols(X, W, (s * np.float32(8.0)).astype(np.float32), 4, 128).sum()
    L3 = oracle.loss_cols(X, -W, s, 4, 128).sum()
    assert np.isclose(L1, L2, rtol=1e-12) and np.isclose(L1, L3, rtol=1e-12)


@pytest.mark.parametrize("bits,group", [(4, 128), (3, 128), (4, 64), (2, 32), (3, 32)])
def test_quantiser_bounds(bits, group):
    """|q| <= 2^(b-1)-1 (the clamp of the concept page), |w' - q delta| <=
    delta/2 (the rounding error lies in [0, 0.5] steps: mudrobot.github.io notes,
    "analysing the quantisation error"), and every non-zero group reaches
    |q| = qmax at its largest element."""
    X, W = _small(16, 512, 64, seed=11)
    a = oracle.act_stats(X).astype(np.float32)
    s = oracle.scales(a, 0.6)
    q, d = oracle.quantize(W, s, bits, group)
    qmax = 2 ** (bits - 1) - 1
    assert np.abs(q.astype(np.int32)).max() <= qmax
    Wp = (s[:, None].astype(np.float32) * W.numpy()).astype(np.float32)
    dd = np.repeat(d, group, axis=0).astype(np.float64)
    err = np.abs(Wp.astype(np.float64) - q.astype(np.float64) * dd)
    assert (err <= dd / 2 * (1 + 1e-6)).all()
    qg = np.abs(q.astype(np.int32)).reshape(-1, group, q.shape[1]).max(axis=1)
    assert (qg[d > 0] == qmax).all()


def test_rounding_error_statistics():
    """The rounding error, in units of delta, is roughly uniform on [0, 0.5]
    with mean ~0.25 (mudrobot.github.io notes, "analysing the quantisation
    error", item 1).  Statistical, loose tolerance."""
    W = synth.make_w(4096, 64, 0.02, 123)
    q, d = oracle.quantize(W, None, 4, 128)
    dd = np.repeat(d, 128, axis=0).astype(np.float64)
    r = np.abs(W.numpy().astype(np.float64) - q * dd) / dd
    assert abs(r.mean() - 0.25) < 0.01
    hist, _ = np.histogram(r, bins=5, range=(0, 0.5))
    frac = hist / hist.sum()
    assert np.all(np.abs(frac - 0.2) < 0.02)


# --------------------------------------------------------------------------
# Statistic, scales, packing
# --------------------------------------------------------------------------

def test_act_stats_matches_numpy():
    X, _ = _small(100, 264, 8, seed=2)
    xf = X.float().numpy().astype(np.float64)
    assert np.allclose(oracle.act_stats(X, oracle.STAT_MEAN), np.abs(xf).mean(axis=0), rtol=1e-14)
    assert np.array_equal(oracle.act_stats(X, oracle.STAT_MAX), np.abs(xf).max(axis=0))


def test_act_stats_hand_worked():
    """Worked 4 x 8 example of the statistic (golden file): mean and max run
    down each input channel's column over the N calibration rows."""
    g = json.load(open(os.path.join(GOLDEN, "act_stats_hand.json")))
    X = _bf16(np.array(g["X_rows"], dtype=np.float32))
    assert X.shape == (g["N"], g["D_in"])
    assert X.float().numpy().tolist() == g["X_rows"]          # every entry exact in bf16
    assert oracle.act_stats(X, oracle.STAT_MEAN).tolist() == g["mean_abs"]
    assert oracle.act_stats(X, oracle.STAT_MAX).tolist() == g["max_abs"]


def test_scales_special_values():
    a = np.array([0.5, 2.0, 0.0, 3.0], dtype=np.float32)
    assert (oracle.scales(a, 0.0) == 1.0).all()
    s1 = oracle.scales(a, 1.0)
    assert s1[0] == 0.5 and s1[1] == 2.0 and s1[3] == 3.0
    assert s1[2] == np.float32(1e-6) * np.float32(3.0)          # floored dead channel
    sh = oracle.scales(a, 0.5)
    assert sh[1] == np.float32(np.sqrt(2.0))
    assert (oracle.scales(np.zeros(4, np.float32), 0.7) == 1.0).all()


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_roundtrip(bits):
    rng = np.random.default_rng(0)
    qmax = 2 ** (bits - 1) - 1
    q = rng.integers(-qmax, qmax + 1, size=(64, 12)).astype(np.int8)
    p = oracle.pack(q, bits)
    u = np.stack([(p >> (4 * i)) & 0xF for i in range(8)], axis=1)   # [D_in/8, 8, D_out]
    back = u.reshape(64, 12).astype(np.int32) - 2 ** (bits - 1)
    assert np.array_equal(back, q.astype(np.int32))


# --------------------------------------------------------------------------
# The loss: library check, literal form, brute-force argmin
# --------------------------------------------------------------------------

def test_loss_matches_numpy_matmul():
    X, W = _small(48, 256, 20, seed=9)
    a = oracle.act_stats(X).astype(np.float32)
    s = oracle.scales(a, 0.45)
    q, d = oracle.quantize(W, s, 4, 128)
    E = q.astype(np.float64) * np.repeat(d, 128, axis=0).astype(np.float64) / s[:, None].astype(np.float64) \
        - W.numpy().astype(np.float64)
    Y = X.float().numpy().astype(np.float64) @ E
    ref = (Y * Y).sum(axis=0)
    got = oracle.loss_cols(X, W, s, 4, 128)
    assert np.allclose(got, ref, rtol=1e-11)
    cols = [3, 17, 0]
    assert np.allclose(oracle.loss_cols(X, W, s, 4, 128, cols=cols), ref[cols], rtol=1e-11)


@pytest.mark.parametrize("D_in,D_out,N,seed", [(128, 4, 8, 0), (256, 8, 16, 1), (256, 3, 5, 2)])
def test_literal_form_and_brute_force_argmin(D_in, D_out, N, seed):
    """Materialise S^-1 and Q(S W) and evaluate ||X S^-1 Q(SW) - X W||^2
    literally (long double) for every alpha: it must equal the oracle's
    column-sum form, and the argmin over the grid must agree."""
    X, W = _small(N, D_in, D_out, seed=seed, n_outlier=2)
    a = oracle.act_stats(X).astype(np.float32)
    alphas = synth.alpha_grid(20).numpy()
    L, best = oracle.search(X, W, a, alphas, 4, 128)
    lit = np.array([oracle.literal_loss(X, W, oracle.scales(a, al), 4, 128) for al in alphas])
    assert np.allclose(L, lit, rtol=1e-9)
    assert best == int(np.argmin(lit))


def test_search_column_subset_sums():
    X, W = _small(40, 256, 16, seed=4)
    a = oracle.act_stats(X).astype(np.float32)
    alphas = synth.alpha_grid(4).numpy()
    L, best, Lc = oracle.search(X, W, a, alphas, 3, 64, want_cols=True)
    assert np.allclose(Lc.sum(axis=1), L, rtol=1e-13)
    cols = [1, 7, 15]
    Ls, _, Lcs = oracle.search(X, W, a, alphas, 3, 64, cols=cols, want_cols=True)
    assert np.allclose(Lcs, Lc[:, cols], rtol=1e-13)
    assert np.allclose(Ls, Lc[:, cols].sum(axis=1), rtol=1e-13)


def test_outlier_channels_pull_alpha_up():
    """Sanity (not a pin): on a layer with strong outlier channels the search
    picks alpha > 0, i.e. scaling beats plain RTN (the pages' central claim)."""
    X, W = _small(128, 512, 32, seed=1, n_outlier=5)
    a = oracle.act_stats(X).astype(np.float32)
    alphas = synth.alpha_grid(20).numpy()
    L, best = oracle.search(X, W, a, alphas, 4, 128)
    assert best > 0 and L[best] < L[0]


# ------------------------------------------------------------------ joint search of shared-input linears
def test_joint_search_one_layer_is_the_search():
    X, W = synth.layer_inputs(synth.small_layer(32, 256, 24, seed=41))
    a = oracle.act_stats(X).astype(np.float32)
    alphas = synth.alpha_grid(10).numpy()
    L, best, per = oracle.search_joint(X, [W], a, alphas, 4, 128)
    L1, b1 = oracle.search(X, W, a, alphas, 4, 128)
    assert np.array_equal(L, L1) and best == b1 and np.array_equal(per[0], L1)


def test_joint_search_equals_search_of_side_by_side_weights():
    """A layer's loss is a sum over its output columns, so the joint loss of
    q/k/v-like layers is the loss of their weights side by side."""
    X, W1 = synth.layer_inputs(synth.small_layer(32, 256, 24, seed=42))
    W2 = synth.make_w(256, 16, 0.02, 7)
    W3 = synth.make_w(256, 8, 0.03, 8)
    a = oracle.act_stats(X).astype(np.float32)
    alphas = synth.alpha_grid(10).numpy()
    L, best, per = oracle.search_joint(X, [W1, W2, W3], a, alphas, 4, 128)
    Lc, bc = oracle.search(X, torch.cat([W1, W2, W3], dim=1), a, alphas, 4, 128)
    assert np.allclose(L, Lc, rtol=1e-12) and best == bc
    assert np.allclose(per.sum(axis=0), L, rtol=0)


# ------------------------------------------------------------------ FP16 delta export
def test_delta16_is_the_ieee_half_rounding_of_delta():
    """delta16 = the IEEE binary16 round-to-nearest-even of the fp32 delta,
    checked against numpy's float16 conversion (an independent routine)."""
    X, W = synth.layer_inputs(synth.small_layer(8, 512, 96, seed=51))
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.5)
    _, d32 = oracle.quantize(W, s, 4, 128)
    _, d16 = oracle.quantize(W, s, 4, 128, delta16=True)
    assert np.array_equal(d16, d32.astype(np.float16).astype(np.float32))
    # tiny and huge magnitudes: subnormal halves and the overflow threshold
    Wt = np.zeros((32, 6), np.float32)
    Wt[0] = [7e-8, 3e-6, 1.0, 6.5e4 * 7, 1e6, -2.5e-7]
    _, dt = oracle.quantize(Wt, None, 4, 32, delta16=True)
    _, dt32 = oracle.quantize(Wt, None, 4, 32)
    with np.errstate(over="ignore"):               # 1e6 / 7 overflows FP16 to infinity on both sides
        assert np.array_equal(dt, dt32.astype(np.float16).astype(np.float32))


def test_delta16_codes_round_with_the_half_delta():
    """With delta16 the codes are those of the FP16 delta: every unclamped
    code is within half a step of w'/delta16, and groups whose fp32 delta is
    already an FP16 value (powers of two) keep the plain codes."""
    X, W = synth.layer_inputs(synth.small_layer(8, 256, 64, seed=52))
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.4)
    q, d = oracle.quantize(W, s, 4, 64, delta16=True)
    wp = s[:, None].astype(np.float64) * W.numpy().astype(np.float64)
    y = wp / np.repeat(d, 64, axis=0).astype(np.float64)
    inside = np.abs(q) < 7
    assert np.all(np.abs(y[inside] - q[inside]) <= 0.5 + 1e-6)
    assert np.abs(q).max() <= 7
    Wp = np.zeros((32, 3), np.float32)
    Wp[:, 0] = np.linspace(-7, 7, 32)            # max 7 -> delta 1
    Wp[:, 1] = np.linspace(-0.875, 0.5, 32)      # max 0.875 -> delta 0.125
    Wp[:, 2] = np.linspace(-14, 3, 32)           # max 14 -> delta 2
    assert np.array_equal(oracle.quantize(Wp, None, 4, 32, delta16=True)[0], oracle.quantize(Wp, None, 4, 32)[0])


# ------------------------------------------------------------------ the quantised layer (W4A16 consumer)
def test_w4a16_exact_on_representable_weights():
    """Weights that are integer multiples of a power-of-two delta, with s = 1,
    quantise exactly, so the layer output is X W (numpy matmul)."""
    rng = np.random.default_rng(61)
    D_in, D_out, N = 128, 24, 5
    codes = rng.integers(-7, 8, size=(D_in, D_out))
    codes[0] = 7                                      # every group reaches qmax: delta = 0.25 exactly
    W = (codes * 0.25).astype(np.float32)
    X = torch.randn(N, D_in, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    q, d = oracle.quantize(W, None, 4, 128)
    assert np.all(d == 0.25) and np.array_equal(q, codes)
    Y = oracle.w4a16(X, np.ones(D_in, np.float32), oracle.pack(q, 4), d, 4, 128)
    assert np.allclose(Y, X.double().numpy() @ W.astype(np.float64), rtol=1e-12, atol=1e-12)


def test_w4a16_is_the_dequantised_search_operand():
    """With scales s the output is X S^-1 Q(S W): the same weights the search's
    loss dequantises, checked with a numpy matmul on the oracle's codes."""
    X, W = synth.layer_inputs(synth.small_layer(6, 256, 40, seed=62))
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.5)
    for bits, group in ((4, 128), (3, 64), (2, 32)):
        q, d = oracle.quantize(W, s, bits, group)
        w_hat = q * np.repeat(d, group, axis=0).astype(np.float64) / s.astype(np.float64)[:, None]
        Y = oracle.w4a16(X, s, oracle.pack(q, bits), d, bits, group)
        assert np.allclose(Y, X.double().numpy() @ w_hat, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- quantiser with delta = max / 2^(b-1)
# (mudrobot.github.io notes, "analysing the quantisation error": Q(w) = delta *
# Round(w / delta), delta = max|w| / 2^(N-1); codes clamped to N bits.)

def test_pow2_quantiser_worked_example():
    # one group of 4 in one column: max |w| = 1 -> delta = 1/8;
    # 0.5 -> 4, -1 -> -8, 0.26 -> round(2.08) = 2, 0.74 -> round(5.92) = 6
    W = np.array([[0.5], [-1.0], [0.26], [0.74]], dtype=np.float32)
    q, d = oracle.quantize(W, None, 4, 4, qmode=oracle.QMODE_POW2)
    assert d[0, 0] == np.float32(0.125)
    assert q[:, 0].tolist() == [4, -8, 2, 6]


def test_pow2_quantiser_clamps_the_positive_maximum():
    # +max maps to 2^(b-1) = 8, one past the largest 4-bit code: clamped to 7
    W = np.array([[1.0], [-0.5], [0.25], [0.0]], dtype=np.float32)
    q, d = oracle.quantize(W, None, 4, 4, qmode=oracle.QMODE_POW2)
    assert d[0, 0] == np.float32(0.125) and q[:, 0].tolist() == [7, -4, 2, 0]
    q3, d3 = oracle.quantize(W, None, 3, 4, qmode=oracle.QMODE_POW2)
    assert d3[0, 0] == np.float32(0.25) and q3[:, 0].tolist() == [3, -2, 1, 0]


def test_pow2_quantiser_brute_force():
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((64, 6)) * np.exp(rng.standard_normal((64, 1)))).astype(np.float32)
    s = (rng.random(64) + 0.5).astype(np.float32)
    for bits in (2, 3, 4):
        q, d = oracle.quantize(W, s, bits, 32, qmode=oracle.QMODE_POW2)
        lo, hi = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
        for g in range(2):
            for n in range(6):
                wp = (s[32 * g:32 * g + 32] * W[32 * g:32 * g + 32, n]).astype(np.float32)
                m = np.max(np.abs(wp))
                assert d[g, n] * (1 << (bits - 1)) == m          # exact power-of-two scaling
                for k in range(32):
                    t = float(np.float32(wp[k] / d[g, n]))
                    cand = np.arange(lo, hi + 1)
                    err = np.abs(cand - t)
                    best = cand[err == err.min()]
                    want = best[0] if len(best) == 1 else best[best % 2 == 0][0]   # ties to even
                    assert q[32 * g + k, n] == want


def test_pow2_quantiser_search_differs_from_symmetric():
    X, W = synth.layer_inputs(synth.small_layer(64, 128, 16, seed=3))
    a = oracle.act_stats(X).astype(np.float32)
    grid = np.array([0.0, 0.5], np.float32)
    L0, _ = oracle.search(X, W, a, grid, 4, 64)
    L1, _ = oracle.search(X, W, a, grid, 4, 64, qmode=oracle.QMODE_POW2)
    assert np.all(L0 > 0) and np.all(L1 > 0) and not np.allclose(L0, L1)
    # the search's loss is the column losses of the same quantiser
    s = oracle.scales(a, 0.5)
    assert np.isclose(L1[1], oracle.loss_cols(X, W, s, 4, 64, qmode=oracle.QMODE_POW2).sum(), rtol=1e-12)


# ---------------------------------------------------------------- balanced scale
# (laojiahuo2003.github.io GPTQ/AWQ/SmoothQuant notes, section 4.4: s_j = mean|X_j|^alpha / mean|W_j|^(1-alpha))

def test_weight_mean_closed_form():
    rng = np.random.default_rng(8)
    W = rng.standard_normal((40, 300)).astype(np.float32)
    want = np.array([math.fsum(np.abs(W[j]).astype(np.float64)) / 300 for j in range(40)], dtype=np.float32)
    assert np.allclose(oracle.weight_mean(W), want, rtol=2e-7, atol=0)


def test_weight_mean_hand_worked():
    """Worked 4 x 5 example of the weight statistic (golden file): the mean
    magnitude of input channel j's row, rounded to fp32 once."""
    g = json.load(open(os.path.join(GOLDEN, "weight_mean_hand.json")))
    W = np.array(g["W_rows"], dtype=np.float32)
    assert W.shape == (g["D_in"], g["D_out"])
    got = oracle.weight_mean(W)
    assert got.dtype == np.float32
    assert got.tolist() == [float(np.float32(v)) for v in g["mean_abs_rows_fp32"]]
    assert hex(int(got[3:4].view(np.uint32)[0])) == g["fp32_bits_row_3"].lower()


def test_balanced_scale_closed_forms():
    rng = np.random.default_rng(9)
    a = (rng.random(50) + 0.1).astype(np.float32)
    b = (rng.random(50) + 0.1).astype(np.float32)
    # alpha = 1: the plain activation scale; alpha = 0: 1 / b; alpha = 1/2: sqrt(a / b)
    assert np.array_equal(oracle.scales(a, 1.0, w_mean=b), oracle.scales(a, 1.0))
    assert np.array_equal(oracle.scales(a, 0.0, w_mean=b), (1.0 / b.astype(np.float64)).astype(np.float32))
    half = np.sqrt(a.astype(np.float64) / b.astype(np.float64)).astype(np.float32)
    assert np.allclose(oracle.scales(a, 0.5, w_mean=b), half, rtol=1e-7, atol=0)


def test_balanced_scale_floors_a_zero_weight_row():
    a = np.array([1.0, 2.0, 4.0], dtype=np.float32)
    b = np.array([0.0, 1.0, 2.0], dtype=np.float32)
    s = oracle.scales(a, 0.0, w_mean=b)
    assert np.isfinite(s).all() and s[0] == np.float32(1.0 / np.float32(1e-6 * np.float32(2.0)))


def test_balanced_search_with_unit_weight_means_is_the_plain_search():
    X, W = synth.layer_inputs(synth.small_layer(48, 128, 12, seed=4))
    a = oracle.act_stats(X).astype(np.float32)
    grid = np.array([0.0, 0.25, 0.5, 1.0], np.float32)
    L0, b0 = oracle.search(X, W, a, grid, 4, 64)
    L1, b1 = oracle.search(X, W, a, grid, 4, 64, w_mean=np.ones(128, np.float32))
    assert np.array_equal(L0, L1) and b0 == b1


# ---------------------------------------------------------------- dense 3-bit packing

def test_pack3_worked_example():
    # codes 0..31 of one column: u_i = q_i + 4 with q_i = (i % 8) - 4, i.e. u_i = i % 8;
    # the 96-bit string is sum_i u_i 2^(3i); read it back 3 bits at a time
    q = ((np.arange(32) % 8) - 4).astype(np.int8).reshape(32, 1)
    w = oracle.pack3(q)
    assert w.shape == (3, 1)
    big = int(w[0, 0]) | (int(w[1, 0]) << 32) | (int(w[2, 0]) << 64)
    assert big == sum((i % 8) << (3 * i) for i in range(32))
    # code 10 straddles words 0 and 1 (bits 30..32), code 21 words 1 and 2 (bits 63..65)
    assert (int(w[0, 0]) >> 30) | ((int(w[1, 0]) & 1) << 2) == 10 % 8
    assert (int(w[1, 0]) >> 31) | ((int(w[2, 0]) & 3) << 1) == 21 % 8


def test_pack3_round_trip_random():
    rng = np.random.default_rng(12)
    q = rng.integers(-4, 4, size=(96, 7)).astype(np.int8)
    w = oracle.pack3(q)
    for j in range(3):
        for n in range(7):
            big = int(w[3 * j, n]) | (int(w[3 * j + 1, n]) << 32) | (int(w[3 * j + 2, n]) << 64)
            got = [((big >> (3 * i)) & 7) - 4 for i in range(32)]
            assert got == q[32 * j:32 * j + 32, n].tolist()


def test_pack3_is_three_quarters_of_the_nibble_format():
    q = np.zeros((256, 5), np.int8)
    assert oracle.pack3(q).size * 4 == oracle.pack(q, 3).size * 3


# ---------------------------------------------------------------- asymmetric (MinMax, zero-point) quantiser
# (compassingai.com concept page, "the AWQ mechanism": absmax or MinMax; "symmetric or
# asymmetric both work".  Range [min(0, min w'), max(0, max w')], delta = range / (2^b - 1),
# z = round(-lo / delta), u = clamp(round(w' / delta) + z, 0, 2^b - 1), w ~ (u - z) delta.)

def test_asym_worked_example():
    W = np.array([[0.5], [-1.0], [0.26], [0.74]], dtype=np.float32)
    q, d, z = oracle.quantize_asym(W, None, 4, 4)
    rng_ = np.float32(np.float32(0.74) - np.float32(-1.0))
    assert d[0, 0] == np.float32(rng_ / np.float32(15.0))              # 1.74 / 15 = 0.116
    assert z[0, 0] == 9                                                # round(1 / 0.116) = round(8.62)
    assert q[:, 0].tolist() == [4, -9, 2, 6]                           # u = 13, 0, 11, 15


def test_asym_one_sided_groups():
    pos = np.array([[0.0], [0.3], [1.5], [0.75]], dtype=np.float32)   # lo = 0: z = 0, max -> 15
    q, d, z = oracle.quantize_asym(pos, None, 4, 4)
    assert z[0, 0] == 0 and q[:, 0].tolist() == [0, 3, 15, 8] and d[0, 0] == np.float32(np.float32(1.5) / 15)
    neg = -pos                                                          # hi = 0: z = 15, min -> u = 0
    q, d, z = oracle.quantize_asym(neg, None, 4, 4)
    assert z[0, 0] == 15 and (q[:, 0] + 15).tolist() == [15, 12, 0, 7]


def test_asym_brute_force_and_invariants():
    rng = np.random.default_rng(21)
    W = (rng.standard_normal((64, 5)) + rng.normal(0, 1, (1, 5))).astype(np.float32)
    W[5, 2] = 0.0
    s = (rng.random(64) + 0.5).astype(np.float32)
    for bits in (2, 3, 4):
        q, d, z = oracle.quantize_asym(W, s, bits, 32)
        umax = (1 << bits) - 1
        for g in range(2):
            for n in range(5):
                wp = (s[32 * g:32 * g + 32] * W[32 * g:32 * g + 32, n]).astype(np.float32)
                lo, hi = min(np.float32(0), wp.min()), max(np.float32(0), wp.max())
                assert d[g, n] == np.float32(np.float32(hi - lo) / np.float32(umax))
                assert 0 <= z[g, n] <= umax
                for k in range(32):
                    u = int(q[32 * g + k, n]) + int(z[g, n])
                    assert 0 <= u <= umax
                    t = float(np.float32(wp[k] / d[g, n]))
                    cand = np.arange(umax + 1) - int(z[g, n])            # signed codes reachable
                    err = np.abs(cand - t)
                    best = cand[err == err.min()]
                    want = best[0] if len(best) == 1 else best[best % 2 == 0][0]   # ties to even
                    assert q[32 * g + k, n] == want
        # an exact zero stays exactly zero
        assert q[5, 2] == 0


def test_asym_search_uses_the_quantiser():
    X, W = synth.layer_inputs(synth.small_layer(64, 128, 16, seed=6))
    a = oracle.act_stats(X).astype(np.float32)
    grid = np.array([0.0, 0.5], np.float32)
    L2, _ = oracle.search(X, W, a, grid, 4, 64, qmode=oracle.QMODE_ASYMMETRIC)
    s = oracle.scales(a, 0.5)
    q, d, z = oracle.quantize_asym(W, s, 4, 64)
    e = q.astype(np.float64) * np.repeat(d, 64, axis=0) / s.astype(np.float64)[:, None] - W.numpy()
    x = X.float().numpy().astype(np.float64)
    assert np.isclose(L2[1], ((x @ e) ** 2).sum(), rtol=1e-10)
    # the asymmetric grid is finer for one-signed groups: a lower loss than the symmetric one here
    L0, _ = oracle.search(X, W, a, grid, 4, 64)
    assert np.all(L2 > 0) and not np.allclose(L0, L2)


def test_pack_unsigned_layout():
    u = (np.arange(16) % 16).astype(np.int16).reshape(16, 1)
    w = oracle.pack_unsigned(u)
    assert w.shape == (2, 1) and int(w[0, 0]) == 0x76543210 and int(w[1, 0]) == 0xFEDCBA98


# ---------------------------------------------------------------- W4A16 from asymmetric (zero-point) codes
def test_w4a16_zp_closed_form():
    """One group of 32 rows, x = 1, s = 1, codes u_k = k mod 16, zero point 3,
    delta 0.5: Y = 0.5 (sum_k u_k - 32 * 3) = 0.5 (2 * 120 - 96) = 72."""
    u = (np.arange(32) % 16).reshape(32, 1)
    packed = oracle.pack_unsigned(u)
    X = torch.ones(1, 32).to(torch.bfloat16)
    Y = oracle.w4a16_zp(X, np.ones(32, np.float32), packed, np.full((1, 1), 0.5, np.float32),
                        np.full((1, 1), 3, np.uint8), 32)
    assert Y.shape == (1, 1) and Y[0, 0] == 72.0


@pytest.mark.parametrize("bits,group", [(4, 128), (3, 64), (2, 32)])
def test_w4a16_zp_with_the_middle_zero_point_is_the_symmetric_consumer(bits, group):
    """z = 2^(b-1) in every group reduces the zero-point consumer to the
    offset-binary one, operation for operation."""
    X, W = synth.layer_inputs(synth.small_layer(5, 256, 24, seed=71))
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.5)
    q, d = oracle.quantize(W, s, bits, group)
    packed = oracle.pack(q, bits)
    z = np.full(d.shape, 1 << (bits - 1), np.uint8)
    assert np.array_equal(oracle.w4a16_zp(X, s, packed, d, z, group), oracle.w4a16(X, s, packed, d, bits, group))


@pytest.mark.parametrize("bits,group", [(4, 128), (3, 64), (2, 32)])
def test_w4a16_zp_applies_the_asymmetric_quantiser(bits, group):
    """Packed u = q + z from the MinMax quantiser, read back through the zero
    points: the output is X S^-1 (q delta) (numpy fp64 matmul on the
    quantiser's own codes), so a wrong nibble, group or zero-point index fails."""
    X, W = synth.layer_inputs(synth.small_layer(7, 256, 40, seed=72))
    W = W + 0.01                                        # groups with non-trivial zero points
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.4)
    q, d, z = oracle.quantize_asym(W, s, bits, group)
    assert len(np.unique(z)) > 1
    u = q.astype(np.int16) + np.repeat(z, group, axis=0).astype(np.int16)
    Y = oracle.w4a16_zp(X, s, oracle.pack_unsigned(u), d, z, group)
    w_hat = q * np.repeat(d, group, axis=0).astype(np.float64) / s.astype(np.float64)[:, None]
    assert np.allclose(Y, X.double().numpy() @ w_hat, rtol=1e-12, atol=1e-12)
