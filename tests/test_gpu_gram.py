"""GPU parity of the Gram form of the alpha search:
L(alpha) = sum_n e_n^T H e_n with H = X^T X, the same quantity as
||X S^-1 Q(S W) - X W||^2 (compassingai.com concept page, flow step 4c),
against the CPU oracle's direct evaluation.

Tolerance, from the arithmetic of the CUDA path: the operand E is rounded to
bf16 once per element (as in the error form: gpu_bounds.rounding_bound), and
H, accumulated in fp32 from the exact bf16 X, is rounded to bf16 once per
entry: L_gpu - L gains sum_jk e_j e_k dH_jk with independent |dH_jk| <=
2^-9 |H_jk|, modelled (generously) as uniform within 2^-8: 6 standard
deviations, 6 U / sqrt(3) sqrt(sum_jk e_j^2 e_k^2 H_jk^2) per column.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_bounds import check_alpha, rounding_bound
from post_weight_only_b200 import synth

pytestmark = pytest.mark.gpu

U = 2.0 ** -8


@pytest.fixture(scope="module")
def awq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from post_weight_only_b200 import awq as mod
    return mod


def _gram_bound(X, W, a, alpha, bits, group, qmode=oracle.QMODE_SYMMETRIC):
    s = oracle.scales(a, alpha)
    q, d = oracle.quantize(W, s, bits, group, qmode=qmode)
    w = W.numpy().astype(np.float64)
    e = q.astype(np.float64) * np.repeat(d, group, axis=0).astype(np.float64) / s.astype(np.float64)[:, None] - w
    x = X.float().numpy().astype(np.float64)
    H = x.T @ x
    tH = np.sqrt(np.einsum("jn,jk,kn->n", e ** 2, H ** 2, e ** 2))
    return 6.0 * U / np.sqrt(3.0) * tH


@pytest.mark.parametrize("N,D_in,D_out,bits,group", [
    (1000, 256, 200, 4, 128),    # N > D_in: the case the Gram form is for
    (1003, 384, 132, 3, 64),     # tokens not a multiple of 8 (padded in X^T), three 128-row tiles of H
    (100, 256, 64, 4, 128),      # N < D_in still evaluates the same loss
    (700, 96, 36, 2, 32),        # D_in not a multiple of 64 (a ragged k block and a ragged row tile of H)
])
def test_gram_search_against_oracle(awq, N, D_in, D_out, bits, group):
    X, W = synth.layer_inputs(synth.small_layer(N, D_in, D_out, seed=N + D_in))
    a = oracle.act_stats(X).astype(np.float32)
    alphas = synth.alpha_grid(10).numpy()
    res = awq.search(X.cuda(), W.cuda(), torch.from_numpy(a).cuda(), alphas.tolist(), bits, group, gram=True,
                     want_cols=True)
    L_gpu = res.L.cpu().numpy()
    L_or, best = oracle.search(X, W, a, alphas, bits, group)
    for i, al in enumerate(alphas):
        bound = rounding_bound(X, W, a, al, bits, group, "error").sum() + _gram_bound(X, W, a, al, bits, group).sum()
        err = abs(L_gpu[i] - L_or[i])
        assert err <= bound, (al, L_gpu[i], L_or[i], bound)
        assert err <= 1e-2 * L_or[i], (al, err / L_or[i])
    assert np.allclose(res.L_col.cpu().numpy().sum(axis=1), L_gpu, rtol=1e-9)
    check_alpha(L_or, best, int(res.alpha_idx.item()))


def test_gram_search_asymmetric(awq):
    """The Gram form with the asymmetric quantiser's operand."""
    N, D_in, D_out, bits, group = 900, 256, 136, 4, 64
    qm = oracle.QMODE_ASYMMETRIC
    X, W = synth.layer_inputs(synth.small_layer(N, D_in, D_out, seed=77))
    a = oracle.act_stats(X).astype(np.float32)
    alphas = synth.alpha_grid(10).numpy()
    res = awq.search(X.cuda(), W.cuda(), torch.from_numpy(a).cuda(), alphas.tolist(), bits, group, gram=True,
                     quantizer=awq.QUANT_ASYMMETRIC)
    L_gpu = res.L.cpu().numpy()
    L_or, best = oracle.search(X, W, a, alphas, bits, group, qmode=qm)
    for i, al in enumerate(alphas):
        bound = (rounding_bound(X, W, a, al, bits, group, "error", qmode=qm).sum()
                 + _gram_bound(X, W, a, al, bits, group, qmode=qm).sum())
        err = abs(L_gpu[i] - L_or[i])
        assert err <= bound, (al, L_gpu[i], L_or[i], bound)
        assert err <= 1e-2 * L_or[i], (al, err / L_or[i])
    check_alpha(L_or, best, int(res.alpha_idx.item()))


def test_gram_search_matches_direct_search(awq):
    """The Gram and direct GPU forms choose alpha* by the contract's rule
    against each other's losses, on a layer where N = 4 D_in."""
    X, W = synth.layer_inputs(synth.small_layer(1024, 256, 256, seed=5))
    a = torch.from_numpy(oracle.act_stats(X).astype(np.float32)).cuda()
    grid = synth.alpha_grid(20).tolist()
    r_dir = awq.search(X.cuda(), W.cuda(), a, grid, 4, 128)
    r_gram = awq.search(X.cuda(), W.cuda(), a, grid, 4, 128, gram=True)
    L_dir, L_gram = r_dir.L.cpu().numpy(), r_gram.L.cpu().numpy()
    assert np.allclose(L_gram, L_dir, rtol=1e-2)
    check_alpha(L_dir, int(r_dir.alpha_idx.item()), int(r_gram.alpha_idx.item()))
