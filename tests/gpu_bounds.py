"""Tolerance on the GPU's loss derived from the arithmetic of the CUDA path,
shared by the GPU parity tests.

The tensor cores see bf16 operands and accumulate in fp32:
  * error form: the operand E = (q - w'/delta) * fl(delta / s_k) is formed in
    fp32 from the quantiser's exact rounding residual (the quotient w'/delta
    taken through the reciprocal of delta, which moves it by at most 1e-6 of
    a step) and rounded to bf16 once, so the noise eta on an element has
    variance var <= E^2 U^2 / 3 + (1e-6 delta / s_k)^2;
  * reference form: the dequantised weight q * fl(delta / s_k) is rounded to
    bf16 once and the reference weight w once: var <= (w_hat^2 + w^2) U^2 / 3.
With independent element errors, L_gpu - L = 2 <XE, X eta> + ||X eta||^2: the
first term has variance 4 sum_kn var_kn (X^T X E)_kn^2, the second the mean
sum_kn (sum_i x_ik^2) var_kn.  The bound is k_sigma standard deviations of the
first plus three times the mean of the second, per output column, computed
from the oracle's own q, delta and s.  The fp32 accumulation error
(~sqrt(D_in) 2^-24 relative) is far below these terms.
"""
import numpy as np

import oracle

U_BF16 = 2.0 ** -8     # largest relative rounding error of one bf16 rounding


def activations64(X):
    """X in fp64 and its per-channel sums of squares, for rounding_bound."""
    x = X.float().numpy().astype(np.float64)
    return x, (x ** 2).sum(axis=0)


def rounding_bound(X, W, a, alpha, bits, group, form="error", cols=None, k_sigma=6.0, x64=None,
                   qmode=0, w_mean=None):
    """Per-column bound on |L_gpu - L| for the columns `cols` (all if None).
    Only those columns of W are quantised and expanded: the quantiser works
    column by column.  x64 = activations64(X) may be passed to save its cost.
    qmode / w_mean: the quantiser and scale variants (see oracle.search)."""
    s = oracle.scales(a, alpha, w_mean=w_mean).astype(np.float64)
    Wc = W if cols is None else W[:, np.asarray(cols)].contiguous()
    q, d = oracle.quantize(Wc, s.astype(np.float32), bits, group, qmode=qmode)
    w = Wc.numpy().astype(np.float64)
    step = np.repeat(d, group, axis=0).astype(np.float64) / s[:, None]      # delta / s_k
    w_hat = q.astype(np.float64) * step
    E = w_hat - w
    x, xsq = activations64(X) if x64 is None else x64
    if form == "reference":
        var = (w_hat ** 2 + w ** 2) * U_BF16 ** 2 / 3.0
    else:
        var = (E * U_BF16) ** 2 / 3.0 + (1e-6 * step) ** 2
    G = x.T @ (x @ E)
    cross_sd = np.sqrt(4.0 * (var * G ** 2).sum(axis=0))          # per column
    quad = (xsq[:, None] * var).sum(axis=0)                        # per column
    return k_sigma * cross_sd + 3.0 * quad


def check_alpha(L_or, best_or, idx_gpu):
    """alpha* identical, or the oracle's loss at the GPU's alpha* within 1% of
    the oracle's minimum."""
    if idx_gpu == best_or:
        return
    assert L_or[idx_gpu] <= 1.01 * L_or[best_or], (idx_gpu, best_or, L_or[idx_gpu], L_or[best_or])
