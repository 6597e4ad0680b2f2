"""GPU parity of the W4A16 consumer of the pack format (the quantised layer
applied to activations) against the oracle, on codes packed by the library
itself.

Tolerance, from the arithmetic: each dequantised weight q * delta / s_k is
rounded to bf16 once (relative error at most 2^-8, modelled as independent
and uniform), X is exact, accumulation is fp32.  Per output
    |Y_gpu - Y| <= 6 sqrt(sum_k x_tk^2 w_kn^2 U^2 / 3) + 1e-5 sum_k |x_tk w_kn|.
"""
import numpy as np
import pytest
import torch

import oracle
from post_weight_only_b200 import synth

pytestmark = pytest.mark.gpu

U = 2.0 ** -8


@pytest.fixture(scope="module")
def awq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from post_weight_only_b200 import awq as mod
    return mod


def _case(awq, N, D_in, D_out, bits, group, seed):
    X, W = synth.layer_inputs(synth.small_layer(max(N, 8), D_in, D_out, seed=seed))
    X = X[:N].contiguous()
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.5)
    Wd = W.cuda()
    sd = torch.from_numpy(s).cuda()
    packed, sc = awq.quantize_pack(Wd, sd, bits, group)
    Y = awq.w4a16_gemm(X.cuda(), sd, packed, sc, bits, group).cpu().numpy().astype(np.float64)
    p_np = packed.cpu().numpy().view(np.uint32)
    sc_np = sc.cpu().numpy()
    Y_or = oracle.w4a16(X, s, p_np, sc_np, bits, group)
    q, d = oracle.quantize(W, s, bits, group)
    w_hat = q * np.repeat(d, group, axis=0).astype(np.float64) / s.astype(np.float64)[:, None]
    x = X.double().numpy()
    bound = 6.0 * np.sqrt((x ** 2) @ (w_hat ** 2) * U * U / 3.0) + 1e-5 * (np.abs(x) @ np.abs(w_hat))
    return Y, Y_or, bound


@pytest.mark.parametrize("N,D_in,D_out,bits,group", [
    (1, 4096, 4096, 4, 128),      # one decode token: split K over a cluster
    (5, 512, 200, 4, 128),        # ragged columns, a few tokens
    (16, 96, 36, 4, 32),          # D_in not a multiple of 64: a half k block
    (37, 384, 132, 3, 64),
    (300, 1024, 260, 4, 128),     # two token tiles of 256, no split
    (64, 256, 128, 2, 128),
])
def test_w4a16_against_oracle(awq, N, D_in, D_out, bits, group):
    Y, Y_or, bound = _case(awq, N, D_in, D_out, bits, group, seed=N + D_in)
    assert np.all(np.abs(Y - Y_or) <= bound), np.max(np.abs(Y - Y_or) / bound)


def test_w4a16_reproducible(awq):
    Y1, _, _ = _case(awq, 3, 1024, 512, 4, 128, seed=1)
    Y2, _, _ = _case(awq, 3, 1024, 512, 4, 128, seed=1)
    assert np.array_equal(Y1, Y2)
