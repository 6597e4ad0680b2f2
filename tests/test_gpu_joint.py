"""GPU parity of the joint search of linears that share one input (q/k/v,
gate/up: one scale vector, the sum of their losses) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_bounds import check_alpha
from post_weight_only_b200 import synth

pytestmark = pytest.mark.gpu

L_RTOL = 1e-2


@pytest.fixture(scope="module")
def awq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from post_weight_only_b200 import awq as mod
    return mod


@pytest.mark.parametrize("N,D_in,douts,bits,group", [
    (300, 512, (256, 64, 64), 4, 128),      # q/k/v-like, grouped-query widths
    (130, 384, (200, 132), 3, 64),          # gate/up-like, ragged widths
    (64, 256, (4,), 4, 128),                # one layer
])
def test_joint_against_oracle(awq, N, D_in, douts, bits, group):
    X, _ = synth.layer_inputs(synth.small_layer(N, D_in, 8, seed=N))
    Ws = [synth.make_w(D_in, d, 0.02, 300 + i) for i, d in enumerate(douts)]
    a = oracle.act_stats(X).astype(np.float32)
    alphas = synth.alpha_grid(20).numpy()
    r = awq.search_joint(X.cuda(), [W.cuda() for W in Ws], torch.from_numpy(a).cuda(), alphas.tolist(), bits, group)
    L_or, best_or, per_or = oracle.search_joint(X, Ws, a, alphas, bits, group)
    L = r.L.cpu().numpy()
    per = r.L_layers.cpu().numpy()
    assert np.allclose(L, L_or, rtol=L_RTOL, atol=0)
    assert np.allclose(per, per_or, rtol=L_RTOL, atol=0)
    assert np.allclose(per.sum(axis=0), L, rtol=1e-12)
    idx = int(r.alpha_idx.item())
    assert idx == int(np.argmin(L))
    check_alpha(L_or, best_or, idx)
    assert float(r.alpha_star.item()) == alphas[idx]


def test_joint_equals_search_of_side_by_side_weights(awq):
    X, _ = synth.layer_inputs(synth.small_layer(700, 512, 8, seed=5))
    Ws = [synth.make_w(512, d, 0.02, 400 + i).cuda() for i, d in enumerate((384, 128, 128))]
    Xd = X.cuda()
    a = awq.act_stats(Xd)
    grid = synth.alpha_grid(20).tolist()
    r = awq.search_joint(Xd, Ws, a, grid, 4, 128)
    rc = awq.search(Xd, torch.cat(Ws, dim=1), a, grid, 4, 128)
    assert torch.equal(r.L, rc.L) and int(r.alpha_idx.item()) == int(rc.alpha_idx.item())
