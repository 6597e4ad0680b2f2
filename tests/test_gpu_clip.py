"""GPU parity of the weight-clipping search and the clipped pack (through the
C ABI) against the CPU oracle on the same seeded inputs.

Acceptance:
  * every loss L_c(g, n) within a bound derived from the arithmetic of the
    CUDA path: the Gram blocks H_g = X_g^T X_g and the operand e are each
    rounded to bf16 once per entry (relative error at most 2^-8, modelled as
    independent and uniform), so
        L_gpu - L ~ sum_jk e_j e_k dH_jk + 2 sum_j de_j (H e)_j,
    and the bound is 6 standard deviations of that (plus the fp32
    accumulation, far smaller);
  * the chosen ratio: identical to the oracle's, or the oracle's loss at the
    GPU's choice within 1% of the oracle's minimum (or within the two bounds);
  * the clipped pack: codes, packed words and scales bit-exact for the ratios
    the GPU chose.
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


def _bound(x, W, s, clip, bits, group):
    """[n_clip, G, D_out] bound on |L_gpu - L| (see the module docstring)."""
    G = W.shape[0] // group
    out = np.empty((len(clip), G, W.shape[1]))
    w = W.numpy().astype(np.float64)
    for i, c in enumerate(clip):
        q, d = oracle.quantize(W, s, bits, group, clip=np.full((G, W.shape[1]), c, np.float32))
        e = q.astype(np.float64) * np.repeat(d, group, axis=0).astype(np.float64) / s.astype(np.float64)[:, None] - w
        for g in range(G):
            sl = slice(g * group, (g + 1) * group)
            H = x[:, sl].T @ x[:, sl]
            eg = e[sl]
            He = H @ eg
            tH = np.sqrt(np.einsum("jn,kn,jk->n", eg ** 2, eg ** 2, H ** 2))
            tE = 2.0 * np.sqrt(((eg * He) ** 2).sum(axis=0))
            out[i, g] = 6.0 * (tH + tE) * U / np.sqrt(3.0) + 1e-30
    return out


@pytest.mark.parametrize("N,D_in,D_out,bits,group", [
    (256, 512, 512, 4, 128),     # the 512 x 512 / 256-token layer
    (300, 384, 200, 3, 64),      # ragged tokens (not a multiple of 8) and columns
    (300, 192, 132, 4, 64),      # three 64-row groups: a half-empty Gram block
    (1000, 1024, 260, 4, 128),   # more units than SMs... and a ragged 128-column block
    (1, 128, 64, 4, 128),        # a single token
    (64, 256, 4, 2, 128),        # four columns, 2-bit
])
def test_clip_search_against_oracle(awq, N, D_in, D_out, bits, group):
    X, W = synth.layer_inputs(synth.small_layer(N, D_in, D_out, seed=N + D_out))
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.5)
    grid = synth.clip_grid(20).numpy()
    res = awq.clip_search(X.cuda(), W.cuda(), torch.from_numpy(s).cuda(), grid.tolist(), bits, group, want_loss=True)
    torch.cuda.synchronize()
    L_gpu = res.loss.cpu().numpy().astype(np.float64)
    idx = res.idx.cpu().numpy()
    clip = res.clip.cpu().numpy()
    best, L_or = oracle.clip_search(X, W, s, grid, bits, group, want_loss=True)
    x = X.float().numpy().astype(np.float64)
    bound = _bound(x, W, s, grid, bits, group)
    assert np.all(np.abs(L_gpu - L_or) <= bound), np.max(np.abs(L_gpu - L_or) / bound)
    # the GPU's running argmin over its own losses
    assert np.array_equal(idx, np.argmin(L_gpu.astype(np.float32), axis=0))
    assert np.array_equal(clip, grid[idx])
    G = D_in // group
    gi, ni = np.meshgrid(np.arange(G), np.arange(D_out), indexing="ij")
    at_choice = L_or[idx, gi, ni]
    at_best = L_or[best, gi, ni]
    slack = np.maximum(0.01 * at_best, bound[idx, gi, ni] + bound[best, gi, ni])
    assert np.all(at_choice <= at_best + slack)
    # the clipped pack with the GPU's ratios, bit-exact
    packed, sc = awq.quantize_pack_clip(W.cuda(), torch.from_numpy(s).cuda(), res.clip, bits, group)
    q_or, d_or = oracle.quantize(W, s, bits, group, clip=clip)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack(q_or, bits))
    assert np.array_equal(sc.cpu().numpy(), d_or)


@pytest.mark.parametrize("bits,group,D_in,D_out", [(4, 128, 256, 203), (3, 64, 192, 132), (4, 32, 96, 40)])
def test_clipped_pack_bit_exact(awq, bits, group, D_in, D_out):
    """Random ratios on both pack kernels (D_out % 4 != 0 takes the untiled one)."""
    X, W = synth.layer_inputs(synth.small_layer(8, D_in, D_out, seed=D_out))
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.35)
    rng = np.random.default_rng(D_in)
    clip = synth.clip_grid(20).numpy()[rng.integers(0, 21, size=(D_in // group, D_out))]
    packed, sc = awq.quantize_pack_clip(W.cuda(), torch.from_numpy(s).cuda(), torch.from_numpy(clip).cuda(), bits,
                                        group)
    q_or, d_or = oracle.quantize(W, s, bits, group, clip=clip)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack(q_or, bits))
    assert np.array_equal(sc.cpu().numpy(), d_or)


def test_clip_one_equals_plain_pack(awq):
    X, W = synth.layer_inputs(synth.small_layer(8, 256, 128, seed=9))
    s = torch.from_numpy(oracle.scales(oracle.act_stats(X).astype(np.float32), 0.5)).cuda()
    p0, s0 = awq.quantize_pack(W.cuda(), s, 4, 128)
    p1, s1 = awq.quantize_pack_clip(W.cuda(), s, torch.ones(2, 128, device="cuda"), 4, 128)
    assert torch.equal(p0, p1) and torch.equal(s0, s1)


def test_clip_search_reproducible(awq):
    X, W = synth.layer_inputs(synth.small_layer(500, 512, 256, seed=4))
    s = torch.from_numpy(oracle.scales(oracle.act_stats(X).astype(np.float32), 0.5)).cuda()
    grid = synth.clip_grid(20).tolist()
    r1 = awq.clip_search(X.cuda(), W.cuda(), s, grid, 4, 128, want_loss=True)
    r2 = awq.clip_search(X.cuda(), W.cuda(), s, grid, 4, 128, want_loss=True)
    assert torch.equal(r1.loss, r2.loss) and torch.equal(r1.idx, r2.idx)
