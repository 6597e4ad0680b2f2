"""GPU parity of the pack with FP16 deltas (mudrobot.github.io AWQ notes:
delta stored in FP16): codes, packed words and the FP16 scales bit-exact
against the oracle, with and without clip ratios, on both pack kernels."""
import numpy as np
import pytest
import torch

import oracle
from post_weight_only_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def awq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from post_weight_only_b200 import awq as mod
    return mod


@pytest.mark.parametrize("bits,group,D_in,D_out,use_clip", [
    (4, 128, 256, 200, False),
    (3, 64, 192, 132, True),
    (4, 32, 96, 203, False),        # D_out % 4 != 0: the untiled kernel
    (4, 128, 1024, 4096, True),
    (2, 128, 128, 36, True),
])
def test_pack_delta_fp16(awq, bits, group, D_in, D_out, use_clip):
    X, W = synth.layer_inputs(synth.small_layer(16, D_in, D_out, seed=D_in + D_out + bits))
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.45)
    clip = None
    if use_clip:
        rng = np.random.default_rng(D_out)
        clip = synth.clip_grid(20).numpy()[rng.integers(0, 21, size=(D_in // group, D_out))]
    packed, sc = awq.quantize_pack_ex(W.cuda(), torch.from_numpy(s).cuda(), bits, group,
                                      clip=None if clip is None else torch.from_numpy(clip).cuda(), delta_fp16=True)
    assert sc.dtype == torch.float16
    q_or, d_or = oracle.quantize(W, s, bits, group, clip=clip, delta16=True)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack(q_or, bits))
    assert np.array_equal(sc.cpu().numpy().astype(np.float32), d_or)


def test_pack_ex_without_flags_is_the_plain_pack(awq):
    X, W = synth.layer_inputs(synth.small_layer(16, 256, 128, seed=3))
    s = torch.from_numpy(oracle.scales(oracle.act_stats(X).astype(np.float32), 0.5)).cuda()
    p0, s0 = awq.quantize_pack(W.cuda(), s, 4, 128)
    p1, s1 = awq.quantize_pack_ex(W.cuda(), s, 4, 128)
    assert torch.equal(p0, p1) and torch.equal(s0, s1)
