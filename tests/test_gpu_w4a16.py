"""GPU parity of the W4A16 consumer of the pack format (the quantised layer
applied to activations) against the oracle, on codes packed by the library
itself.

Three CUDA paths: one or two tokens run the CUDA-core GEMV (fp32 throughout:
x / s rounded once to fp32, exact integer weights, delta applied per group);
three to eight tokens run the mma.sync GEMV (x / s rounded once to bf16,
exact integer codes, fp32 accumulation, the fp32 delta applied per group;
longer rows than it stages take the neighbouring path); more tokens run the
tcgen05 GEMM.  The bound below, derived for the GEMM, covers the GEMVs'
smaller errors too.

Tolerance, from the arithmetic of the tensor-core path: x_tk / s_k is rounded to
bf16 once, each weight q * bf16(delta) is rounded to bf16 once (relative
errors at most 2^-9 each, modelled as independent and uniform; the model
allows uniform errors up to U = 2^-8 per term, which covers both), and delta
is rounded to bf16 once per (group, column): a relative error of at most
2^-9 shared by the whole group, bounded deterministically.  Accumulation is
fp32.  Per output
    |Y_gpu - Y| <= 6 sqrt(sum_k x_tk^2 w_kn^2 U^2 / 3)
                   + 2^-9 sum_g |sum_{k in g} x_tk w_kn| + 1e-5 sum_k |x_tk w_kn|.
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


def _bound(x, w_hat, group):
    """x [N][D_in] fp64, w_hat [D_in][D_out] the exact dequantised weights
    (with 1/s)."""
    G = w_hat.shape[0] // group
    per_group = np.zeros((x.shape[0], w_hat.shape[1]))
    for g in range(G):
        sl = slice(g * group, (g + 1) * group)
        per_group += np.abs(x[:, sl] @ w_hat[sl])
    return (6.0 * np.sqrt((x ** 2) @ (w_hat ** 2) * U * U / 3.0) + 2.0 ** -9 * per_group
            + 1e-5 * (np.abs(x) @ np.abs(w_hat)))


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
    bound = _bound(X.double().numpy(), w_hat, group)
    return Y, Y_or, bound


@pytest.mark.parametrize("N,D_in,D_out,bits,group", [
    (1, 4096, 4096, 4, 128),      # one decode token: the GEMV, split K
    (2, 512, 200, 4, 128),        # GEMV: ragged second column tile
    (4, 1024, 132, 3, 64),        # mma.sync GEMV, 3-bit, ragged column tile
    (1, 32, 4, 4, 32),            # GEMV: one group, four k8 rows (fewer than the warps), one column quad
    (2, 2048, 256, 4, 256),       # GEMV, group 256
    (3, 256, 1000, 2, 32),        # mma.sync GEMV, 2-bit, group 32
    (1, 256, 38912, 4, 128),      # GEMV: more column tiles (304) than resident CTAs, one CTA per whole tile
    (2, 1024, 38916, 4, 64),      # the same with a ragged last tile of one column quad, 8-row batches
    (1, 128, 2048, 4, 64),        # GEMV: too few batches for clusters, stream-K shares and the reduce launch
    (4, 1024, 32768, 4, 128),     # mma.sync GEMV, four tokens: 256 tiles, unsplit
    (3, 1024, 32768, 2, 32),      # mma.sync GEMV, three tokens, 2-bit, group 32: 256 tiles, unsplit
    (5, 512, 200, 4, 128),        # ragged columns, a few tokens
    (16, 96, 36, 4, 32),          # D_in not a multiple of 64: a half k block
    (37, 384, 132, 3, 64),
    (300, 1024, 260, 4, 128),     # two token tiles of 256, no split
    (64, 256, 128, 2, 128),
    (33, 4160, 1024, 4, 32),      # D_in % 64 == 32 (a half k block), two groups per k block, split K
    (1000, 512, 4096, 4, 64),     # 128 units of (128 columns x 256 tokens): more units than one per CTA
    (17, 8192, 2048, 3, 128),     # Nt = 32, 16 column tiles: stream-K, shares inside one unit
    (8, 256, 65536, 4, 128),      # 512 units of 4 k blocks: a CTA's share spans whole units + partial ends
    (5, 1024, 200, 4, 256),       # group 256: one delta row per 4-k-block stage
    (300, 768, 256, 4, 256),      # group 256, large token tile (one k block per stage)
    (32, 2048, 640, 4, 64),       # the largest 4-k-block-stage token tile (Nt = 32), group 64
    (33, 2048, 640, 4, 128),      # the smallest 2-k-block-stage token tile (Nt = 48)
    (3, 1056, 96, 2, 32),         # group 32 (two groups per k block), 2-bit, D_in not a multiple of 256
    (3, 65536, 128, 4, 128),      # 3-4 tokens: eight CTAs of 8192 rows, the largest X' in shared memory
    (3, 65792, 64, 4, 256),       # past that range: the CUDA-core GEMV at three tokens
    (4, 4096, 1280, 3, 64),       # 3-4 tokens: ten tiles split eight ways
    (4, 96, 4, 4, 32),            # 3-4 tokens: three groups over eight warps, one column quad
    (6, 4096, 1028, 2, 32),       # 5-8 tokens: 256-column tiles, ragged last tile, 2-bit
    (8, 32768, 512, 4, 128),      # eight tokens: eight CTAs of 4096 rows, the largest X' in shared memory
    (5, 33024, 64, 4, 256),       # past that range: the tcgen05 GEMM at five tokens
])
def test_w4a16_against_oracle(awq, N, D_in, D_out, bits, group):
    Y, Y_or, bound = _case(awq, N, D_in, D_out, bits, group, seed=N + D_in)
    assert np.all(np.abs(Y - Y_or) <= bound), np.max(np.abs(Y - Y_or) / bound)


def test_w4a16_reproducible(awq):
    Y1, _, _ = _case(awq, 3, 1024, 512, 4, 128, seed=1)
    Y2, _, _ = _case(awq, 3, 1024, 512, 4, 128, seed=1)
    assert np.array_equal(Y1, Y2)


@pytest.mark.parametrize("N,D_in,D_out", [
    (1, 28672, 8192),     # the timed decode configuration (split K, two x~ chunks per split)
    (4, 28672, 8192),
    (2, 8192, 32768),     # few splits, long splits: two x~ chunks each
])
def test_w4a16_decode_full_size(awq, N, D_in, D_out):
    """A 70B-class down projection (D_in 28672, D_out 8192) at one and four
    tokens, the GEMV configuration that is timed, and a wide layer; sampled
    columns checked against the oracle's definition."""
    bits, group = 4, 128
    g = torch.Generator().manual_seed(11 + N)
    X = (torch.randn(N, D_in, generator=g) * 0.5).to(torch.bfloat16)
    s = torch.rand(D_in, generator=g) + 0.5
    packed = torch.randint(-2 ** 31, 2 ** 31 - 1, (D_in // 8, D_out), generator=g, dtype=torch.int64).to(torch.int32)
    scales = torch.rand(D_in // group, D_out, generator=g) * 0.01 + 1e-3
    Y = awq.w4a16_gemm(X.cuda(), s.cuda(), packed.cuda(), scales.cuda(), bits, group).cpu().numpy()
    cols = np.random.default_rng(0).choice(D_out, size=64, replace=False)
    p_np = packed.numpy().view(np.uint32)[:, cols]
    sc_np = scales.numpy()[:, cols]
    Y_or = oracle.w4a16(X, s.numpy(), np.ascontiguousarray(p_np), np.ascontiguousarray(sc_np), bits, group)
    k = np.arange(D_in)
    u = (p_np[k // 8] >> (4 * (k % 8))[:, None]) & 0xF
    w_hat = (u.astype(np.float64) - 8) * np.repeat(sc_np, group, axis=0).astype(np.float64) / \
        s.numpy().astype(np.float64)[:, None]
    bound = _bound(X.double().numpy(), w_hat, group)
    assert np.all(np.abs(Y[:, cols] - Y_or) <= bound), np.max(np.abs(Y[:, cols] - Y_or) / bound)


@pytest.mark.parametrize("N,D_in,D_out", [(1, 4096, 512), (2, 64, 128), (3, 1024, 256), (8, 1024, 256)])
def test_w4a16_output_only_4_byte_aligned(awq, N, D_in, D_out):
    """Y may be 4-byte aligned only (the ABI's requirement): the GEMVs then
    store scalars (the mma.sync GEMV always does); the values are those of an
    aligned Y, bit for bit (the same sums in the same order)."""
    X, W = synth.layer_inputs(synth.small_layer(max(N, 8), D_in, D_out, seed=3))
    X = X[:N].contiguous().cuda()
    s = torch.from_numpy(oracle.scales(oracle.act_stats(X.cpu()).astype(np.float32), 0.5)).cuda()
    packed, sc = awq.quantize_pack(W.cuda(), s, 4, 64)
    Y_ref = awq.w4a16_gemm(X, s, packed, sc, 4, 64)
    buf = torch.full((N * D_out + 1,), float("nan"), device="cuda")
    Y_off = buf[1:].view(N, D_out)                    # 4 bytes past a 256-byte-aligned allocation
    assert Y_off.data_ptr() % 16 == 4
    awq.w4a16_gemm(X, s, packed, sc, 4, 64, out=Y_off)
    assert torch.equal(Y_off, Y_ref)


def test_w4a16_rejects_unaligned_columns(awq):
    X = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")
    s = torch.ones(128, device="cuda")
    packed = torch.zeros(16, 6, dtype=torch.int32, device="cuda")
    scales = torch.ones(1, 6, device="cuda")
    with pytest.raises(awq.AwqError):
        awq.w4a16_gemm(X, s, packed, scales, 4, 128)


# ------------------------------------------------------------ asymmetric (zero-point) codes
def _zp_case(awq, N, D_in, D_out, bits, group, seed):
    """Codes, deltas and zero points from the oracle's MinMax quantiser
    (oracle.quantize_asym, packed by oracle.pack_unsigned), applied by the CUDA
    consumer and by oracle.w4a16_zp."""
    X, W = synth.layer_inputs(synth.small_layer(max(N, 8), D_in, D_out, seed=seed))
    X = X[:N].contiguous()
    s = oracle.scales(oracle.act_stats(X).astype(np.float32), 0.5)
    q, d, z = oracle.quantize_asym(W, s, bits, group)
    u = q.astype(np.int16) + np.repeat(z, group, axis=0).astype(np.int16)
    packed = oracle.pack_unsigned(u)
    Y = awq.w4a16_gemm(X.cuda(), torch.from_numpy(s).cuda(), torch.from_numpy(packed.view(np.int32)).cuda(),
                       torch.from_numpy(d).cuda(), bits, group,
                       zeros=torch.from_numpy(z).cuda()).cpu().numpy().astype(np.float64)
    Y_or = oracle.w4a16_zp(X, s, packed, d, z, group)
    w_hat = q * np.repeat(d, group, axis=0).astype(np.float64) / s.astype(np.float64)[:, None]
    return Y, Y_or, _bound(X.double().numpy(), w_hat, group)


@pytest.mark.parametrize("N,D_in,D_out,bits,group", [
    (1, 4096, 512, 4, 128),       # GEMV, split K
    (3, 1024, 132, 3, 64),        # GEMV, ragged column tile
    (4, 256, 1000, 2, 32),        # GEMV, 2-bit, group 32
    (2, 2048, 256, 4, 256),       # GEMV, group 256
    (1, 1024, 32768, 4, 128),     # GEMV: stream-K shares and the reduce launch
    (3, 256, 38912, 4, 64),       # GEMV: one CTA per whole tile
    (5, 512, 200, 4, 128),        # mma.sync GEMV, ragged columns
    (7, 1024, 520, 3, 64),        # mma.sync GEMV, seven tokens
    (9, 512, 200, 4, 128),        # tensor cores, stream-K, ragged columns
    (37, 384, 132, 3, 64),
    (17, 8192, 2048, 4, 128),     # stream-K shares inside one unit
    (300, 1024, 260, 4, 128),     # two token tiles, no split
    (64, 1056, 96, 2, 32),        # group 32: two delta and zero rows per k block; half k block
    (300, 768, 256, 4, 256),      # group 256, large token tile
])
def test_w4a16_zero_point_against_oracle(awq, N, D_in, D_out, bits, group):
    Y, Y_or, bound = _zp_case(awq, N, D_in, D_out, bits, group, seed=N + 7 * D_in)
    assert np.all(np.abs(Y - Y_or) <= bound), np.max(np.abs(Y - Y_or) / bound)


def test_w4a16_zero_point_matches_symmetric_at_the_midpoint(awq):
    """With every zero point equal to 2^(b-1) the asymmetric consumer reads the
    offset-binary codes of the symmetric pack: both paths give the same Y bit
    for bit (GEMV and tensor cores)."""
    for N in (2, 40):
        X, W = synth.layer_inputs(synth.small_layer(max(N, 8), 1024, 256, seed=N))
        X = X[:N].contiguous().cuda()
        s = torch.from_numpy(oracle.scales(oracle.act_stats(X.cpu()).astype(np.float32), 0.5)).cuda()
        packed, sc = awq.quantize_pack(W.cuda(), s, 4, 128)
        z = torch.full((1024 // 128, 256), 8, dtype=torch.uint8, device="cuda")
        assert torch.equal(awq.w4a16_gemm(X, s, packed, sc, 4, 128, zeros=z), awq.w4a16_gemm(X, s, packed, sc, 4, 128))
