"""The exact-arithmetic identities the W4A16 kernels rest on, checked on the
CPU with IEEE float32/bfloat16 bit patterns (no GPU):

  * GEMV: for a nibble u at bits 4i..4i+3 (i < 4) of a word,
    (word & (0xF << 4i)) | 0x4B000000 read as fp32 is 2^23 + 16^i u exactly,
    and subtracting 2^23 + 16^i off leaves 16^i (u - off) exactly; a product
    (x 16^-i) * 16^i (u - off) equals x (u - off) rounded once;
  * tensor-core dequantiser: ((word >> 4q) & 0x000F000F) | 0x43004300 read as
    two bf16 values is {128 + u_q, 128 + u_{q+4}} exactly, and subtracting
    128 + off in bf16 is exact.
"""
import numpy as np
import pytest
import torch


def _f32(bits):
    return np.asarray(bits, dtype=np.uint32).view(np.float32)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_gemv_nibble_magic_is_exact(bits):
    off = 1 << (bits - 1)
    for i in range(4):
        u = np.arange(1 << bits, dtype=np.uint32)
        # every other nibble of the word set to 0xF: the mask must isolate nibble i
        word = (u << (4 * i)) | (np.uint32(0xFFFFFFFF) ^ np.uint32(0xF << (4 * i)))
        f = _f32((word & np.uint32(0xF << (4 * i))) | np.uint32(0x4B000000))
        assert np.array_equal(f.astype(np.float64), 2.0 ** 23 + 16.0 ** i * u)
        bias = np.float32(2.0 ** 23 + 16.0 ** i * off)
        v = f - bias                                            # one fp32 subtraction
        assert np.array_equal(v.astype(np.float64), 16.0 ** i * (u.astype(np.float64) - off))


def test_gemv_high_nibbles_after_shift():
    rng = np.random.default_rng(0)
    w = rng.integers(0, 2 ** 32, size=1000, dtype=np.uint64).astype(np.uint32)
    wh = w >> np.uint32(16)
    for i in range(4):
        u_direct = (w >> np.uint32(4 * (i + 4))) & np.uint32(0xF)
        f = _f32((wh & np.uint32(0xF << (4 * i))) | np.uint32(0x4B000000))
        assert np.array_equal(f.astype(np.float64), 2.0 ** 23 + 16.0 ** i * u_direct)


def test_gemv_power_of_two_folding_is_exact():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(4096) * np.exp(rng.uniform(-8, 8, 4096))).astype(np.float32)
    for i in range(4):
        xt = x * np.float32(16.0 ** -i)                         # exact: a power of two, no underflow here
        assert np.array_equal(xt.astype(np.float64) * 16.0 ** i, x.astype(np.float64))
        for k in range(-8, 8):
            lhs = np.float32(xt * np.float32(16.0 ** i * k))   # x~ * 16^i (u - off)
            rhs = np.float32(x * np.float32(k))                # x (u - off)
            assert np.array_equal(lhs, rhs)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_tensor_core_bf16_pair_magic_is_exact(bits):
    off = 1 << (bits - 1)
    rng = np.random.default_rng(bits)
    w = rng.integers(0, 2 ** 32, size=4096, dtype=np.uint64).astype(np.uint32)
    mask = np.uint32((1 << bits) - 1)
    w = w & np.uint32(int("".join(["{:x}".format((1 << bits) - 1)] * 8), 16))   # codes below 2^bits
    for q in range(4):
        pair = ((w >> np.uint32(4 * q)) & np.uint32(0x000F000F)) | np.uint32(0x43004300)
        lo = torch.from_numpy((pair & np.uint32(0xFFFF)).astype(np.int32).astype(np.int16)).view(torch.bfloat16)
        hi = torch.from_numpy((pair >> np.uint32(16)).astype(np.int32).astype(np.int16)).view(torch.bfloat16)
        u_lo = (w >> np.uint32(4 * q)) & mask
        u_hi = (w >> np.uint32(4 * (q + 4))) & mask
        assert np.array_equal(lo.double().numpy(), 128.0 + u_lo)
        assert np.array_equal(hi.double().numpy(), 128.0 + u_hi)
        bias = torch.tensor(128.0 + off, dtype=torch.bfloat16)
        assert np.array_equal((lo - bias).double().numpy(), u_lo.astype(np.float64) - off)
        assert np.array_equal((hi - bias).double().numpy(), u_hi.astype(np.float64) - off)
