"""The C-ABI library builds, loads and exports every symbol its header
declares; host-side argument checks reject bad calls before any device work
(no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "awq_b200.h")


@pytest.fixture(scope="module")
def lib():
    from post_weight_only_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^AWQ_API\s+[\w\s\*]+?\b(awq_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("awq_act_stats", "awq_search", "awq_quantize_pack", "awq_scales", "awq_get_last_error"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_lists_every_export():
    from post_weight_only_b200 import awq
    assert sorted(awq.EXPORTS) == declared_functions()


def _err(lib):
    lib.awq_get_last_error.restype = ctypes.c_char_p
    return lib.awq_get_last_error().decode()


def test_argument_checks_without_gpu(lib):
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    f = lib.awq_act_stats
    f.argtypes = [P, I64, I64, I, P, P]
    f.restype = I
    fake = 0x10000  # never dereferenced: checks run first
    assert f(fake, 0, 64, 0, fake, None) == 1            # N = 0
    assert "N = 0" in _err(lib)
    assert f(fake, 16, 12, 0, fake, None) == 1           # D_in not a multiple of 8
    assert f(fake, 16, 64, 7, fake, None) == 1           # bad stat
    assert f(fake + 4, 16, 64, 0, fake, None) == 2       # misaligned X
    assert f(None, 16, 64, 0, fake, None) == 1           # NULL X

    s = lib.awq_search
    s.argtypes = [P, P, P, I64, I64, I64, P, I, I, I, I, P, P, P, P, P, ctypes.c_size_t, P, P]
    s.restype = I
    grid = (ctypes.c_float * 3)(0.0, 0.5, 1.0)
    args = dict(X=fake, W=fake, a=fake, N=64, D_in=256, D_out=64, grid=grid, A=3, bits=4, group=128, form=0,
                L=fake, Lc=None, astar=fake, aidx=fake, ws=fake, wsb=1 << 20, st=None, stream=None)

    def call(**kw):
        d = dict(args, **kw)
        return s(d["X"], d["W"], d["a"], d["N"], d["D_in"], d["D_out"], d["grid"], d["A"], d["bits"], d["group"],
                 d["form"], d["L"], d["Lc"], d["astar"], d["aidx"], d["ws"], d["wsb"], d["st"], d["stream"])

    assert call(bits=5) == 3
    assert call(bits=1) == 3
    assert call(group=96) == 3
    assert call(group=512) == 3
    assert call(group=256, D_in=384) == 1                 # not a multiple of group 256
    assert call(D_in=192) == 1                            # not a multiple of group 128
    assert call(A=0) == 3
    assert call(A=65) == 3
    assert call(D_out=6) == 1
    assert call(N=0) == 1
    assert call(W=fake + 8) == 2
    assert call(grid=None) == 1
    assert call(form=2) == 1

    c = lib.awq_clip_search
    c.argtypes = [P, P, P, I64, I64, I64, P, I, I, I, P, P, P, P, ctypes.c_size_t, P, P]
    c.restype = I
    cgrid = (ctypes.c_float * 3)(1.0, 0.75, 0.5)
    cargs = dict(X=fake, W=fake, s=fake, N=64, D_in=256, D_out=64, grid=cgrid, C=3, bits=4, group=128, clip=fake,
                 idx=None, loss=None, ws=fake, wsb=1 << 20, st=None, stream=None)

    def ccall(**kw):
        d = dict(cargs, **kw)
        return c(d["X"], d["W"], d["s"], d["N"], d["D_in"], d["D_out"], d["grid"], d["C"], d["bits"], d["group"],
                 d["clip"], d["idx"], d["loss"], d["ws"], d["wsb"], d["st"], d["stream"])

    assert ccall(group=32) == 3                           # the clipping search takes groups of 64 and 128
    assert ccall(bits=5) == 3
    assert ccall(C=0) == 3
    assert ccall(D_in=192) == 1
    assert ccall(grid=None) == 1
    assert ccall(grid=(ctypes.c_float * 3)(1.0, 0.0, 0.5)) == 1         # ratios must lie in (0, 1]
    assert ccall(grid=(ctypes.c_float * 3)(1.0, 1.5, 0.5)) == 1
    assert ccall(clip=None) == 1
    assert ccall(s=fake + 4) == 2
    cws = lib.awq_clip_search_workspace_size
    cws.argtypes = [I64, I64, I64, I, I, I]
    cws.restype = ctypes.c_size_t
    assert cws(64, 256, 64, 3, 4, 32) == 0
    assert cws(64, 256, 64, 3, 4, 128) > 0                 # the layout needs no device

    q = lib.awq_quantize_pack
    q.argtypes = [P, P, I64, I64, I, I, P, P, P]
    q.restype = I
    assert q(fake, fake, 256, 64, 4, 100, fake, fake, None) == 3
    assert q(fake, fake, 200, 64, 4, 128, fake, fake, None) == 1
    assert q(fake, fake, 256, 64, 6, 128, fake, fake, None) == 3

    g = lib.awq_w4a16_gemm
    SZ = ctypes.c_size_t
    g.argtypes = [P, P, P, P, I64, I64, I64, I, I, P, P, SZ, P, P]
    g.restype = I
    gws = lib.awq_w4a16_workspace_size
    gws.argtypes = [I64, I64, I64]
    gws.restype = SZ
    assert gws(16, 4096, 4096) >= 16 * 4096 * 2            # the scaled activations, bf16
    for n in (1, 2, 4):                                    # decode GEMV: two tiles of CTA sums per CTA
        assert gws(n, 4096, 4096) >= 1024 * 2 * n * 128 * 4
    assert gws(5, 4096, 4096) >= 5 * 4096 * 2              # five tokens: the tensor-core layout
    gargs = dict(X=fake, s=fake, P=fake, sc=fake, N=16, D_in=256, D_out=64, bits=4, group=128, Y=fake, ws=fake,
                 wsb=gws(16, 256, 64), st=fake, stream=None)

    def gcall(**kw):
        d = dict(gargs, **kw)
        return g(d["X"], d["s"], d["P"], d["sc"], d["N"], d["D_in"], d["D_out"], d["bits"], d["group"], d["Y"],
                 d["ws"], d["wsb"], d["st"], d["stream"])

    assert gcall(D_out=66) == 1                           # rows of packed words must be 16-byte multiples
    assert gcall(N=0) == 1
    assert gcall(group=512) == 3
    assert gcall(D_in=192) == 1
    assert gcall(s=fake + 4) == 2                          # s is read as float4
    assert gcall(ws=None) == 4
    assert gcall(wsb=gws(16, 256, 64) - 1) == 4
    assert gcall(st=None) == 1                             # the status word is required

    class Opts(ctypes.Structure):
        _fields_ = [("quantizer", ctypes.c_int), ("w_mean", ctypes.c_void_p), ("gram_form", ctypes.c_int),
                    ("ldw", ctypes.c_int64)]

    x = lib.awq_search_ex
    x.argtypes = [P, P, P, I64, I64, I64, P, I, I, I, I, ctypes.POINTER(Opts), P, P, P, P, P, ctypes.c_size_t, P, P]
    x.restype = I

    def xcall(opts, **kw):
        d = dict(args, **kw)
        return x(d["X"], d["W"], d["a"], d["N"], d["D_in"], d["D_out"], d["grid"], d["A"], d["bits"], d["group"],
                 d["form"], opts, d["L"], d["Lc"], d["astar"], d["aidx"], d["ws"], d["wsb"], d["st"], d["stream"])

    assert xcall(ctypes.byref(Opts(3, None, 0))) == 1        # unknown quantiser
    assert xcall(ctypes.byref(Opts(1, fake + 2, 0))) == 2    # misaligned weight means
    assert xcall(ctypes.byref(Opts(1, None, 0)), bits=5) == 3   # the common checks still apply
    assert xcall(ctypes.byref(Opts(0, None, 0, 32))) == 1    # row stride below D_out
    assert xcall(ctypes.byref(Opts(0, None, 0, 66))) == 1    # row stride not a multiple of 4
    xws = lib.awq_search_ex_workspace_size
    xws.argtypes = [I64, I64, I64, I, I, I, I, ctypes.POINTER(Opts)]
    xws.restype = ctypes.c_size_t
    assert xws(64, 256, 64, 3, 4, 128, 1, ctypes.byref(Opts(0, None, 1))) == 0   # Gram form: error form only
    wm = lib.awq_weight_mean
    wm.argtypes = [P, I64, I64, P, P]
    wm.restype = I
    assert wm(fake, 0, 16, fake, None) == 1
    assert wm(fake + 4, 16, 16, fake, None) == 2
    se = lib.awq_scales_ex
    se.argtypes = [P, P, I64, ctypes.c_float, P, P, P]
    se.restype = I
    assert se(fake, fake, 16, 1.5, None, fake, None) == 1    # alpha outside [0, 1]
    assert se(fake, fake + 2, 16, 0.5, None, fake, None) == 2
    pe = lib.awq_quantize_pack_ex
    pe.argtypes = [P, P, P, I64, I64, I, I, I, P, P, P]
    pe.restype = I
    assert pe(fake, fake, None, 256, 64, 4, 128, 8, fake, fake, None) == 1   # unknown flag bit
    assert pe(fake, fake, None, 256, 64, 4, 128, 4, fake, fake, None) == 1   # dense packing needs 3-bit codes
    assert pe(fake, fake, None, 256, 66, 3, 64, 4, fake, fake, None) == 3    # dense, D_out % 4 != 0, group 64
    zp = lib.awq_quantize_pack_zp
    zp.argtypes = [P, P, I64, I64, I, I, I, P, P, P, P]
    zp.restype = I
    assert zp(fake, fake, 256, 64, 4, 128, 2, fake, fake, fake, None) == 1     # no power-of-two delta
    assert zp(fake, fake, 256, 64, 4, 128, 0, fake, fake, None, None) == 1     # zeros is required
    assert zp(fake, fake, 256, 64, 4, 128, 4, fake, fake, fake, None) == 1     # dense needs 3-bit codes
    assert zp(fake, fake, 250, 64, 4, 128, 0, fake, fake, fake, None) == 1     # D_in % group != 0

    t = lib.awq_selftest_wait_timeout
    t.argtypes = [P, I64, P]
    t.restype = I
    assert t(fake, 10, None) == 1                          # timeout below 1 us
    dv = lib.awq_selftest_divide
    dv.argtypes = [I, P, P]
    dv.restype = I
    assert dv(0, fake, None) == 1                          # divisor below 1
    assert dv(256, fake, None) == 1                        # divisor above 255
    assert dv(7, fake + 4, None) == 2                      # misaligned output


def test_no_device_is_reported_not_crashed(lib):
    """On a machine without a usable sm_100 GPU a well-formed call fails with
    AWQ_ECUDA or AWQ_EUNSUPPORTED; it never falls back to a CPU path."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    f = lib.awq_act_stats
    f.argtypes = [P, I64, I64, I, P, P]
    f.restype = I
    rc = f(0x10000, 16, 64, 0, 0x10000, None)
    assert rc in (3, 5)


def test_version(lib):
    lib.awq_version.restype = ctypes.c_int
    assert lib.awq_version() >= 100
