"""CPU oracle for the AWQ per-layer scale search (numpy front end).

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg are the only code allowed to import this package; the
library's product path never does.  The arithmetic lives in plain C
(``awq_oracle.c``), built here with gcc on first use.

Each wrapper names the passage of the AWQ pages it follows; see the C file's
header for the page list and the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "awq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_awq.so")

STAT_MEAN = 0
STAT_MAX = 1

# quantiser modes: delta = max / (2^(b-1) - 1), codes in +-(2^(b-1) - 1); or
# delta = max / 2^(b-1), codes in [-2^(b-1), 2^(b-1) - 1]
QMODE_SYMMETRIC = 0
QMODE_POW2 = 1
QMODE_ASYMMETRIC = 2     # MinMax with a zero point: codes u in [0, 2^b - 1], w ~ (u - z) delta

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE fp32 quantiser: no fast-math, no FMA
    contraction).  Returns the path of the shared library."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        F = ctypes.c_float
        lib.oracle_act_stats.argtypes = [P, I64, I64, I, P]
        lib.oracle_act_stats.restype = None
        lib.oracle_scales.argtypes = [P, I64, F, P]
        lib.oracle_scales.restype = None
        lib.oracle_quantize.argtypes = [P, P, I64, I64, I, I, P, P]
        lib.oracle_quantize.restype = None
        lib.oracle_quantize_clip.argtypes = [P, P, P, I64, I64, I, I, P, P]
        lib.oracle_quantize_clip.restype = None
        lib.oracle_quantize_ex.argtypes = [P, P, P, I64, I64, I, I, I, P, P]
        lib.oracle_quantize_ex.restype = None
        lib.oracle_w4a16.argtypes = [P, P, P, P, I64, I64, I64, I, I, P]
        lib.oracle_w4a16.restype = None
        lib.oracle_w4a16_zp.argtypes = [P, P, P, P, P, I64, I64, I64, I, P]
        lib.oracle_w4a16_zp.restype = None
        lib.oracle_clip_loss.argtypes = [P, P, P, I64, I64, I64, P, I, I, I, P, I64, P, P]
        lib.oracle_clip_loss.restype = None
        lib.oracle_pack3.argtypes = [P, I64, I64, P]
        lib.oracle_pack3.restype = None
        lib.oracle_pack.argtypes = [P, I64, I64, I, P]
        lib.oracle_pack.restype = None
        lib.oracle_loss_cols.argtypes = [P, P, P, I64, I64, I64, I, I, I, P, I64, P]
        lib.oracle_loss_cols.restype = None
        lib.oracle_search.argtypes = [P, P, P, I64, I64, I64, P, I, I, I, P, I64, P, P]
        lib.oracle_search.restype = I
        lib.oracle_quantize_mode.argtypes = [P, P, P, I64, I64, I, I, I, I, P, P]
        lib.oracle_quantize_mode.restype = None
        lib.oracle_quantize_asym.argtypes = [P, P, I64, I64, I, I, I, P, P, P]
        lib.oracle_quantize_asym.restype = None
        lib.oracle_weight_mean.argtypes = [P, I64, I64, P]
        lib.oracle_weight_mean.restype = None
        lib.oracle_scales_balanced.argtypes = [P, P, I64, F, P]
        lib.oracle_scales_balanced.restype = None
        lib.oracle_loss_cols_mode.argtypes = [P, P, P, I64, I64, I64, I, I, I, I, P, I64, P]
        lib.oracle_loss_cols_mode.restype = None
        lib.oracle_search_mode.argtypes = [P, P, P, P, I64, I64, I64, P, I, I, I, I, P, I64, P, P]
        lib.oracle_search_mode.restype = I
        lib.oracle_literal_loss.argtypes = [P, P, P, I64, I64, I64, I, I]
        lib.oracle_literal_loss.restype = ctypes.c_longdouble
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = I
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _as_bf16_bits(X) -> np.ndarray:
    """Accept a torch bf16 tensor or a uint16 array of bf16 bit patterns."""
    if isinstance(X, np.ndarray):
        assert X.dtype == np.uint16
        return np.ascontiguousarray(X)
    import torch
    assert X.dtype == torch.bfloat16
    return np.ascontiguousarray(X.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _f32(a) -> np.ndarray:
    if not isinstance(a, np.ndarray):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def act_stats(X, stat: int = STAT_MEAN) -> np.ndarray:
    """a_j = mean_i |X_ij| (or max), fp64.  compassingai.com concept page,
    "statistical basis of salient channels"."""
    Xb = _as_bf16_bits(X)
    N, D = Xb.shape
    a = np.empty(D, dtype=np.float64)
    _load().oracle_act_stats(_ptr(Xb), N, D, stat, _ptr(a))
    return a


def scales(a, alpha: float, w_mean=None) -> np.ndarray:
    """s_j = a_j^alpha (floored), fp32.  compassingai.com concept page, flow
    step 3.  With w_mean: the balanced scale s_j = a_j^alpha /
    w_mean_j^(1 - alpha) (laojiahuo2003.github.io GPTQ/AWQ/SmoothQuant notes, section 4.4, "the scale
    per channel"), both statistics floored."""
    a = _f32(a)
    s = np.empty_like(a)
    if w_mean is None:
        _load().oracle_scales(_ptr(a), a.shape[0], float(alpha), _ptr(s))
    else:
        b = _f32(w_mean)
        _load().oracle_scales_balanced(_ptr(a), _ptr(b), a.shape[0], float(alpha), _ptr(s))
    return s


def weight_mean(W) -> np.ndarray:
    """w_mean_j = mean_n |W_jn| over input channel j's row (fp64 sum, one fp32
    rounding): the weight statistic of the balanced scale."""
    W = _f32(W)
    out = np.empty(W.shape[0], dtype=np.float32)
    _load().oracle_weight_mean(_ptr(W), W.shape[0], W.shape[1], _ptr(out))
    return out


def quantize(W, s, bits: int, group: int, clip=None, delta16: bool = False,
             qmode: int = QMODE_SYMMETRIC) -> Tuple[np.ndarray, np.ndarray]:
    """Codes q [D_in, D_out] (int8) and deltas [D_in/group, D_out] (fp32) of
    diag(s).W.  compassingai.com concept page, "quantisation math".  clip:
    optional [D_in/group, D_out] fp32 clip ratios (the group maximum is
    replaced by fl32(clip * max) before delta is formed).  delta16: delta is
    rounded to FP16 (mudrobot.github.io notes: delta stored in FP16) and the
    codes use that value; the returned deltas are then FP16-representable.
    qmode QMODE_POW2: delta = max / 2^(b-1) (mudrobot.github.io notes,
    "analysing the quantisation error"), codes clamped to [-2^(b-1), 2^(b-1) - 1]."""
    W = _f32(W)
    D_in, D_out = W.shape
    s = None if s is None else _f32(s)
    q = np.empty((D_in, D_out), dtype=np.int8)
    d = np.empty((D_in // group, D_out), dtype=np.float32)
    c = None
    if clip is not None:
        c = _f32(clip)
        assert c.shape == (D_in // group, D_out)
    _load().oracle_quantize_mode(_ptr(W), _ptr(s), _ptr(c), D_in, D_out, bits, group, int(bool(delta16)),
                                 int(qmode), _ptr(q), _ptr(d))
    return q, d


def quantize_asym(W, s, bits: int, group: int, delta16: bool = False):
    """The asymmetric (MinMax, zero-point) quantiser of diag(s).W (concept
    page, "the AWQ mechanism": absmax or MinMax; symmetric or asymmetric).
    Returns (signed codes q = u - z [D_in, D_out] int8, deltas
    [D_in/group, D_out] fp32, zero points z [D_in/group, D_out] uint8); the
    stored codes are u = q + z in [0, 2^b - 1]."""
    W = _f32(W)
    D_in, D_out = W.shape
    s = None if s is None else _f32(s)
    q = np.empty((D_in, D_out), dtype=np.int8)
    d = np.empty((D_in // group, D_out), dtype=np.float32)
    z = np.empty((D_in // group, D_out), dtype=np.uint8)
    _load().oracle_quantize_asym(_ptr(W), _ptr(s), D_in, D_out, bits, group, int(bool(delta16)), _ptr(q), _ptr(d),
                                 _ptr(z))
    return q, d, z


def pack_unsigned(u: np.ndarray) -> np.ndarray:
    """Nibble packing of unsigned codes u in [0, 15] (natural order, no
    offset): the layout of pack() with u in place of q + 2^(b-1)."""
    u = np.asarray(u, dtype=np.int16)
    return pack((u - 8).astype(np.int8), 4)


def clip_search(X, W, s, clip_grid, bits: int, group: int, cols: Optional[Sequence[int]] = None,
                want_loss: bool = False):
    """Weight-clipping search (mudrobot.github.io notes, "searching the optimal
    scale": weight clipping to minimise the quantisation MSE): for every clip
    ratio of the grid, group and column, the fp64 squared error of that group's
    share of the layer output.  Returns (best [D_in/group, nc] int32 grid
    indices, loss [n_clip, D_in/group, nc] fp64 or None)."""
    Xb = _as_bf16_bits(X)
    W = _f32(W)
    s = None if s is None else _f32(s)
    grid = _f32(clip_grid)
    N, D_in = Xb.shape
    D_out = W.shape[1]
    c = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    nc = D_out if c is None else c.shape[0]
    G = D_in // group
    best = np.empty((G, nc), dtype=np.int32)
    loss = np.empty((grid.shape[0], G, nc), dtype=np.float64) if want_loss else None
    _load().oracle_clip_loss(_ptr(Xb), _ptr(W), _ptr(s), N, D_in, D_out, _ptr(grid), grid.shape[0], bits, group,
                             _ptr(c), 0 if c is None else nc, _ptr(loss), _ptr(best))
    return best, loss


def pack(q: np.ndarray, bits: int) -> np.ndarray:
    """uint32 [D_in/8, D_out]: 8 offset-binary codes per word, row 8k8+i in
    nibble i."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    D_in, D_out = q.shape
    out = np.empty((D_in // 8, D_out), dtype=np.uint32)
    _load().oracle_pack(_ptr(q), D_in, D_out, bits, _ptr(out))
    return out


def pack3(q: np.ndarray) -> np.ndarray:
    """Dense 3-bit packing of codes in [-4, 3]: words [D_in/32 * 3][D_out]
    (uint32), code i of rows 32j..32j+31 at bits 3i..3i+2 of the 96-bit string
    made of words 3j, 3j+1, 3j+2 (little-endian), as u = q + 4."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    D_in, D_out = q.shape
    out = np.empty((D_in // 32 * 3, D_out), dtype=np.uint32)
    _load().oracle_pack3(_ptr(q), D_in, D_out, _ptr(out))
    return out


def loss_cols(X, W, s, bits: int, group: int, cols: Optional[Sequence[int]] = None,
              quantize_w: bool = True, qmode: int = QMODE_SYMMETRIC) -> np.ndarray:
    """Per-column share of ||X S^-1 Q(S W) - X W||^2 (fp64) for one scale
    vector.  compassingai.com concept page, flow step 4c."""
    Xb = _as_bf16_bits(X)
    W = _f32(W)
    N, D_in = Xb.shape
    D_out = W.shape[1]
    s = None if s is None else _f32(s)
    c = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    nc = D_out if c is None else c.shape[0]
    out = np.empty(nc, dtype=np.float64)
    _load().oracle_loss_cols_mode(_ptr(Xb), _ptr(W), _ptr(s), N, D_in, D_out, bits, group,
                                  1 if quantize_w else 0, int(qmode), _ptr(c), 0 if c is None else nc, _ptr(out))
    return out


def search(X, W, a, alphas, bits: int, group: int, cols: Optional[Sequence[int]] = None,
           want_cols: bool = False, qmode: int = QMODE_SYMMETRIC, w_mean=None):
    """Grid search over alpha: returns (L [n_alpha] fp64, best index[, L_col]).

    compassingai.com concept page, flow steps 3-5; mudrobot.github.io notes,
    "searching the optimal scale" (alpha* = argmin L(s_X^alpha) on [0, 1]).
    qmode selects the quantiser (see quantize); w_mean switches to the
    balanced scale (see scales)."""
    Xb = _as_bf16_bits(X)
    W = _f32(W)
    a = _f32(a)
    al = _f32(alphas)
    N, D_in = Xb.shape
    D_out = W.shape[1]
    c = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    nc = D_out if c is None else c.shape[0]
    L = np.empty(al.shape[0], dtype=np.float64)
    Lc = np.empty((al.shape[0], nc), dtype=np.float64) if want_cols else None
    b = None if w_mean is None else _f32(w_mean)
    best = _load().oracle_search_mode(_ptr(Xb), _ptr(W), _ptr(a), _ptr(b), N, D_in, D_out, _ptr(al), al.shape[0],
                                      bits, group, int(qmode), _ptr(c), 0 if c is None else nc, _ptr(L), _ptr(Lc))
    if want_cols:
        return L, int(best), Lc
    return L, int(best)


def literal_loss(X, W, s, bits: int, group: int) -> float:
    """||(X S^-1) Q(S W) - X W||_F^2 with every matrix materialised, in long
    double (tiny layers only)."""
    Xb = _as_bf16_bits(X)
    W = _f32(W)
    s = _f32(s)
    N, D_in = Xb.shape
    return float(_load().oracle_literal_loss(_ptr(Xb), _ptr(W), _ptr(s), N, D_in, W.shape[1], bits, group))


def search_joint(X, Ws, a, alphas, bits: int, group: int):
    """Joint search of linears sharing one input and one scale vector
    (mudrobot.github.io AWQ notes: 1/s is fused into the previous operator, so
    q/k/v, or gate/up, take the same s): L(alpha) = sum_l L_l(alpha), each
    L_l the single-layer loss above; alpha* = argmin, lowest index on ties.
    Returns (L [n_alpha], best, L_layers [n_layers, n_alpha])."""
    per = np.stack([search(X, W, a, alphas, bits, group)[0] for W in Ws])
    L = per.sum(axis=0)
    best = int(np.flatnonzero(L == L.min())[0])
    return L, best, per


def w4a16(X, s, packed, scales, bits: int, group: int) -> np.ndarray:
    """Y = X diag(1/s) Dequant(W_q) in fp64 from the packed words and the
    per-group deltas (compassingai.com concept page, "inference-time
    equivalent")."""
    Xb = _as_bf16_bits(X)
    s = _f32(s)
    packed = np.ascontiguousarray(packed).view(np.uint32)
    scales = _f32(scales)
    N, D_in = Xb.shape
    D_out = packed.shape[1]
    Y = np.empty((N, D_out), dtype=np.float64)
    _load().oracle_w4a16(_ptr(Xb), _ptr(s), _ptr(packed), _ptr(scales), N, D_in, D_out, bits, group, _ptr(Y))
    return Y


def w4a16_zp(X, s, packed, scales, zeros, group: int) -> np.ndarray:
    """Y = X diag(1/s) Dequant(W_q) in fp64 from asymmetric codes: the stored
    u = q + z of quantize_asym, packed by pack_unsigned, minus each group's
    zero point z, times its delta."""
    Xb = _as_bf16_bits(X)
    s = _f32(s)
    packed = np.ascontiguousarray(packed).view(np.uint32)
    scales = _f32(scales)
    zeros = np.ascontiguousarray(zeros, dtype=np.uint8)
    N, D_in = Xb.shape
    D_out = packed.shape[1]
    Y = np.empty((N, D_out), dtype=np.float64)
    _load().oracle_w4a16_zp(_ptr(Xb), _ptr(s), _ptr(packed), _ptr(scales), _ptr(zeros), N, D_in, D_out, group,
                            _ptr(Y))
    return Y

