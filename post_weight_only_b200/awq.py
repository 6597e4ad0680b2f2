"""Thin Python binding of the C ABI in ``include/awq_b200.h``.

Argument marshalling only: every step of the computation runs in the CUDA
library ``libawq_b200.so`` built in this package directory.  PyTorch supplies
device memory and the current stream.  There is no CPU fallback: importing this
module raises if the library is missing, and every call raises on a non-OK
status.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libawq_b200.so")

AWQ_OK, AWQ_EINVAL, AWQ_EALIGN, AWQ_EUNSUPPORTED, AWQ_EWORKSPACE, AWQ_ECUDA, AWQ_ETIMEOUT = range(7)
STAT_MEAN, STAT_MAX = 0, 1
LOSS_ERROR, LOSS_REFERENCE = 0, 1
MAX_ALPHA = 64

EXPORTS = (
    "awq_act_stats", "awq_scales", "awq_scales_dev", "awq_search_workspace_size", "awq_search",
    "awq_search_batched_workspace_size", "awq_search_batched", "awq_quantize_pack",
    "awq_layer_output_workspace_size", "awq_layer_output", "awq_selftest_wait_timeout", "awq_selftest_divide",
    "awq_get_last_error", "awq_version", "awq_profile_enable", "awq_profile_reset", "awq_profile_read",
    "awq_search_noalloc", "awq_clip_search_workspace_size", "awq_clip_search", "awq_quantize_pack_clip",
    "awq_search_joint_workspace_size", "awq_search_joint", "awq_quantize_pack_ex", "awq_w4a16_gemm",
    "awq_w4a16_workspace_size", "awq_search_ex", "awq_weight_mean", "awq_scales_ex", "awq_search_ex_workspace_size",
    "awq_quantize_pack_zp", "awq_w4a16_gemm_zp", "awq_w4a16_zp_workspace_size", "awq_act_stats_batched",
)
STAGES = ("act_stats", "scale_table", "search_operand", "search_gemm", "loss_reduce", "quantize_pack",
          "weight_t", "clip_gram", "clip_operand", "clip_loss", "w4a16")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m post_weight_only_b200.build` "
        "(nvcc, sm_100a); there is no fallback implementation")

_lib = ctypes.CDLL(LIB_PATH)

P = ctypes.c_void_p
I64 = ctypes.c_int64
I = ctypes.c_int
F = ctypes.c_float
SZ = ctypes.c_size_t


class AwqLayer(ctypes.Structure):
    _fields_ = [("X", P), ("W", P), ("a", P), ("N", I64), ("D_in", I64), ("D_out", I64),
                ("L", P), ("L_col", P), ("alpha_star", P), ("alpha_idx", P)]


def _sig(name, res, args):
    fn = getattr(_lib, name)
    fn.restype = res
    fn.argtypes = args
    return fn


_act_stats = _sig("awq_act_stats", I, [P, I64, I64, I, P, P])
_scales = _sig("awq_scales", I, [P, I64, F, P, P])
_scales_dev = _sig("awq_scales_dev", I, [P, I64, P, P, P])
_scales_ex = _sig("awq_scales_ex", I, [P, P, I64, F, P, P, P])
_weight_mean = _sig("awq_weight_mean", I, [P, I64, I64, P, P])
_search_ws = _sig("awq_search_workspace_size", SZ, [I64, I64, I64, I, I, I, I])
_search = _sig("awq_search", I, [P, P, P, I64, I64, I64, P, I, I, I, I, P, P, P, P, P, SZ, P, P])


class AwqSearchOptions(ctypes.Structure):
    _fields_ = [("quantizer", ctypes.c_int), ("w_mean", P), ("gram_form", ctypes.c_int), ("ldw", I64)]


QUANT_SYMMETRIC = 0
QUANT_DELTA_POW2 = 1
QUANT_ASYMMETRIC = 2
PACK_DELTA_POW2 = 2
PACK_DENSE3 = 4
_search_ex_ws = _sig("awq_search_ex_workspace_size", SZ, [I64, I64, I64, I, I, I, I,
                                                          ctypes.POINTER(AwqSearchOptions)])
_search_ex = _sig("awq_search_ex", I, [P, P, P, I64, I64, I64, P, I, I, I, I, ctypes.POINTER(AwqSearchOptions), P, P,
                                       P, P, P, SZ, P, P])
_batched_ws = _sig("awq_search_batched_workspace_size", SZ, [ctypes.POINTER(AwqLayer), I, I, I, I, I])
_batched = _sig("awq_search_batched", I, [ctypes.POINTER(AwqLayer), I, P, I, I, I, I, P, SZ, P, P])
_pack = _sig("awq_quantize_pack", I, [P, P, I64, I64, I, I, P, P, P])
_out_ws = _sig("awq_layer_output_workspace_size", SZ, [I64, I64, I64])
_out = _sig("awq_layer_output", I, [P, P, I64, I64, I64, P, P, SZ, P, P])
_selftest = _sig("awq_selftest_wait_timeout", I, [P, I64, P])
_selftest_div = _sig("awq_selftest_divide", I, [I, P, P])
_last_error = _sig("awq_get_last_error", ctypes.c_char_p, [])
_prof_enable = _sig("awq_profile_enable", I, [I])
_prof_reset = _sig("awq_profile_reset", I, [])
_prof_read = _sig("awq_profile_read", I, [I, P, P])
_version = _sig("awq_version", I, [])
_clip_ws = _sig("awq_clip_search_workspace_size", SZ, [I64, I64, I64, I, I, I])
_clip = _sig("awq_clip_search", I, [P, P, P, I64, I64, I64, P, I, I, I, P, P, P, P, SZ, P, P])
_pack_clip = _sig("awq_quantize_pack_clip", I, [P, P, P, I64, I64, I, I, P, P, P])
_joint_ws = _sig("awq_search_joint_workspace_size", SZ, [I64, I64, P, I, I, I, I, I])
_pack_ex = _sig("awq_quantize_pack_ex", I, [P, P, P, I64, I64, I, I, I, P, P, P])
_pack_zp = _sig("awq_quantize_pack_zp", I, [P, P, I64, I64, I, I, I, P, P, P, P])
PACK_DELTA_FP16 = 1
_w4a16 = _sig("awq_w4a16_gemm", I, [P, P, P, P, I64, I64, I64, I, I, P, P, SZ, P, P])
_w4a16_ws = _sig("awq_w4a16_workspace_size", SZ, [I64, I64, I64])
_w4a16_zp = _sig("awq_w4a16_gemm_zp", I, [P, P, P, P, P, I64, I64, I64, I, I, P, P, SZ, P, P])
_stats_batched = _sig("awq_act_stats_batched", I, [P, P, P, I, I, P, P])
_w4a16_zp_ws = _sig("awq_w4a16_zp_workspace_size", SZ, [I64, I64, I64, I])
_joint = _sig("awq_search_joint", I, [P, P, P, I, P, I64, I64, P, I, I, I, I, P, P, P, P, P, SZ, P, P])


class AwqError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"awq status {code}: {msg}")
        self.code = code


def _check(rc: int) -> None:
    if rc != AWQ_OK:
        raise AwqError(rc, _last_error().decode(errors="replace"))


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor, dtype: torch.dtype, name: str) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.contiguous()


def version() -> int:
    return int(_version())


def act_stats(X: torch.Tensor, stat: int = STAT_MEAN) -> torch.Tensor:
    """a_j = mean_i |X_ij| (or max): ``awq_act_stats``."""
    X = _dev(X, torch.bfloat16, "X")
    N, D = X.shape
    a = torch.empty(D, dtype=torch.float32, device=X.device)
    _check(_act_stats(_ptr(X), N, D, stat, _ptr(a), _stream()))
    return a


def act_stats_batched(Xs: Sequence[torch.Tensor], stat: int = STAT_MEAN) -> list:
    """The statistic of several inputs in one launch: ``awq_act_stats_batched``.
    Returns one fp32 [D_in] tensor per input."""
    Xs = [_dev(X, torch.bfloat16, "X") for X in Xs]
    outs = [torch.empty(X.shape[1], dtype=torch.float32, device=X.device) for X in Xs]
    n = len(Xs)
    xp = (ctypes.c_void_p * n)(*[X.data_ptr() for X in Xs])
    ns = (ctypes.c_int64 * n)(*[X.shape[0] for X in Xs])
    ds = (ctypes.c_int64 * n)(*[X.shape[1] for X in Xs])
    ap = (ctypes.c_void_p * n)(*[a.data_ptr() for a in outs])
    _check(_stats_batched(xp, ns, ds, n, stat, ap, _stream()))
    return outs


def weight_mean(W: torch.Tensor) -> torch.Tensor:
    """w_mean[j] = mean_n |W[j][n]|: ``awq_weight_mean`` (the weight statistic
    of the balanced scale)."""
    W = _dev(W, torch.float32, "W")
    out = torch.empty(W.shape[0], dtype=torch.float32, device=W.device)
    _check(_weight_mean(_ptr(W), W.shape[0], W.shape[1], _ptr(out), _stream()))
    return out


def scales(a: torch.Tensor, alpha, w_mean: Optional[torch.Tensor] = None) -> torch.Tensor:
    """s = a^alpha (floored): ``awq_scales`` for a host alpha, ``awq_scales_dev``
    when alpha is a one-element CUDA tensor; with w_mean the balanced
    a^alpha / w_mean^(1 - alpha) (``awq_scales_ex``)."""
    a = _dev(a, torch.float32, "a")
    s = torch.empty_like(a)
    if w_mean is not None:
        b = _dev(w_mean, torch.float32, "w_mean")
        if isinstance(alpha, torch.Tensor):
            al = _dev(alpha.reshape(1), torch.float32, "alpha")
            _check(_scales_ex(_ptr(a), _ptr(b), a.numel(), 0.0, _ptr(al), _ptr(s), _stream()))
        else:
            _check(_scales_ex(_ptr(a), _ptr(b), a.numel(), float(alpha), None, _ptr(s), _stream()))
        return s
    if isinstance(alpha, torch.Tensor):
        al = _dev(alpha.reshape(1), torch.float32, "alpha")
        _check(_scales_dev(_ptr(a), a.numel(), _ptr(al), _ptr(s), _stream()))
    else:
        _check(_scales(_ptr(a), a.numel(), float(alpha), _ptr(s), _stream()))
    return s


def search_workspace_size(N: int, D_in: int, D_out: int, n_alpha: int, bits: int, group: int,
                          loss_form: int = LOSS_ERROR) -> int:
    n = int(_search_ws(N, D_in, D_out, n_alpha, bits, group, loss_form))
    if n == 0:
        raise AwqError(AWQ_EINVAL, _last_error().decode(errors="replace"))
    return n


@dataclass
class SearchResult:
    L: torch.Tensor                 # [n_alpha] fp64
    alpha_star: torch.Tensor        # [1] fp32
    alpha_idx: torch.Tensor         # [1] int32
    L_col: Optional[torch.Tensor]   # [n_alpha, D_out] fp64 or None
    status: torch.Tensor            # [1] int32 device status word


class Workspace:
    """A reusable device workspace (grown on demand, 256-byte aligned)."""

    def __init__(self, device=None):
        self.buf = None
        self.device = device

    def get(self, nbytes: int, device) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != device:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        return self.buf


_default_ws = Workspace()


def search(X: torch.Tensor, W: torch.Tensor, a: torch.Tensor, alpha_grid: Sequence[float], bits: int = 4,
           group: int = 128, want_cols: bool = False, workspace: Optional[Workspace] = None,
           check_status: bool = True, loss_form: int = LOSS_ERROR, quantizer: int = QUANT_SYMMETRIC,
           w_mean: Optional[torch.Tensor] = None, gram: bool = False) -> SearchResult:
    """Grid search over alpha for one layer: ``awq_search``, or
    ``awq_search_ex`` with a quantiser variant, the balanced scale, the Gram
    form of the loss, or a W whose rows are further apart than D_out (a slice
    of output columns of a wider matrix, e.g. ``W[:, c0:c1]``, searched in
    place through the row stride ``ldw``)."""
    X = _dev(X, torch.bfloat16, "X")
    ldw = 0
    if (W.is_cuda and W.dtype == torch.float32 and W.dim() == 2 and W.stride(1) == 1
            and W.stride(0) > W.shape[1] and W.stride(0) % 4 == 0 and W.data_ptr() % 16 == 0):
        ldw = W.stride(0)           # a column slice: passed in place
    else:
        W = _dev(W, torch.float32, "W")
    a = _dev(a, torch.float32, "a")
    N, D_in = X.shape
    D_out = W.shape[1]
    grid = (ctypes.c_float * len(alpha_grid))(*[float(v) for v in alpha_grid])
    A = len(alpha_grid)
    dev = X.device
    L = torch.empty(A, dtype=torch.float64, device=dev)
    Lc = torch.empty(A, D_out, dtype=torch.float64, device=dev) if want_cols else None
    astar = torch.empty(1, dtype=torch.float32, device=dev)
    aidx = torch.empty(1, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    plain = quantizer == QUANT_SYMMETRIC and w_mean is None and not gram and ldw == 0
    b = None if w_mean is None else _dev(w_mean, torch.float32, "w_mean")
    opts = AwqSearchOptions(int(quantizer), _ptr(b), 1 if gram else 0, ldw)
    nbytes = (search_workspace_size(N, D_in, D_out, A, bits, group, loss_form) if plain
              else int(_search_ex_ws(N, D_in, D_out, A, bits, group, loss_form, ctypes.byref(opts))))
    if nbytes == 0:
        raise AwqError(AWQ_EINVAL, "awq_search_ex_workspace_size: invalid arguments")
    ws = (workspace or _default_ws).get(nbytes, dev)
    if plain:
        _check(_search(_ptr(X), _ptr(W), _ptr(a), N, D_in, D_out, grid, A, bits, group, loss_form, _ptr(L), _ptr(Lc),
                       _ptr(astar), _ptr(aidx), _ptr(ws), ws.numel(), _ptr(status), _stream()))
    else:
        _check(_search_ex(_ptr(X), _ptr(W), _ptr(a), N, D_in, D_out, grid, A, bits, group, loss_form,
                          ctypes.byref(opts), _ptr(L), _ptr(Lc), _ptr(astar), _ptr(aidx), _ptr(ws), ws.numel(),
                          _ptr(status), _stream()))
    res = SearchResult(L, astar, aidx, Lc, status)
    if check_status:
        check_device_status(status)
    return res


@dataclass
class ClipResult:
    clip: torch.Tensor                  # [D_in/group, D_out] fp32 chosen ratio
    idx: torch.Tensor                   # [D_in/group, D_out] int32 grid index
    loss: Optional[torch.Tensor]        # [n_clip, D_in/group, D_out] fp32, if asked for
    status: torch.Tensor


def clip_search(X: torch.Tensor, W: torch.Tensor, s: torch.Tensor, clip_grid: Sequence[float], bits: int = 4,
                group: int = 128, want_loss: bool = False, workspace: Optional[Workspace] = None,
                check_status: bool = True) -> ClipResult:
    """Weight-clipping search after the scale search: ``awq_clip_search``."""
    X = _dev(X, torch.bfloat16, "X")
    W = _dev(W, torch.float32, "W")
    s = _dev(s, torch.float32, "s")
    N, D_in = X.shape
    D_out = W.shape[1]
    C = len(clip_grid)
    grid = (ctypes.c_float * C)(*[float(v) for v in clip_grid])
    dev = X.device
    G = D_in // group
    clip = torch.empty(G, D_out, dtype=torch.float32, device=dev)
    idx = torch.empty(G, D_out, dtype=torch.int32, device=dev)
    loss = torch.empty(C, G, D_out, dtype=torch.float32, device=dev) if want_loss else None
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    nbytes = int(_clip_ws(N, D_in, D_out, C, bits, group))
    if nbytes == 0:
        raise AwqError(AWQ_EINVAL, _last_error().decode(errors="replace"))
    ws = (workspace or _default_ws).get(nbytes, dev)
    _check(_clip(_ptr(X), _ptr(W), _ptr(s), N, D_in, D_out, grid, C, bits, group, _ptr(clip), _ptr(idx), _ptr(loss),
                 _ptr(ws), ws.numel(), _ptr(status), _stream()))
    res = ClipResult(clip, idx, loss, status)
    if check_status:
        check_device_status(status)
    return res


def quantize_pack_ex(W: torch.Tensor, s: torch.Tensor, bits: int = 4, group: int = 128,
                     clip: Optional[torch.Tensor] = None, delta_fp16: bool = False, delta_pow2: bool = False,
                     dense3: bool = False):
    """``awq_quantize_pack_ex``: the final pack with optional clip ratios and
    FP16 deltas.  Returns (packed int32 view [D_in/8, D_out], scales
    [D_in/group, D_out] as float16 when delta_fp16 else float32)."""
    W = _dev(W, torch.float32, "W")
    s = _dev(s, torch.float32, "s")
    if clip is not None:
        clip = _dev(clip, torch.float32, "clip")
    D_in, D_out = W.shape
    rows = D_in // 32 * 3 if dense3 else D_in // 8
    packed = torch.empty(rows, D_out, dtype=torch.int32, device=W.device)
    sc = torch.empty(D_in // group, D_out, dtype=torch.float16 if delta_fp16 else torch.float32, device=W.device)
    flags = ((PACK_DELTA_FP16 if delta_fp16 else 0) | (PACK_DELTA_POW2 if delta_pow2 else 0)
             | (PACK_DENSE3 if dense3 else 0))
    _check(_pack_ex(_ptr(W), _ptr(s), _ptr(clip), D_in, D_out, bits, group, flags, _ptr(packed), _ptr(sc), _stream()))
    return packed, sc


def quantize_pack_zp(W: torch.Tensor, s: torch.Tensor, bits: int = 4, group: int = 128,
                     delta_fp16: bool = False, dense3: bool = False):
    """``awq_quantize_pack_zp``: the final pack with the asymmetric quantiser.
    Returns (packed int32 view, scales, zeros uint8 [D_in/group, D_out]); the
    codes are u = q + z."""
    W = _dev(W, torch.float32, "W")
    s = _dev(s, torch.float32, "s")
    D_in, D_out = W.shape
    rows = D_in // 32 * 3 if dense3 else D_in // 8
    packed = torch.empty(rows, D_out, dtype=torch.int32, device=W.device)
    sc = torch.empty(D_in // group, D_out, dtype=torch.float16 if delta_fp16 else torch.float32, device=W.device)
    zeros = torch.empty(D_in // group, D_out, dtype=torch.uint8, device=W.device)
    flags = (PACK_DELTA_FP16 if delta_fp16 else 0) | (PACK_DENSE3 if dense3 else 0)
    _check(_pack_zp(_ptr(W), _ptr(s), D_in, D_out, bits, group, flags, _ptr(packed), _ptr(sc), _ptr(zeros), _stream()))
    return packed, sc, zeros


def w4a16_gemm(X: torch.Tensor, s: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, bits: int = 4,
               group: int = 128, check_status: bool = True,
               workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
               zeros: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y = X diag(1/s) Dequant(packed, scales), fp32: ``awq_w4a16_gemm``, or
    with ``zeros`` (uint8 [D_in/group, D_out], from ``quantize_pack_zp``) the
    asymmetric codes' ``awq_w4a16_gemm_zp``.  ``workspace`` (uint8, at least
    ``w4a16_workspace_size(N, D_in, D_out[, group, zp=True])`` bytes) is
    allocated per call when not given; ``out`` (contiguous fp32 [N, D_out] on
    the same device) receives Y when given."""
    X = _dev(X, torch.bfloat16, "X")
    s = _dev(s, torch.float32, "s")
    if packed.dtype not in (torch.int32, torch.uint32):
        raise ValueError("packed must hold 32-bit words")
    packed = packed.contiguous()
    scales = _dev(scales, torch.float32, "scales")
    N, D_in = X.shape
    D_out = packed.shape[1]
    if out is None:
        Y = torch.empty(N, D_out, dtype=torch.float32, device=X.device)
    else:
        if out.dtype != torch.float32 or out.device != X.device or tuple(out.shape) != (N, D_out) \
                or not out.is_contiguous():
            raise ValueError("out must be a contiguous float32 [N, D_out] tensor on X's device")
        Y = out
    status = torch.empty(1, dtype=torch.int32, device=X.device)        # the call clears it
    nbytes = w4a16_workspace_size(N, D_in, D_out, group, zp=zeros is not None)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=X.device)
    if zeros is None:
        _check(_w4a16(_ptr(X), _ptr(s), _ptr(packed), _ptr(scales), N, D_in, D_out, bits, group, _ptr(Y),
                      _ptr(workspace), workspace.numel(), _ptr(status), _stream()))
    else:
        zeros = _dev(zeros, torch.uint8, "zeros")
        _check(_w4a16_zp(_ptr(X), _ptr(s), _ptr(packed), _ptr(scales), _ptr(zeros), N, D_in, D_out, bits, group,
                         _ptr(Y), _ptr(workspace), workspace.numel(), _ptr(status), _stream()))
    if check_status:
        check_device_status(status)
    return Y


def w4a16_workspace_size(N: int, D_in: int, D_out: int, group: int = 128, zp: bool = False) -> int:
    """Workspace bytes of ``w4a16_gemm``; zp: for asymmetric codes (zeros given)."""
    n = int(_w4a16_zp_ws(N, D_in, D_out, group) if zp else _w4a16_ws(N, D_in, D_out))
    if n == 0:
        raise AwqError(AWQ_EINVAL, "w4a16 workspace size: invalid arguments")
    return n


def quantize_pack_clip(W: torch.Tensor, s: torch.Tensor, clip: torch.Tensor, bits: int = 4, group: int = 128):
    """``awq_quantize_pack_clip``: the final pack with a clip ratio per
    (group, column).  Returns (packed int32 view [D_in/8, D_out], scales fp32
    [D_in/group, D_out])."""
    W = _dev(W, torch.float32, "W")
    s = _dev(s, torch.float32, "s")
    clip = _dev(clip, torch.float32, "clip")
    D_in, D_out = W.shape
    packed = torch.empty(D_in // 8, D_out, dtype=torch.int32, device=W.device)
    sc = torch.empty(D_in // group, D_out, dtype=torch.float32, device=W.device)
    _check(_pack_clip(_ptr(W), _ptr(s), _ptr(clip), D_in, D_out, bits, group, _ptr(packed), _ptr(sc), _stream()))
    return packed, sc


@dataclass
class JointResult:
    L: torch.Tensor             # [n_alpha] fp64 joint loss
    L_layers: torch.Tensor      # [n_layers, n_alpha] fp64
    alpha_star: torch.Tensor    # [1] fp32
    alpha_idx: torch.Tensor     # [1] int32
    status: torch.Tensor


def search_joint(X: torch.Tensor, Ws: Sequence[torch.Tensor], a: torch.Tensor, alpha_grid: Sequence[float],
                 bits: int = 4, group: int = 128, workspace: Optional[Workspace] = None, check_status: bool = True,
                 loss_form: int = LOSS_ERROR) -> JointResult:
    """One scale vector for several linears that share X: ``awq_search_joint``."""
    X = _dev(X, torch.bfloat16, "X")
    Ws = [_dev(W, torch.float32, "W") for W in Ws]
    a = _dev(a, torch.float32, "a")
    N, D_in = X.shape
    nl = len(Ws)
    ptrs = (ctypes.c_void_p * nl)(*[W.data_ptr() for W in Ws])
    douts = (ctypes.c_int64 * nl)(*[W.shape[1] for W in Ws])
    A = len(alpha_grid)
    grid = (ctypes.c_float * A)(*[float(v) for v in alpha_grid])
    dev = X.device
    L = torch.empty(A, dtype=torch.float64, device=dev)
    Ll = torch.empty(nl, A, dtype=torch.float64, device=dev)
    astar = torch.empty(1, dtype=torch.float32, device=dev)
    aidx = torch.empty(1, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    nbytes = int(_joint_ws(N, D_in, douts, nl, A, bits, group, loss_form))
    if nbytes == 0:
        raise AwqError(AWQ_EINVAL, _last_error().decode(errors="replace"))
    ws = (workspace or _default_ws).get(nbytes, dev)
    _check(_joint(_ptr(X), ptrs, douts, nl, _ptr(a), N, D_in, grid, A, bits, group, loss_form, _ptr(L), _ptr(Ll),
                  _ptr(astar), _ptr(aidx), _ptr(ws), ws.numel(), _ptr(status), _stream()))
    res = JointResult(L, Ll, astar, aidx, status)
    if check_status:
        check_device_status(status)
    return res


def check_device_status(status: torch.Tensor) -> None:
    v = int(status.item())
    if v != 0:
        raise AwqError(v & 0xFF, f"device status {v:#x} (code {v & 0xFF}, site {v >> 8})")


def search_batched(layers, alpha_grid: Sequence[float], bits: int = 4, group: int = 128,
                   want_cols: bool = False, workspace: Optional[Workspace] = None, loss_form: int = LOSS_ERROR,
                   check_status: bool = True):
    """Independent searches of several layers in one call: ``awq_search_batched``.
    ``layers`` is a sequence of (X, W, a).  Returns one SearchResult per layer;
    with check_status=False nothing waits for the device (check
    ``result.status`` after synchronising)."""
    A = len(alpha_grid)
    grid = (ctypes.c_float * A)(*[float(v) for v in alpha_grid])
    descs = (AwqLayer * len(layers))()
    results, keep = [], []
    dev = None
    for i, (X, W, a) in enumerate(layers):
        X = _dev(X, torch.bfloat16, "X")
        W = _dev(W, torch.float32, "W")
        a = _dev(a, torch.float32, "a")
        dev = X.device
        N, D_in = X.shape
        D_out = W.shape[1]
        L = torch.empty(A, dtype=torch.float64, device=dev)
        Lc = torch.empty(A, D_out, dtype=torch.float64, device=dev) if want_cols else None
        astar = torch.empty(1, dtype=torch.float32, device=dev)
        aidx = torch.empty(1, dtype=torch.int32, device=dev)
        keep += [X, W, a]
        descs[i] = AwqLayer(_ptr(X), _ptr(W), _ptr(a), N, D_in, D_out, _ptr(L), _ptr(Lc), _ptr(astar), _ptr(aidx))
        results.append(SearchResult(L, astar, aidx, Lc, None))
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    nbytes = int(_batched_ws(descs, len(layers), A, bits, group, loss_form))
    if nbytes == 0:
        raise AwqError(AWQ_EINVAL, _last_error().decode(errors="replace"))
    ws = (workspace or _default_ws).get(nbytes, dev)
    _check(_batched(descs, len(layers), grid, A, bits, group, loss_form, _ptr(ws), ws.numel(), _ptr(status),
                    _stream()))
    if check_status:
        check_device_status(status)
    for r in results:
        r.status = status
    return results


def quantize_pack(W: torch.Tensor, s: torch.Tensor, bits: int = 4, group: int = 128):
    """INT codes (offset binary, 8 per uint32 word) + per-group scales:
    ``awq_quantize_pack``.  Returns (packed int32 view [D_in/8, D_out],
    scales fp32 [D_in/group, D_out])."""
    W = _dev(W, torch.float32, "W")
    s = _dev(s, torch.float32, "s")
    D_in, D_out = W.shape
    packed = torch.empty(D_in // 8, D_out, dtype=torch.int32, device=W.device)
    sc = torch.empty(D_in // group, D_out, dtype=torch.float32, device=W.device)
    _check(_pack(_ptr(W), _ptr(s), D_in, D_out, bits, group, _ptr(packed), _ptr(sc), _stream()))
    return packed, sc


def layer_output(X: torch.Tensor, W: torch.Tensor, workspace: Optional[Workspace] = None) -> torch.Tensor:
    """Y = X bf16(W) on the search's tensor-core GEMM: ``awq_layer_output``."""
    X = _dev(X, torch.bfloat16, "X")
    W = _dev(W, torch.float32, "W")
    N, D_in = X.shape
    D_out = W.shape[1]
    Y = torch.empty(N, D_out, dtype=torch.float32, device=X.device)
    status = torch.zeros(1, dtype=torch.int32, device=X.device)
    nbytes = int(_out_ws(N, D_in, D_out))
    if nbytes == 0:
        raise AwqError(AWQ_EINVAL, _last_error().decode(errors="replace"))
    ws = (workspace or _default_ws).get(nbytes, X.device)
    _check(_out(_ptr(X), _ptr(W), N, D_in, D_out, _ptr(Y), _ptr(ws), ws.numel(), _ptr(status), _stream()))
    check_device_status(status)
    return Y


def selftest_divide(divisor: int):
    """``awq_selftest_divide``: (quotients that differ from the IEEE ones,
    reciprocals more than one ulp off) over every non-negative finite float."""
    out = torch.zeros(2, dtype=torch.int64, device="cuda")
    _check(_selftest_div(int(divisor), _ptr(out), _stream()))
    a, b = out.cpu().tolist()
    return a, b


def selftest_wait_timeout(timeout_ns: int = 1_000_000) -> int:
    """Run the bounded-wait self test; returns the device status word."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(_selftest(_ptr(status), int(timeout_ns), _stream()))
    torch.cuda.synchronize()
    return int(status.item())


def last_error() -> str:
    return _last_error().decode(errors="replace")


def profile_enable(on: bool = True) -> None:
    """Record CUDA events around every kernel the library launches."""
    _check(_prof_enable(1 if on else 0))


def profile_reset() -> None:
    _check(_prof_reset())


def profile_read() -> dict:
    """{stage: (total device ms, launches)} since the last reset."""
    out = {}
    for i, name in enumerate(STAGES):
        ms = ctypes.c_double(0.0)
        n = ctypes.c_int32(0)
        _check(_prof_read(i, ctypes.byref(ms), ctypes.byref(n)))
        out[name] = (ms.value, n.value)
    return out


@dataclass
class LayerResult:
    a: torch.Tensor             # [D_in] activation statistic
    search: SearchResult        # L(alpha), alpha*, status
    s_star: torch.Tensor        # [D_in] scales for alpha*
    packed: torch.Tensor        # [D_in/8, D_out] int32 words of offset-binary codes
    scales: torch.Tensor        # [D_in/group, D_out] fp32 deltas


def quantize_layer(X: torch.Tensor, W: torch.Tensor, alpha_grid: Sequence[float], bits: int = 4,
                   group: int = 128, stat: int = STAT_MEAN, workspace: Optional[Workspace] = None,
                   want_cols: bool = False, loss_form: int = LOSS_ERROR) -> LayerResult:
    """The whole per-layer path on the device, with no host synchronisation:
    statistic -> grid search -> s* = a^alpha* (alpha* read on the device) ->
    quantise + pack.  Check ``result.search.status`` after synchronising."""
    a = act_stats(X, stat)
    res = search(X, W, a, alpha_grid, bits, group, want_cols=want_cols, workspace=workspace, check_status=False,
                 loss_form=loss_form)
    s_star = scales(a, res.alpha_star)
    packed, sc = quantize_pack(W, s_star, bits, group)
    return LayerResult(a, res, s_star, packed, sc)


def quantize_layer_host(X_host: torch.Tensor, W_host: torch.Tensor, alpha_grid: Sequence[float], bits: int = 4,
                        group: int = 128, stat: int = STAT_MEAN, device="cuda",
                        workspace: Optional[Workspace] = None, out: Optional[dict] = None,
                        loss_form: int = LOSS_ERROR) -> dict:
    """The per-layer path from host buffers to host buffers: copies X and W to
    the device (pinned host memory gives asynchronous copies), runs
    :func:`quantize_layer`, copies L, alpha*, the packed codes and the scales
    back, synchronises the stream and checks the device status word."""
    X = X_host.to(device, non_blocking=True)
    W = W_host.to(device, non_blocking=True)
    r = quantize_layer(X, W, alpha_grid, bits, group, stat, workspace, loss_form=loss_form)
    if out is None:
        pin = X_host.is_pinned()
        out = {
            "L": torch.empty(r.search.L.shape, dtype=r.search.L.dtype, pin_memory=pin),
            "alpha_star": torch.empty(1, dtype=torch.float32, pin_memory=pin),
            "status": torch.empty(1, dtype=torch.int32, pin_memory=pin),
            "packed": torch.empty(r.packed.shape, dtype=r.packed.dtype, pin_memory=pin),
            "scales": torch.empty(r.scales.shape, dtype=r.scales.dtype, pin_memory=pin),
        }
    out["L"].copy_(r.search.L, non_blocking=True)
    out["alpha_star"].copy_(r.search.alpha_star, non_blocking=True)
    out["status"].copy_(r.search.status, non_blocking=True)
    out["packed"].copy_(r.packed, non_blocking=True)
    out["scales"].copy_(r.scales, non_blocking=True)
    torch.cuda.current_stream().synchronize()
    v = int(out["status"][0])
    if v != 0:
        raise AwqError(v & 0xFF, f"device status {v:#x}")
    return out


def quantize_block(xs: Sequence[torch.Tensor], layers, alpha_grid: Sequence[float], bits: int = 4,
                   group: int = 128, stat: int = STAT_MEAN, workspace: Optional[Workspace] = None,
                   loss_form: int = LOSS_ERROR):
    """Every linear of a block on the device, with no host synchronisation.

    ``xs`` are the block's distinct layer inputs (bf16 [N, D_in] each);
    ``layers`` is a sequence of (input index, W fp32 [D_in, D_out]).  The
    statistic of each input is computed once, all layers are searched in one
    ``awq_search_batched`` call (each layer independently: compassingai.com
    concept page, "full scale-optimisation flow", final note), and each layer
    gets s* = a^alpha* and its quantise + pack (the statistics of all inputs in
    one ``awq_act_stats_batched`` launch).  Returns one LayerResult per
    layer; check each ``result.search.status`` after synchronising."""
    a = act_stats_batched(xs, stat)
    res = search_batched([(xs[xi], W, a[xi]) for xi, W in layers], alpha_grid, bits, group, workspace=workspace,
                         loss_form=loss_form, check_status=False)
    out = []
    for (xi, W), r in zip(layers, res):
        s_star = scales(a[xi], r.alpha_star)
        packed, sc = quantize_pack(W, s_star, bits, group)
        out.append(LayerResult(a[xi], r, s_star, packed, sc))
    return out


class BlockHostState:
    """Device copies of a block's inputs and pinned host result buffers, kept
    between calls of :func:`quantize_block_host` on blocks of one shape: two
    sets of device buffers (one being computed on, one receiving the next
    block's upload when a call is given ``prefetch``), the copy and result
    streams, and the upload issued ahead, if any."""

    def __init__(self):
        self.bufs = [None, None]       # per set: (device inputs, device weights)
        self.cur = 0
        self.pending = None            # (host key, set, input events, weight events) of an upload ahead
        self.results = None
        self.copy_stream = None
        self.back_stream = None


def _block_order(layers_host):
    """The order the block's layers run in: the smallest W first (the device
    starts early), the second smallest last (the last results to copy back are
    small), the others as given."""
    by_size = sorted(range(len(layers_host)), key=lambda i: (layers_host[i][1].numel(), i))
    if len(by_size) > 2:
        first, last = by_size[0], by_size[1]
        return [first] + [i for i in range(len(layers_host)) if i not in (first, last)] + [last]
    return by_size


def _host_key(xs_host, layers_host):
    return (tuple((x.data_ptr(), tuple(x.shape)) for x in xs_host),
            tuple((xi, w.data_ptr(), tuple(w.shape)) for xi, w in layers_host))


def _block_buffers(st, b, xs_host, layers_host, dev):
    """Device buffers of set b for a block of this shape (reallocated if the shape changed)."""
    shapes = ([tuple(x.shape) for x in xs_host], [tuple(w.shape) for _, w in layers_host])
    cur = st.bufs[b]
    if cur is None or ([tuple(x.shape) for x in cur[0]], [tuple(w.shape) for w in cur[1]]) != shapes:
        st.bufs[b] = ([torch.empty(x.shape, dtype=x.dtype, device=dev) for x in xs_host],
                      [torch.empty(w.shape, dtype=w.dtype, device=dev) for _, w in layers_host])
    return st.bufs[b]


def _block_upload(st, b, order, xs_host, layers_host):
    """On the copy stream, in the layers' run order: each input before the first
    layer that reads it, and each layer's W; returns the ready events."""
    xs_d, ws_d = st.bufs[b]
    x_ready, w_ready = {}, {}
    with torch.cuda.stream(st.copy_stream):
        for i in order:
            xi, wh = layers_host[i]
            if xi not in x_ready:
                xs_d[xi].copy_(xs_host[xi], non_blocking=True)
                x_ready[xi] = torch.cuda.Event()
                x_ready[xi].record(st.copy_stream)
            ws_d[i].copy_(wh, non_blocking=True)
            w_ready[i] = torch.cuda.Event()
            w_ready[i].record(st.copy_stream)
    return x_ready, w_ready


def quantize_block_host(xs_host: Sequence[torch.Tensor], layers_host, alpha_grid: Sequence[float], bits: int = 4,
                        group: int = 128, stat: int = STAT_MEAN, device="cuda",
                        workspace: Optional[Workspace] = None, state: Optional[BlockHostState] = None,
                        loss_form: int = LOSS_ERROR, prefetch=None):
    """A block's linears from host buffers to host results, copies overlapped
    with compute.

    ``xs_host``: the distinct layer inputs (bf16, pinned for asynchronous
    copies); ``layers_host``: (input index, W fp32 on the host) per layer.
    The layers run smallest W first, second smallest last, the others as
    given.  A copy stream uploads, in that order, each input before the first
    layer that reads it and each layer's W; the current stream computes an
    input's statistic before its first layer, then each layer's search
    (``awq_search``), s* and pack as soon as its W has landed; a third stream
    copies each layer's L, alpha*, status, codes and scales back as soon as
    they are done.

    ``prefetch``: the next block's ``(xs_host, layers_host)``.  Their upload is
    queued on the copy stream behind this block's, into the state's other set
    of device buffers, so that it runs while this block computes; the next
    call with the same host buffers (and ``state``) finds them uploaded and
    starts at once.  Those host buffers must keep their contents until that
    call.  Synchronises the compute and result streams (not an upload ahead),
    checks every status word and returns a list of dicts of host tensors in
    the layers' given order (reused across calls through ``state``: read them
    before the next call)."""
    dev = torch.device(device)
    st = state if state is not None else BlockHostState()
    compute = torch.cuda.current_stream(dev)
    if st.copy_stream is None:
        st.copy_stream = torch.cuda.Stream(dev)
        st.back_stream = torch.cuda.Stream(dev)
    order = _block_order(layers_host)
    key = _host_key(xs_host, layers_host)
    if st.pending is not None and st.pending[0] == key:
        _, b, x_ready, w_ready = st.pending    # uploaded ahead by the previous call
    else:
        b = st.cur
        _block_buffers(st, b, xs_host, layers_host, dev)
        # the previous call's device work on these buffers has finished (it synchronised)
        st.copy_stream.wait_stream(compute)
        x_ready, w_ready = _block_upload(st, b, order, xs_host, layers_host)
    st.pending = None
    st.cur = b
    xs_d, ws_d = st.bufs[b]
    pin = all(x.is_pinned() for x in xs_host)
    if st.results is None or len(st.results) != len(layers_host):
        st.results = []
        for (xi, _), wd in zip(layers_host, ws_d):
            D_in, D_out = wd.shape
            st.results.append({
                "L": torch.empty(len(alpha_grid), dtype=torch.float64, pin_memory=pin),
                "alpha_star": torch.empty(1, dtype=torch.float32, pin_memory=pin),
                "status": torch.empty(1, dtype=torch.int32, pin_memory=pin),
                "packed": torch.empty(D_in // 8, D_out, dtype=torch.int32, pin_memory=pin),
                "scales": torch.empty(D_in // group, D_out, dtype=torch.float32, pin_memory=pin),
            })
    a = {}
    for i in order:
        xi, _ = layers_host[i]
        wd = ws_d[i]
        if xi not in a:                            # the input's statistic, before its first layer
            compute.wait_event(x_ready[xi])
            a[xi] = act_stats(xs_d[xi], stat)
        compute.wait_event(w_ready[i])
        r = search(xs_d[xi], wd, a[xi], alpha_grid, bits, group, workspace=workspace, check_status=False,
                   loss_form=loss_form)
        s_star = scales(a[xi], r.alpha_star)
        packed, sc = quantize_pack(wd, s_star, bits, group)
        done = torch.cuda.Event()
        done.record(compute)
        st.back_stream.wait_event(done)
        host = st.results[i]
        with torch.cuda.stream(st.back_stream):
            for name, t in (("L", r.L), ("alpha_star", r.alpha_star), ("status", r.status), ("packed", packed),
                            ("scales", sc)):
                t.record_stream(st.back_stream)
                host[name].copy_(t, non_blocking=True)
    if prefetch is not None:
        nxs, nlayers = prefetch
        nb = 1 - b
        # set nb was last read by an earlier call, whose device work has finished
        _block_buffers(st, nb, nxs, nlayers, dev)
        nx_ready, nw_ready = _block_upload(st, nb, _block_order(nlayers), nxs, nlayers)
        st.pending = (_host_key(nxs, nlayers), nb, nx_ready, nw_ready)
    st.back_stream.synchronize()
    compute.synchronize()
    for host in st.results:
        v = int(host["status"][0])
        if v != 0:
            raise AwqError(v & 0xFF, f"device status {v:#x}")
    return st.results
