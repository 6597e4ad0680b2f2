"""Seeded synthetic inputs for the AWQ per-layer scale search.

The AWQ pages calibrate on a few hundred samples of pre-training text and
evaluate LLaMA / OPT layers (mudrobot.github.io AWQ notes, "Experimental
setup": Pile calibration set, group size 128; compassingai.com AWQ concept
page, "AWQ pipeline" diagram: 128-512 calibration samples).  Neither the data
nor the weights exist here, so these generators stand in for them with the
same shapes, dtypes and the one structural feature the method depends on:
about 1% of input channels whose activations are far larger than the rest
(compassingai.com concept page, "core mechanism": ~1% salient channels).

This module holds no part of the method's arithmetic.  It only draws random
numbers, and both the CUDA path and the CPU oracle consume the bytes it
produces.  Everything is drawn on the CPU from ``torch.Generator`` so the bytes
are identical on every machine with the same torch version.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch

__all__ = [
    "LayerSpec", "Workload", "WORKLOADS", "alpha_grid", "clip_grid", "make_x", "make_w",
    "layer_inputs", "workload",
]


def alpha_grid(n_intervals: int) -> torch.Tensor:
    """The alpha candidates k / n_intervals, k = 0..n_intervals, as float32.

    Each point is computed as an exact integer ratio in float64 and then
    rounded once to float32 (20 intervals gives the 21-point grid
    {0, 0.05, ..., 1} of the compassingai.com concept page, "scale search",
    step 3; 40 intervals gives the 41-point grid used by the bit-width sweep).
    """
    k = torch.arange(n_intervals + 1, dtype=torch.float64)
    return (k / n_intervals).to(torch.float32)


def clip_grid(n_intervals: int = 20, lo: float = 0.5) -> torch.Tensor:
    """Weight-clipping ratios from 1 (no clipping, index 0) down to `lo` in
    n_intervals equal steps: c_i = 1 - (1 - lo) i / n_intervals, formed in fp64
    and rounded once to fp32."""
    i = torch.arange(n_intervals + 1, dtype=torch.float64)
    return (1.0 - (1.0 - lo) * i / n_intervals).to(torch.float32)


@dataclass(frozen=True)
class XSpec:
    """How the calibration activations of one layer input are drawn."""
    kind: str                 # "normal" | "silu_gate" | "student_t3"
    n_outlier: int            # number of outlier input channels
    lo: float                 # outlier multiplier ~ U(lo, hi), one per channel
    hi: float
    seed: int


@dataclass(frozen=True)
class LayerSpec:
    """One linear layer Y = X.W with X: N x D_in (bf16), W: D_in x D_out (fp32)."""
    name: str
    N: int
    D_in: int
    D_out: int
    x: XSpec
    w_std: float
    w_seed: int


@dataclass(frozen=True)
class Workload:
    name: str
    layers: Tuple[LayerSpec, ...]
    quant: Tuple[Tuple[int, int], ...]          # (bits, group) settings searched
    n_intervals: int                             # alpha grid = k / n_intervals
    x_variants: Tuple[XSpec, ...] = field(default_factory=tuple)

    @property
    def n_alpha(self) -> int:
        return self.n_intervals + 1


def _silu(z: torch.Tensor) -> torch.Tensor:
    return z * torch.sigmoid(z)


def make_x(N: int, D: int, spec: XSpec) -> torch.Tensor:
    """Draw an N x D bf16 activation matrix on the CPU.

    kind "normal":      X ~ N(0, 1)
    kind "silu_gate":   X = SiLU(z1) * z2, z1, z2 ~ N(0, 1) i.i.d. (the input
                        of an MLP down projection)
    kind "student_t3":  X ~ Student-t with 3 degrees of freedom, drawn as
                        z / sqrt(chi2_3 / 3) with chi2_3 a sum of three squared
                        standard normals (heavy-tailed activations)
    Then ``n_outlier`` channels, chosen without replacement from the same
    generator, have their whole column multiplied by one factor U(lo, hi) each,
    and the result is rounded to bf16 once.
    """
    g = torch.Generator().manual_seed(spec.seed)
    if spec.kind == "normal":
        x = torch.randn(N, D, generator=g, dtype=torch.float32)
    elif spec.kind == "silu_gate":
        z1 = torch.randn(N, D, generator=g, dtype=torch.float32)
        z2 = torch.randn(N, D, generator=g, dtype=torch.float32)
        x = _silu(z1).mul_(z2)
        del z1, z2
    elif spec.kind == "student_t3":
        x = torch.randn(N, D, generator=g, dtype=torch.float32)
        chi2 = torch.zeros(N, D, dtype=torch.float32)
        for _ in range(3):
            chi2.add_(torch.randn(N, D, generator=g, dtype=torch.float32).square_())
        x.div_(chi2.div_(3.0).sqrt_())
        del chi2
    else:
        raise ValueError(f"unknown activation kind {spec.kind!r}")
    if spec.n_outlier > 0:
        idx = torch.randperm(D, generator=g)[: spec.n_outlier]
        fac = spec.lo + (spec.hi - spec.lo) * torch.rand(spec.n_outlier, generator=g, dtype=torch.float32)
        x[:, idx] *= fac
    return x.to(torch.bfloat16)


def make_w(D_in: int, D_out: int, std: float, seed: int) -> torch.Tensor:
    """Draw a D_in x D_out fp32 weight matrix ~ N(0, std^2) on the CPU."""
    g = torch.Generator().manual_seed(seed)
    return torch.randn(D_in, D_out, generator=g, dtype=torch.float32).mul_(std)


def layer_inputs(layer: LayerSpec) -> Tuple[torch.Tensor, torch.Tensor]:
    """(X bf16 [N, D_in], W fp32 [D_in, D_out]) for one layer, on the CPU."""
    return make_x(layer.N, layer.D_in, layer.x), make_w(layer.D_in, layer.D_out, layer.w_std, layer.w_seed)


def _one_pct(D: int) -> int:
    return max(1, round(0.01 * D))


def _build() -> dict:
    w = {}
    # Single linear layer, 512 x 512, 256 calibration tokens.
    x = XSpec("normal", 5, 20.0, 50.0, seed=0)
    w["linear_512_n256"] = Workload(
        "linear_512_n256",
        (LayerSpec("linear", 256, 512, 512, x, 0.02, 100),),
        ((4, 128),), 20)
    # LLaMA-7B-shaped attention projection, 4096 x 4096, 4096 tokens (8 x 512).
    x = XSpec("normal", 41, 20.0, 100.0, seed=0)
    w["llama7b_attn_proj"] = Workload(
        "llama7b_attn_proj",
        (LayerSpec("attn_proj", 4096, 4096, 4096, x, 0.02, 100),),
        ((4, 128),), 20)
    # LLaMA-7B-shaped MLP down projection, 11008 -> 4096.
    x = XSpec("silu_gate", _one_pct(11008), 10.0, 60.0, seed=0)
    w["llama7b_mlp_down"] = Workload(
        "llama7b_mlp_down",
        (LayerSpec("down_proj", 4096, 11008, 4096, x, 0.015, 100),),
        ((4, 128),), 20)
    # 70B-shaped decoder block: all seven linears.  q/k/v share one input,
    # gate/up share one input; o and down have their own.
    h, kv, ff, N = 8192, 1024, 28672, 4096
    xs = [XSpec("student_t3", _one_pct(d), 20.0, 100.0, seed=s)
          for s, d in enumerate((h, h, h, ff))]
    layers = (
        LayerSpec("q_proj", N, h, h, xs[0], 0.01, 100),
        LayerSpec("k_proj", N, h, kv, xs[0], 0.01, 101),
        LayerSpec("v_proj", N, h, kv, xs[0], 0.01, 102),
        LayerSpec("o_proj", N, h, h, xs[1], 0.01, 103),
        LayerSpec("gate_proj", N, h, ff, xs[2], 0.01, 104),
        LayerSpec("up_proj", N, h, ff, xs[2], 0.01, 105),
        LayerSpec("down_proj", N, ff, h, xs[3], 0.01, 106),
    )
    w["llama70b_block"] = Workload("llama70b_block", layers, ((4, 128),), 20)
    # Bit-width / group sweep on a 4096 -> 11008 layer, 16384 tokens, two
    # outlier densities (0.1% and 1% of channels), 41-point grid.
    v01 = XSpec("student_t3", 4, 20.0, 100.0, seed=0)
    v1 = XSpec("student_t3", 41, 20.0, 100.0, seed=1)
    w["sweep_4096x11008_n16k"] = Workload(
        "sweep_4096x11008_n16k",
        (LayerSpec("up_proj_0.1pct", 16384, 4096, 11008, v01, 0.02, 100),
         LayerSpec("up_proj_1pct", 16384, 4096, 11008, v1, 0.02, 100)),
        ((4, 128), (4, 64), (3, 128)), 40)
    return w


WORKLOADS = _build()


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def small_layer(N: int, D_in: int, D_out: int, seed: int = 0, n_outlier: Optional[int] = None,
                kind: str = "normal", lo: float = 20.0, hi: float = 50.0,
                w_std: float = 0.02) -> LayerSpec:
    """A small layer with the same recipe, for parity tests that span several
    tiles plus a ragged tail."""
    if n_outlier is None:
        n_outlier = max(1, D_in // 100)
    return LayerSpec(f"small_{N}x{D_in}x{D_out}_s{seed}", N, D_in, D_out,
                     XSpec(kind, n_outlier, lo, hi, seed), w_std, seed + 100)
