"""Seeded synthetic inputs for the ButterflyMoE expert layer.

This module only draws random numbers. It holds none of the layer's
arithmetic (no rotation, routing, packing or contraction), so both the CUDA
path and the fp64 oracle can take their inputs from it without sharing any
of the method.

Five workloads are defined, each named by its shape:

=============  =====  ===  =  =====  =====  ============================
name           d      N    k  T      x      W_base / alpha
=============  =====  ===  =  =====  =====  ============================
tiny           64     8    2  128    f32    P(0)=1/3, alpha=1
headline       512    64   2  4096   bf16   P(0)=0.4, alpha=mean|G|
many_experts   512    256  2  16384  bf16   P(0)=0.4, alpha=mean|G|
llm_width      4096   64   2  8192   bf16   P(0)=1/3, alpha=mean|G|
vit            1024   64   1  12608  bf16   P(0)=1/3, alpha=mean|G|
=============  =====  ===  =  =====  =====  ============================

Distributions (the pages train on WikiText and CIFAR-100, which are not
available; these draws stand in for their activations):

* x ~ N(0, 1), with a fixed set of "outlier" channels scaled up (the
  activation outliers the ButterflyMoE and ButterflyViT pages describe in
  their methodology sections), then rounded to bf16 (round to nearest even)
  except for the fp32 tiny case.
* W_base iid ternary in {-1, 0, +1}.
* alpha = mean |G| for G ~ N(0, 1/d) of shape d x d (1 for tiny).
* theta, phi ~ U[-pi, pi), fp32, shape [N][log2 d][d/2]  (the pages
  initialise the butterfly angles randomly and independently per expert).
* router logits ~ N(0, sigma^2), fp32; sigma^2 = 2 for many_experts so that
  expert loads are skewed.

Draw order with ``numpy.random.Generator(PCG64(seed))``: x, outlier
channels, W_base, alpha draw, theta, phi, logits.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    d: int
    N: int
    k: int
    T: int
    dtype: str            # "f32" or "bf16": dtype of x and y
    seed: int
    p_zero: float         # P(W_base == 0); the rest split evenly over +-1
    outlier_frac: float   # fraction of channels scaled
    outlier_scale: float
    logit_std: float
    unit_alpha: bool      # alpha = 1 instead of mean|G|

    @property
    def L(self) -> int:
        return int(round(math.log2(self.d)))

    @property
    def R(self) -> int:
        return self.T * self.k


WORKLOADS = {
    "tiny": Workload("tiny", 64, 8, 2, 128, "f32", 0, 1.0 / 3.0, 0.0, 1.0, 1.0, True),
    "headline": Workload("headline", 512, 64, 2, 4096, "bf16", 1, 0.4, 0.01, 20.0, 1.0, False),
    "many_experts": Workload("many_experts", 512, 256, 2, 16384, "bf16", 2, 0.4, 0.01, 20.0,
                             math.sqrt(2.0), False),
    "llm_width": Workload("llm_width", 4096, 64, 2, 8192, "bf16", 3, 1.0 / 3.0, 0.005, 50.0, 1.0,
                          False),
    "vit": Workload("vit", 1024, 64, 1, 64 * 197, "bf16", 4, 1.0 / 3.0, 0.01, 20.0, 1.0, False),
}


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32
    holding exactly representable bf16 values.  NaN is kept as NaN."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    out = (r & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    nan = np.isnan(a)
    if nan.any():
        out = out.copy()
        out[nan] = np.nan
    return out


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of fp32 values that are already bf16-representable."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


@dataclasses.dataclass
class Inputs:
    wl: Workload
    x: np.ndarray          # [T][d] fp32 (bf16-representable unless dtype f32)
    w_base: np.ndarray     # [d][d] int8 in {-1,0,1}
    alpha: float           # fp32 value
    theta: np.ndarray      # [N][L][d/2] fp32
    phi: np.ndarray        # [N][L][d/2] fp32
    logits: np.ndarray     # [T][N] fp32
    outlier_channels: np.ndarray


def make_inputs(wl: Workload | str, T: int | None = None, seed: int | None = None) -> Inputs:
    """Draw the inputs of a workload.  ``T`` overrides the token count (the
    first ``T`` tokens are NOT a prefix of the full draw; every array is drawn
    at the requested size) and ``seed`` overrides the seed."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    if T is not None or seed is not None:
        wl = dataclasses.replace(wl, T=wl.T if T is None else T, seed=wl.seed if seed is None else seed)
    d, N, L = wl.d, wl.N, wl.L
    rng = np.random.Generator(np.random.PCG64(wl.seed))
    x = rng.standard_normal((wl.T, d), dtype=np.float32)
    n_out = int(round(wl.outlier_frac * d))
    ch = np.sort(rng.choice(d, n_out, replace=False)) if n_out > 0 else np.zeros(0, np.int64)
    if n_out > 0:
        x[:, ch] *= np.float32(wl.outlier_scale)
    if wl.dtype == "bf16":
        x = round_to_bf16(x)
    p_pm = (1.0 - wl.p_zero) / 2.0
    w = rng.choice(np.array([-1, 0, 1], dtype=np.int8), size=(d, d), p=[p_pm, wl.p_zero, p_pm])
    w = np.ascontiguousarray(w, dtype=np.int8)
    if wl.unit_alpha:
        alpha = 1.0
    else:
        g = rng.standard_normal((d, d)) * (1.0 / math.sqrt(d))
        alpha = float(np.float32(np.mean(np.abs(g))))
    theta = rng.uniform(-math.pi, math.pi, size=(N, L, d // 2)).astype(np.float32)
    phi = rng.uniform(-math.pi, math.pi, size=(N, L, d // 2)).astype(np.float32)
    logits = (rng.standard_normal((wl.T, N)) * wl.logit_std).astype(np.float32)
    return Inputs(wl, x, w, alpha, theta, phi, logits, ch)


def random_ternary(rng: np.random.Generator, d: int, p_zero: float = 1.0 / 3.0) -> np.ndarray:
    p_pm = (1.0 - p_zero) / 2.0
    return np.ascontiguousarray(
        rng.choice(np.array([-1, 0, 1], dtype=np.int8), size=(d, d), p=[p_pm, p_zero, p_pm]))


def random_angles(rng: np.random.Generator, N: int, d: int) -> np.ndarray:
    L = int(round(math.log2(d)))
    return rng.uniform(-math.pi, math.pi, size=(N, L, d // 2)).astype(np.float32)
