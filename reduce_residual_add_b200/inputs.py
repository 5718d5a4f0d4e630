"""Seeded synthetic workloads for the fused reduce + residual-add + RMSNorm
(+FP8) epilogue.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests.  It holds the workloads' shapes, distributions and seeds and draws the
random inputs -- and nothing of the method's arithmetic.  All draws use a
CPU ``torch.Generator`` so that every run, on any machine, sees the same bits.

Draw recipe for one workload (in this order, one generator seeded with
``seed``):

1. outlier rows, when ``outlier_frac > 0``: ``randperm(T)[:ceil(frac*T)]``;
2. for r in 0..W-1: ``randn(T, H) * partial_sigma`` (fp32), the outlier rows
   multiplied by ``outlier_mult``, then cast (round to nearest even) to the
   model dtype;
3. the residual: ``randn(T, H) * residual_sigma``, cast;
4. gamma: ``rand(H) * (hi - lo) + lo`` (uniform) or ``randn(H) * sigma +
   mean`` (normal), cast.

``N(0, s)`` in a workload's description names the standard deviation s.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional, Tuple

import numpy as np
import torch

PATTERN_AR_RESIDUAL_RMSNORM = 0
PATTERN_FP8_STATIC = 1
PATTERN_FP8_TOKEN = 2
PATTERN_FP8_TENSOR = 3
PATTERN_FP8_GROUP = 4

_TORCH_DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16}


@dataclass(frozen=True)
class Workload:
    """One synthetic problem: W partials of shape (T, H) plus residual/gamma."""

    name: str
    W: int
    T: int
    H: int
    dtype: str = "bf16"
    partial_sigma: float = 1.0
    residual_sigma: float = 1.0
    gamma_dist: str = "uniform"          # "uniform" (lo, hi) or "normal" (mean, sigma)
    gamma_a: float = 0.5
    gamma_b: float = 1.5
    eps: float = 1e-6
    weight_bias: float = 0.0
    pattern: int = PATTERN_AR_RESIDUAL_RMSNORM
    static_scale: Optional[float] = None
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0
    seed: int = 0
    batch_shape: Optional[Tuple[int, ...]] = None   # e.g. (4, 256) for a 3-D view
    has_residual: bool = True
    group_size: int = 0                               # per-group FP8: elements per group

    @property
    def torch_dtype(self) -> torch.dtype:
        return _TORCH_DTYPES[self.dtype]

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The synthetic configurations the library is checked and measured on.
WORKLOADS = {
    # small: W=2, T=8, H=64, bf16; partials/residual N(0,1); gamma U(0.5,1.5)
    "c1_small": Workload("c1_small", W=2, T=8, H=64, seed=0),
    # decode regime: W=8, H=4096, bf16; partials N(0,0.5); residual N(0,1)
    **{
        "c2_decode_T%d" % T: Workload(
            "c2_decode_T%d" % T, W=8, T=T, H=4096, partial_sigma=0.5,
            seed=1000 + T)
        for T in (1, 8, 32, 80)
    },
    # 3-D [batch=4, tokens=256, hidden=2048] viewed as (1024, 2048); W=2
    "c3_3d": Workload("c3_3d", W=2, T=1024, H=2048, gamma_a=0.8, gamma_b=1.2,
                      seed=2, batch_shape=(4, 256)),
    # prefill: W=4, T=8192, H=8192, bf16, 1% outlier rows x50, residual
    # N(0,2), eps=1e-5, static per-tensor FP8 with scale 0.05
    "c4_prefill_fp8_static": Workload(
        "c4_prefill_fp8_static", W=4, T=8192, H=8192, residual_sigma=2.0,
        eps=1e-5, pattern=PATTERN_FP8_STATIC, static_scale=0.05,
        outlier_frac=0.01, outlier_mult=50.0, seed=3),
    # the prefill workload with dynamic per-tensor FP8 (one scale per call)
    "c4_prefill_fp8_tensor": Workload(
        "c4_prefill_fp8_tensor", W=4, T=8192, H=8192, residual_sigma=2.0,
        eps=1e-5, pattern=PATTERN_FP8_TENSOR, outlier_frac=0.01, outlier_mult=50.0, seed=3),
    # the prefill workload with per-group FP8, groups of 128 elements
    "c4_prefill_fp8_group128": Workload(
        "c4_prefill_fp8_group128", W=4, T=8192, H=8192, residual_sigma=2.0,
        eps=1e-5, pattern=PATTERN_FP8_GROUP, outlier_frac=0.01, outlier_mult=50.0, seed=3,
        group_size=128),
    # W=8, T=4096, H=7168, Gemma-style weight_bias=1.0 with gamma N(0,0.1),
    # dynamic per-token FP8; in bf16 and in fp16
    **{
        "c5_gemma_fp8_token_%s" % dt: Workload(
            "c5_gemma_fp8_token_%s" % dt, W=8, T=4096, H=7168, dtype=dt,
            gamma_dist="normal", gamma_a=0.0, gamma_b=0.1, weight_bias=1.0,
            pattern=PATTERN_FP8_TOKEN, seed=4)
        for dt in ("bf16", "fp16")
    },
}


def outlier_count(wl: Workload) -> int:
    return int(math.ceil(wl.outlier_frac * wl.T)) if wl.outlier_frac > 0 else 0


def make_inputs(wl: Workload, rows: Optional[int] = None) -> dict:
    """Draw the workload's inputs on the CPU.

    Returns ``{"partials": [W x (T, H)], "residual": (T, H) or None,
    "gamma": (H,), "scale_in": float or None, "outlier_rows": LongTensor}``
    as CPU tensors of the model dtype.  With ``rows`` only the first ``rows``
    rows are kept (the draws are the same as for the full workload).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed)
    T, H = wl.T, wl.H
    n_out = outlier_count(wl)
    outliers = torch.randperm(T, generator=g)[:n_out] if n_out else torch.empty(0, dtype=torch.long)
    partials = []
    for _ in range(wl.W):
        x = torch.randn(T, H, generator=g, dtype=torch.float32)
        x.mul_(wl.partial_sigma)
        if n_out:
            x[outliers] *= wl.outlier_mult
        partials.append(x.to(wl.torch_dtype))
        del x
    residual = None
    if wl.has_residual:
        r = torch.randn(T, H, generator=g, dtype=torch.float32)
        r.mul_(wl.residual_sigma)
        residual = r.to(wl.torch_dtype)
        del r
    if wl.gamma_dist == "uniform":
        gam = torch.rand(H, generator=g, dtype=torch.float32) * (wl.gamma_b - wl.gamma_a) + wl.gamma_a
    elif wl.gamma_dist == "normal":
        gam = torch.randn(H, generator=g, dtype=torch.float32) * wl.gamma_b + wl.gamma_a
    else:
        raise ValueError(wl.gamma_dist)
    gamma = gam.to(wl.torch_dtype)
    if rows is not None:
        partials = [p[:rows].clone() for p in partials]
        residual = None if residual is None else residual[:rows].clone()
    return {"partials": partials, "residual": residual, "gamma": gamma,
            "scale_in": wl.static_scale, "outlier_rows": outliers}


def random_inputs(W: int, T: int, H: int, dtype: str = "bf16", seed: int = 0,
                  partial_sigma: float = 1.0, residual_sigma: float = 1.0,
                  has_residual: bool = True) -> dict:
    """Inputs of an arbitrary shape (edge cases), same recipe as ``make_inputs``."""
    wl = Workload("adhoc", W=W, T=T, H=H, dtype=dtype, seed=seed,
                  partial_sigma=partial_sigma, residual_sigma=residual_sigma,
                  has_residual=has_residual)
    return make_inputs(wl)


def as_u16(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a bf16/fp16 CPU tensor, as a numpy uint16 array."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_u16(a: np.ndarray, dtype: str) -> torch.Tensor:
    """Inverse of ``as_u16``."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(_TORCH_DTYPES[dtype])
