"""Seeded synthetic inputs for the fused add + RMSNorm + dynamic-quant operator.

This module draws random numbers and rounds them to the 16-bit input dtype;
it holds none of the operator's arithmetic.  The CUDA path's tests, the
oracle's tests and the benchmark all take their inputs from here, so both
sides of every comparison read the same bit patterns.

Every 16-bit tensor is returned as its raw bit pattern (``numpy.uint16``),
produced by drawing binary32 values with ``numpy.random.default_rng(seed)``
(PCG64) and rounding them to the dtype with torch's round-to-nearest-even
casts.  Parameters (gamma, beta, smooth scales) are drawn after the two
activations, in that order, so changing one optional tensor does not shift
the others.

The named workloads reproduce the shapes and value distributions of the five
benchmark configurations (N(mu, sigma) takes sigma as the standard deviation).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple

import numpy as np
import torch

_TORCH_DT = {"bf16": torch.bfloat16, "fp16": torch.float16}


def to_bits(values: np.ndarray, dtype: str) -> np.ndarray:
    """binary32 values -> uint16 bit patterns of bf16/fp16 (torch RNE cast)."""
    t = torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32))
    return t.to(_TORCH_DT[dtype]).view(torch.int16).numpy().view(np.uint16)


def bits_to_float(bits: np.ndarray, dtype: str) -> np.ndarray:
    """uint16 bit patterns -> binary32 values (exact widening, via torch)."""
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(_TORCH_DT[dtype]).float().numpy()


@dataclass
class Workload:
    name: str
    rows: int
    n: int
    dtype: str                      # "bf16" | "fp16": x1, x2, params, xOut
    qdtype: str                     # "int8" | "int4": y1, y2
    eps: float
    mask: Optional[Tuple[bool, bool]]  # None = outputMask absent
    x1: np.ndarray                  # [rows, n] uint16 bits
    x2: np.ndarray                  # [rows, n] uint16 bits
    gamma: np.ndarray               # [n] uint16 bits
    beta: Optional[np.ndarray] = None
    smooth1: Optional[np.ndarray] = None
    smooth2: Optional[np.ndarray] = None
    seed: int = 0
    recipe: dict = field(default_factory=dict)


def _normal(rng, shape, sigma=1.0):
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(sigma)).astype(np.float32)


def _uniform(rng, shape, lo, hi):
    return rng.uniform(lo, hi, shape).astype(np.float32)


def random_case(rows: int, n: int, *, dtype="bf16", qdtype="int8", seed=0, eps=1e-6,
                mask=None, beta=False, smooth1=False, smooth2=False, x_sigma=(1.0, 1.0),
                gamma_range=(0.5, 1.5), beta_sigma=0.1, s1_range=(0.5, 2.0),
                s2_range=(0.25, 4.0), outlier_frac=0.0, outlier_mult=50.0,
                student_t=None, name=None) -> Workload:
    """A seeded workload of the given shape and distributions.

    x1 ~ N(0, x_sigma[0]), x2 ~ N(0, x_sigma[1]) (or, with student_t=(df, k),
    both k * Student-t(df)); gamma ~ U(gamma_range); beta ~ N(0, beta_sigma);
    smooth1 ~ U(s1_range); smooth2 ~ U(s2_range).  beta=0.0 passes an all-zero
    beta tensor.  outlier_frac > 0 picks round(outlier_frac * n) channels
    without replacement and multiplies x1 and x2 there by outlier_mult before
    rounding.
    """
    rng = np.random.default_rng(seed)
    shape = (rows, n)
    if student_t is not None:
        df, k = student_t
        a = (rng.standard_t(df, shape) * k).astype(np.float32)
        b = (rng.standard_t(df, shape) * k).astype(np.float32)
    else:
        a = _normal(rng, shape, x_sigma[0])
        b = _normal(rng, shape, x_sigma[1])
    gamma = _uniform(rng, (n,), *gamma_range)
    # beta: False/None -> absent, True -> N(0, beta_sigma), a float 0.0 -> all zeros
    beta_zero = beta is not True and beta is not False and beta is not None
    beta_v = None
    if beta_zero:
        beta_v = np.zeros((n,), np.float32)
    elif beta is True:
        beta_v = _normal(rng, (n,), beta_sigma)
    s1 = _uniform(rng, (n,), *s1_range) if smooth1 else None
    s2 = _uniform(rng, (n,), *s2_range) if smooth2 else None
    if outlier_frac > 0.0:
        k = int(round(outlier_frac * n))
        cols = rng.choice(n, size=k, replace=False)
        a[:, cols] *= np.float32(outlier_mult)
        b[:, cols] *= np.float32(outlier_mult)
    recipe = dict(seed=seed, x_sigma=x_sigma, student_t=student_t, gamma=gamma_range,
                  beta=("zeros" if beta_zero else (f"N(0,{beta_sigma})" if beta is True else None)),
                  smooth1=s1_range if smooth1 else None, smooth2=s2_range if smooth2 else None,
                  outliers=(outlier_frac, outlier_mult) if outlier_frac else None)
    return Workload(
        name=name or f"random_{rows}x{n}_{dtype}_{qdtype}", rows=rows, n=n, dtype=dtype,
        qdtype=qdtype, eps=eps, mask=mask, x1=to_bits(a, dtype), x2=to_bits(b, dtype),
        gamma=to_bits(gamma, dtype), beta=None if beta_v is None else to_bits(beta_v, dtype),
        smooth1=None if s1 is None else to_bits(s1, dtype),
        smooth2=None if s2 is None else to_bits(s2, dtype), seed=seed, recipe=recipe)


# --- the five benchmark configurations --------------------------------------

def config1() -> Workload:
    """64 x 1024 bf16, x1, x2 ~ N(0,1), gamma ~ U(0.5,1.5), no beta, no smooth,
    eps 1e-6, mask absent: one INT8 output + scale + xOut.  Seed 0."""
    return random_case(64, 1024, seed=0, name="add_rmsnorm_dynquant_64x1024_bf16_int8")


def config2() -> Workload:
    """8192 x 4096 bf16, x1 ~ N(0,1), x2 ~ N(0,0.5), gamma ~ U(0.5,1.5),
    beta ~ N(0,0.1), smooth1 ~ U(0.5,2), outputMask [True, False], INT8.  Seed 1."""
    return random_case(8192, 4096, seed=1, x_sigma=(1.0, 0.5), beta=True, smooth1=True,
                       mask=(True, False), name="add_rmsnorm_dynquant_8192x4096_bf16_int8")


def config3() -> Workload:
    """4096 x 7168 bf16, dual INT8 output (mask [True, True]), smooth1 ~ U(0.5,2),
    smooth2 ~ U(0.25,4), gamma ~ U(0.5,1.5), no beta, 1% of channels (72)
    scaled x50 in x1 and x2.  Seed 2."""
    return random_case(4096, 7168, seed=2, smooth1=True, smooth2=True, mask=(True, True),
                       outlier_frac=0.01, name="add_rmsnorm_dynquant_4096x7168_bf16_dual_int8")


def config4() -> Workload:
    """16384 x 5120 fp16, x1, x2 = 0.5 * Student-t(3), gamma ~ U(0.8,1.2),
    beta = 0 passed as a tensor, no smooth, mask absent, packed INT4.  Seed 3."""
    return random_case(16384, 5120, dtype="fp16", qdtype="int4", seed=3, student_t=(3, 0.5),
                       gamma_range=(0.8, 1.2), beta=0.0,
                       name="add_rmsnorm_dynquant_16384x5120_fp16_int4")


def config5(rows: int) -> Workload:
    """rows x 16384 bf16 (rows in {1, 8, 128, 2048}), x1, x2 ~ N(0,1),
    gamma ~ U(0.5,1.5), beta ~ N(0,0.1), smooth1 ~ U(0.5,2), mask absent,
    one INT8 output.  Seed 4 + rows."""
    return random_case(rows, 16384, seed=4 + rows, beta=True, smooth1=True,
                       name=f"add_rmsnorm_dynquant_{rows}x16384_bf16_int8")


CONFIGS = {
    "c1": config1,
    "c2": config2,
    "c3": config3,
    "c4": config4,
    "c5a": lambda: config5(1),
    "c5b": lambda: config5(8),
    "c5c": lambda: config5(128),
    "c5d": lambda: config5(2048),
}
