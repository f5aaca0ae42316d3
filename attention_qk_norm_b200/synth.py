"""Seeded synthetic inputs for QK-Norm workloads.

This module holds no QK-Norm arithmetic: it only draws random activations
and weights with the shapes and value distributions of the workloads, and
stores them in bf16 or fp16 (round-to-nearest-even from float32), FP8 E4M3
(round-to-nearest-even; magnitudes beyond its largest finite value, 448,
become 448, which also turns the stress recipe's 1e4 outliers into 448), or
fp32.  The
oracle (``oracle/``) and the CUDA path both consume what it produces; it
imports neither of them.

Layout of every activation buffer: the fused QKV row-major buffer
``[T, row_stride]`` of the "combined QKV projection" lesson (GQA section):
columns ``[0, Hq*D)`` are Q, ``[Hq*D, (Hq+Hk)*D)`` are K, the next ``Hk*D``
are V, and the rest up to ``row_stride`` is padding.  All of it is filled
with random values, so that a write outside Q/K shows up.

Recipe (one ``numpy.random.default_rng(seed)`` stream, drawn in this order):

1. ``x ~ N(0, 1)`` float32 over the whole ``[T, row_stride]`` buffer;
2. optional per-token scale: ``lognormal(0, 1)`` (fused GQA workload), or
   ``clip(exp(N(0, 2.3)), 1e-3, 1e3)`` (stress workload, spanning 1e-3..1e3
   at about three sigma);
3. optional zero rows: ``ceil(1%)`` of the tokens get their whole Q+K span
   set to 0 (every head of the row takes the epsilon branch);
4. optional outlier rows: another ``ceil(1%)`` of the tokens get one random
   Q+K column set to +-1e4;
5. ``gamma_q, gamma_k = 1 + 0.1 * N(0, 1)`` float32, of length D (per-head)
   or Hq*D / Hk*D (layerwise).

``make_case_torch`` follows the same recipe with a ``torch.Generator`` on
the target device for workloads too large to draw on the host quickly; its
random stream differs from numpy's, its distribution does not.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

BF16 = "bf16"
FP32 = "fp32"
FP16 = "fp16"
FP8 = "fp8_e4m3"
E4M3_MAX = 448.0


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits.

    Inputs here are finite, so no NaN handling is needed.
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return ((b + bias) >> np.uint32(16)).astype(np.uint16)


def f32_to_fp16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to IEEE binary16 (nearest, ties to even); uint16 bits."""
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def _e4m3_magnitudes() -> np.ndarray:
    """Values of the non-negative finite FP8 E4M3 codes 0..126, increasing:
    4 exponent bits (bias 7) and 3 mantissa bits, subnormals at exponent 0;
    code 127 is NaN, so 126 (448) is the largest finite value."""
    codes = np.arange(127)
    e, m = codes >> 3, codes & 7
    return np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 7))


_E4M3 = _e4m3_magnitudes()


def f32_to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """Round to FP8 E4M3 (nearest, ties to the even code); magnitudes beyond
    448 become 448.  Returns uint8 codes (sign in bit 7)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(_E4M3, a, side="left"), 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_lo, d_hi = a - _E4M3[lo], _E4M3[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    return code | (np.signbit(x).astype(np.uint8) << np.uint8(7))


def store(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 values in the storage format of ``dtype`` (bits or values)."""
    if dtype == BF16:
        return f32_to_bf16_bits(x)
    if dtype == FP16:
        return f32_to_fp16_bits(x)
    if dtype == FP8:
        return f32_to_e4m3_bits(x)
    if dtype == FP32:
        return np.ascontiguousarray(x, dtype=np.float32)
    raise ValueError("unknown dtype %r" % (dtype,))


@dataclasses.dataclass
class Case:
    """One synthetic QK-Norm input: fused buffer, weights and shape."""

    qkv: np.ndarray  # [T, row_stride]; uint16 bf16/fp16 bits, uint8 e4m3 codes, or float32
    gamma_q: np.ndarray  # float32
    gamma_k: Optional[np.ndarray]  # float32 or None when Hk == 0
    T: int
    Hq: int
    Hk: int
    D: int
    row_stride: int
    dtype: str
    eps: float
    layerwise: bool


def _counts(T: int, frac: float) -> int:
    return 0 if frac <= 0 else max(1, int(math.ceil(frac * T)))


def make_case(T, Hq, Hk, D, *, dtype=BF16, seed=0, row_stride=None, layerwise=False,
              scale=None, zero_frac=0.0, outlier_frac=0.0, eps=1e-6) -> Case:
    """Draw one case with numpy (``scale`` in {None, 'lognormal', 'stress'})."""
    W = (Hq + 2 * Hk) * D
    stride = W if row_stride is None else int(row_stride)
    if stride < W:
        raise ValueError("row_stride must be >= (Hq + 2*Hk) * D")
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, stride), dtype=np.float32)
    if scale == "lognormal":
        s = rng.lognormal(0.0, 1.0, size=T).astype(np.float32)
        x *= s[:, None]
    elif scale == "stress":
        s = np.clip(np.exp(rng.normal(0.0, 2.3, size=T)), 1e-3, 1e3).astype(np.float32)
        x *= s[:, None]
    elif scale is not None:
        raise ValueError("unknown scale recipe %r" % (scale,))
    qk = (Hq + Hk) * D
    nz, no = _counts(T, zero_frac), _counts(T, outlier_frac)
    if nz + no > 0:
        picked = rng.choice(T, size=min(T, nz + no), replace=False)
        zero_rows, out_rows = picked[:nz], picked[nz:]
        x[zero_rows, :qk] = 0.0
        cols = rng.integers(0, qk, size=out_rows.size)
        signs = rng.choice(np.array([-1.0, 1.0], dtype=np.float32), size=out_rows.size)
        x[out_rows, cols] = signs * np.float32(1e4)
    lq, lk = (Hq * D, Hk * D) if layerwise else (D, D)
    gamma_q = (1.0 + 0.1 * rng.standard_normal(lq)).astype(np.float32)
    gamma_k = (1.0 + 0.1 * rng.standard_normal(lk)).astype(np.float32) if Hk > 0 else None
    qkv = store(x, dtype)
    return Case(qkv, gamma_q, gamma_k, T, Hq, Hk, D, stride, dtype, eps, layerwise)


def make_case_torch(T, Hq, Hk, D, *, device, dtype=BF16, seed=0, row_stride=None,
                    layerwise=False, scale=None, zero_frac=0.0, outlier_frac=0.0, eps=1e-6):
    """Same recipe drawn with torch on ``device``; returns a dict of tensors."""
    import torch

    W = (Hq + 2 * Hk) * D
    stride = W if row_stride is None else int(row_stride)
    if stride < W:
        raise ValueError("row_stride must be >= (Hq + 2*Hk) * D")
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    tdt = {BF16: torch.bfloat16, FP32: torch.float32, FP16: torch.float16,
           FP8: torch.float8_e4m3fn}[dtype]
    qkv = torch.empty((T, stride), dtype=tdt, device=device)
    # Draw in float32 slabs so the temporary stays small for multi-GB buffers.
    slab = max(1, (1 << 26) // max(1, stride))
    for t0 in range(0, T, slab):
        t1 = min(T, t0 + slab)
        x = torch.randn((t1 - t0, stride), generator=g, device=device, dtype=torch.float32)
        if scale == "lognormal":
            s = torch.randn((t1 - t0, 1), generator=g, device=device).exp()
            x *= s
        elif scale == "stress":
            s = (torch.randn((t1 - t0, 1), generator=g, device=device) * 2.3).exp()
            x *= s.clamp_(1e-3, 1e3)
        elif scale is not None:
            raise ValueError("unknown scale recipe %r" % (scale,))
        if dtype == FP8:
            x.clamp_(-E4M3_MAX, E4M3_MAX)  # E4M3 has no infinities
        qkv[t0:t1] = x.to(tdt)
        del x
    qk = (Hq + Hk) * D
    nz, no = _counts(T, zero_frac), _counts(T, outlier_frac)
    if nz + no > 0:
        picked = torch.randperm(T, generator=g, device=device)[: min(T, nz + no)]
        zero_rows, out_rows = picked[:nz], picked[nz:]
        qkv[zero_rows, :qk] = 0
        cols = torch.randint(0, qk, (out_rows.numel(),), generator=g, device=device)
        signs = torch.randint(0, 2, (out_rows.numel(),), generator=g, device=device) * 2 - 1
        big = E4M3_MAX if dtype == FP8 else 1e4
        qkv[out_rows, cols] = (signs.float() * big).to(tdt)
    lq, lk = (Hq * D, Hk * D) if layerwise else (D, D)
    gamma_q = 1.0 + 0.1 * torch.randn(lq, generator=g, device=device, dtype=torch.float32)
    gamma_k = (1.0 + 0.1 * torch.randn(lk, generator=g, device=device, dtype=torch.float32)
               if Hk > 0 else None)
    return dict(qkv=qkv, gamma_q=gamma_q, gamma_k=gamma_k, T=T, Hq=Hq, Hk=Hk, D=D,
                row_stride=stride, dtype=dtype, eps=eps, layerwise=layerwise)


# Named workloads (shapes and distributions of the five configurations).
SMOKE = dict(T=4, Hq=16, Hk=2, D=128, dtype=BF16, seed=0, eps=1e-6)
SWEEP_HEADS = (16, 32, 48)
SWEEP_T = tuple(2 ** k for k in range(13))  # 1 .. 4096
SWEEP_SEED = 1001
GQA = dict(Hq=32, Hk=8, D=128, dtype=BF16, scale="lognormal", eps=1e-6)
GQA_T = (1, 64, 1024, 4096, 16384)
GQA_SEED = 1002
LAYERWISE = dict(Hq=32, Hk=8, D=128, dtype=BF16, layerwise=True, eps=1e-6)
LAYERWISE_T = (1, 16, 256, 4096, 8192)
LAYERWISE_NSHARDS = (1, 2, 4, 8)
LAYERWISE_SEED = 1003
STRESS = dict(Hq=64, Hk=8, T=32768, scale="stress", zero_frac=0.01, outlier_frac=0.01)
STRESS_D = (64, 128, 256)
STRESS_DTYPES = (BF16, FP32)
STRESS_EPS = (1e-6, 1e-5)
STRESS_SEED = 1004


def sweep_case(H: int, T: int, seed: int = SWEEP_SEED) -> Case:
    """Per-head sweep point: Q-style contiguous ``[T, H, 128]`` (Hk = 0)."""
    return make_case(T, H, 0, 128, dtype=BF16, seed=seed + 97 * H + T, eps=1e-6)
