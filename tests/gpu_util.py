"""Helpers shared by the GPU parity tests (no test functions here).

Tolerances (per output element o of the float64 oracle, g of the kernel):
* bf16 outputs: |g - o| <= 7.9e-3 * |o|  (one bf16 ulp relative, 2^-7);
* fp16 outputs: |g - o| <= 9.8e-4 * |o| + 2^-24 (one fp16 ulp relative, 2^-10,
  plus half the subnormal spacing);
* fp32 outputs: |g - o| <= 1e-5 * |o|;
* FP8 E4M3 outputs are codes, so they are compared as codes: g must be the
  round-to-nearest-even code of o (saturating at 448), except where o lies
  within 1e-5 relative of the midpoint between two codes, where the kernel's
  fp32 value may fall on either side and both neighbours are accepted;
* o == 0 (all-zero rows): g must be exactly zero.
V columns and row padding must come back bit-identical.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from attention_qk_norm_b200 import synth

TOL = {synth.BF16: 7.9e-3, synth.FP32: 1e-5, synth.FP16: 9.8e-4}
ABS = {synth.BF16: 0.0, synth.FP32: 0.0, synth.FP16: 2.0 ** -24}
# Decoded value of every E4M3 code, from torch (a library decode, independent
# of the oracle's and of the input generator's tables).
E4M3 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
E4M3_POS = E4M3[:127]  # codes 0..126: the non-negative finite values, increasing


def to_device(case: synth.Case, device="cuda", extra_rows: int = 0):
    """Upload a numpy case.  ``extra_rows`` appends guard rows after the buffer."""
    if case.dtype == synth.BF16:
        host = torch.from_numpy(case.qkv.view(np.int16).copy()).view(torch.bfloat16)
    elif case.dtype == synth.FP16:
        host = torch.from_numpy(case.qkv.view(np.int16).copy()).view(torch.float16)
    elif case.dtype == synth.FP8:
        host = torch.from_numpy(case.qkv.copy()).view(torch.float8_e4m3fn)
    else:
        host = torch.from_numpy(case.qkv.copy())
    full = torch.empty((case.T + extra_rows, case.row_stride), dtype=host.dtype, device=device)
    full[: case.T] = host.to(device)
    if extra_rows:
        fill = torch.full((extra_rows, case.row_stride), -7.25, dtype=host.dtype)
        full[case.T:] = fill.to(device)
    gq = torch.from_numpy(case.gamma_q).to(device)
    gk = None if case.gamma_k is None else torch.from_numpy(case.gamma_k).to(device)
    return full, gq, gk


def stored_bits(t: torch.Tensor) -> np.ndarray:
    """Host copy of a device tensor's stored elements (uint16 bits or float32)."""
    t = t.detach().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def as_f64(stored: np.ndarray, dtype: str) -> np.ndarray:
    """float64 value of stored elements (exact).  Test-side conversion."""
    if dtype == synth.BF16:
        return (stored.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if dtype == synth.FP16:
        return stored.view(np.float16).astype(np.float64)
    if dtype == synth.FP8:
        return E4M3[stored]
    return stored.astype(np.float64)


def e4m3_codes_ok(g: np.ndarray, o: np.ndarray) -> np.ndarray:
    """Per element: is code g acceptable for the exact value o (see above)?"""
    a = np.minimum(np.abs(o), 448.0)
    hi = np.clip(np.searchsorted(E4M3_POS, a, side="left"), 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_lo, d_hi = a - E4M3_POS[lo], E4M3_POS[hi] - a
    rne = np.where((d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0)), hi, lo)
    mid = 0.5 * (E4M3_POS[lo] + E4M3_POS[hi])
    near_mid = np.abs(a - mid) <= 1e-5 * a
    sign = np.where(np.signbit(o), 0x80, 0)
    mag, gsign = g & 0x7F, g & 0x80
    same_sign = (gsign == sign) | (mag == 0)
    ok = same_sign & ((mag == rne) | (near_mid & ((mag == lo) | (mag == hi))))
    return np.where(o == 0, mag == 0, ok)


def oracle_out(case_like, kind: str, x_stored: np.ndarray, T: int):
    c = case_like
    fn = oracle.per_head if kind == "per_head" else oracle.layerwise
    return fn(x_stored, c.dtype, T, c.Hq, c.Hk, c.D, c.row_stride, c.gamma_q, c.gamma_k, c.eps,
              nthreads=oracle.max_threads())


def check(gpu_stored: np.ndarray, want: np.ndarray, x_stored: np.ndarray, dtype: str,
          qk_cols: int, what: str = ""):
    """Compare Q/K columns within tolerance, V/padding bit for bit."""
    g = as_f64(gpu_stored[:, :qk_cols], dtype)
    o = want[:, :qk_cols]
    err = np.abs(g - o)
    if dtype == synth.FP8:
        bad = ~e4m3_codes_ok(gpu_stored[:, :qk_cols], o)
    else:
        bad = ~(err <= TOL[dtype] * np.abs(o) + ABS[dtype])
    if bad.any():
        idx = np.argwhere(bad)[:5].tolist()
        raise AssertionError("%s: %d elements out of tolerance, e.g. %s: gpu %s oracle %s" % (
            what, int(bad.sum()), idx, [g[tuple(i)] for i in idx], [o[tuple(i)] for i in idx]))
    assert np.array_equal(gpu_stored[:, qk_cols:], x_stored[:, qk_cols:]), \
        "%s: V or padding changed" % what
    nz = o != 0
    return float((err[nz] / np.abs(o[nz])).max()) if nz.any() else 0.0


class Sampled:
    """Shape and weights of a device case, in the form ``oracle_out`` takes."""

    def __init__(self, d: dict):
        self.dtype = d["dtype"]
        self.Hq, self.Hk, self.D = d["Hq"], d["Hk"], d["D"]
        self.row_stride = d["row_stride"]
        self.eps = d["eps"]
        self.gamma_q = d["gamma_q"].cpu().numpy()
        self.gamma_k = None if d["gamma_k"] is None else d["gamma_k"].cpu().numpy()


def sample_tokens(qkv: torch.Tensor, qk_cols: int, n_random: int, seed: int) -> torch.Tensor:
    """Token indices: random ones, the ends, and the special rows (all-zero
    Q+K span, or an element of magnitude >= 9000)."""
    T = qkv.shape[0]
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    pick = [torch.randint(0, T, (n_random,), generator=g), torch.tensor([0, T - 1])]
    span = qkv[:, :qk_cols]
    zero = torch.nonzero((span == 0).all(dim=1)).flatten()[:64].cpu()
    big = torch.nonzero((span.float().abs() >= 9000).any(dim=1)).flatten()[:64].cpu()
    return torch.unique(torch.cat(pick + [zero, big])).to(qkv.device)
