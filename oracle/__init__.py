"""Float64 CPU oracle for QK-Norm (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package.  The product path never does, and this
package imports nothing from the product package: the C source
``qknorm_oracle.c`` is compiled by ``gcc`` on its own and called through
ctypes.

Definitions followed (the header of ``qknorm_oracle.c`` states them in full):

* RMSNorm ``y = x * g / sqrt(mean(x^2) + eps)`` -- SwiftQK review
  (pith.science verdict for arXiv 2608.09160), ``core_discovery`` and
  ``key_machinery``.
* per-head rows of length ``head_dim`` with one weight for Q and one for K --
  sglang PR #13189, Motivation and Modifications (``hidden_size <= 128``).
* layerwise rows over the full q / k vector, and the sharded scalar combine --
  SwiftQK abstract and review ``key_machinery``.
* fused ``[T, (Hq + 2*Hk) * D]`` buffer, split by head -- "combined QKV
  projection" lesson, GQA section and tensor-parallel follow-up.

Inputs are widened exactly to float64 here: bf16 bit patterns (uint16) are
shifted into the high half of a float32, fp16 bit patterns are read as IEEE
binary16, FP8 E4M3 codes are decoded from the format's definition, float32
values are cast.  The
oracle is pinned by closed forms and invariants (``tests/pins.py``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "qknorm_oracle.c")
_LIB = os.path.join(HERE, "libqknorm_oracle.so")
_lock = threading.Lock()
_default = None

BF16 = "bf16"
FP32 = "fp32"
FP16 = "fp16"
FP8 = "fp8_e4m3"


def _e4m3_table() -> np.ndarray:
    """float64 value of each of the 256 FP8 E4M3 codes: sign bit 7, exponent
    bits 6..3 with bias 7, mantissa bits 2..0; exponent 0 is subnormal
    (m * 2^-9); 0x7f and 0xff are NaN (the format has no infinities)."""
    out = np.empty(256)
    for c in range(256):
        sign = -1.0 if c & 0x80 else 1.0
        e, m = (c >> 3) & 0xF, c & 0x7
        if e == 0xF and m == 0x7:
            out[c] = np.nan
        elif e == 0:
            out[c] = sign * m * 2.0 ** -9
        else:
            out[c] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


_E4M3 = _e4m3_table()


def compile_source(src: str, out: str) -> str:
    """Compile one oracle C source with gcc (-O2, OpenMP, no fast-math)."""
    tmp = out + ".%d.tmp" % os.getpid()
    subprocess.check_call(
        ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", src, "-o", tmp, "-lm"]
    )
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Build ``libqknorm_oracle.so`` next to its source when stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(SOURCE):
        compile_source(SOURCE, _LIB)
    return _LIB


def widen(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of stored elements: bf16 / fp16 bits as uint16, FP8
    E4M3 codes as uint8, or fp32 values."""
    if dtype == BF16:
        bits = np.ascontiguousarray(x, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
        return bits.view(np.float32).astype(np.float64)
    if dtype == FP32:
        return np.ascontiguousarray(x, dtype=np.float32).astype(np.float64)
    if dtype == FP16:
        return np.ascontiguousarray(x, dtype=np.uint16).view(np.float16).astype(np.float64)
    if dtype == FP8:
        return _E4M3[np.ascontiguousarray(x, dtype=np.uint8)]
    raise ValueError("dtype must be 'bf16', 'fp32', 'fp16' or 'fp8_e4m3'")


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


class Oracle:
    """ctypes front end of one compiled oracle library."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        common = [dp, dp, i64, i32, i32, i32, i64, dp, dp, f64]
        lib.oracle_per_head.argtypes = common + [i32]
        lib.oracle_per_head.restype = None
        lib.oracle_layerwise.argtypes = common + [i32]
        lib.oracle_layerwise.restype = None
        lib.oracle_layerwise_sharded.argtypes = common + [i32, i32]
        lib.oracle_layerwise_sharded.restype = ctypes.c_int
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = ctypes.c_int
        self.lib = lib

    @staticmethod
    def _prep(x, dtype, T, row_stride, gamma_q, gamma_k):
        xd = np.ascontiguousarray(widen(x, dtype).reshape(T, row_stride))
        gq = np.ascontiguousarray(np.asarray(gamma_q, dtype=np.float64).ravel())
        gk = np.ascontiguousarray(
            np.asarray(gamma_k if gamma_k is not None else np.zeros(1), dtype=np.float64).ravel()
        )
        return xd, np.empty_like(xd), gq, gk

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    def per_head(self, x, dtype, T, Hq, Hk, D, row_stride, gamma_q, gamma_k, eps, nthreads=1):
        """Per-head QK-Norm of a fused buffer; returns float64 ``[T, row_stride]``."""
        xd, y, gq, gk = self._prep(x, dtype, T, row_stride, gamma_q, gamma_k)
        if gq.size < D or (Hk > 0 and gk.size < D):
            raise ValueError("per-head weights must have head_dim elements")
        self.lib.oracle_per_head(_dptr(xd), _dptr(y), T, Hq, Hk, D, row_stride, _dptr(gq),
                                 _dptr(gk), float(eps), int(nthreads))
        return y

    def layerwise(self, x, dtype, T, Hq, Hk, D, row_stride, gamma_q, gamma_k, eps, nthreads=1):
        """Layerwise QK-Norm (no shards); returns float64 ``[T, row_stride]``."""
        xd, y, gq, gk = self._prep(x, dtype, T, row_stride, gamma_q, gamma_k)
        if gq.size < Hq * D or (Hk > 0 and gk.size < Hk * D):
            raise ValueError("layerwise weights must have Hq*D and Hk*D elements")
        self.lib.oracle_layerwise(_dptr(xd), _dptr(y), T, Hq, Hk, D, row_stride, _dptr(gq),
                                  _dptr(gk), float(eps), int(nthreads))
        return y

    def layerwise_sharded(self, x, dtype, T, Hq, Hk, D, row_stride, gamma_q, gamma_k, eps,
                          nshards, nthreads=1):
        """Layerwise QK-Norm through per-shard partial sums and a scalar combine."""
        xd, y, gq, gk = self._prep(x, dtype, T, row_stride, gamma_q, gamma_k)
        if gq.size < Hq * D or (Hk > 0 and gk.size < Hk * D):
            raise ValueError("layerwise weights must have Hq*D and Hk*D elements")
        rc = self.lib.oracle_layerwise_sharded(_dptr(xd), _dptr(y), T, Hq, Hk, D, row_stride,
                                               _dptr(gq), _dptr(gk), float(eps), int(nshards),
                                               int(nthreads))
        if rc != 0:
            raise ValueError("nshards must be >= 1 and divide both Hq and Hk")
        return y


def default() -> Oracle:
    """The oracle built from the committed source."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def per_head(*args, **kwargs):
    return default().per_head(*args, **kwargs)


def layerwise(*args, **kwargs):
    return default().layerwise(*args, **kwargs)


def layerwise_sharded(*args, **kwargs):
    return default().layerwise_sharded(*args, **kwargs)


def max_threads() -> int:
    return default().max_threads()
