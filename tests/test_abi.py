"""The C ABI of libqknorm.so on a host without a GPU.

Loads the library, checks that it exports every entry point declared in
include/qknorm.h, and drives argument validation, which returns before any
CUDA call (no kernel runs here).
"""
import ctypes
import math
import os
import re
import subprocess

import pytest

import attention_qk_norm_b200 as qkn
from attention_qk_norm_b200 import buildlib as qbuild

HEADER = os.path.join(qbuild.INCLUDE, "qknorm.h")
OK, NULL, SHAPE, ALIGN, NSHARDS, UNSUP, CUDA, EPS = 0, -1, -2, -3, -4, -5, -6, -7
BF16, FP32, FP16, FP8 = 0, 1, 2, 3
# Fake, never-dereferenced addresses: validation rejects before any access.
P, G1, G2 = 0x100000, 0x200000, 0x300000


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return qkn.load_library()


def declared_symbols():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(qknorm_\w+)\s*\(", text, re.M)))


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert set(names) == {"qknorm_per_head", "qknorm_layerwise", "qknorm_status_string",
                          "qknorm_last_cuda_error", "qknorm_version", "qknorm_layerwise_partials",
                          "qknorm_layerwise_apply", "qknorm_layerwise_noalloc",
                          "qknorm_wait_timeouts", "qknorm_tp_comm_create",
                          "qknorm_tp_comm_connect", "qknorm_tp_comm_create_local",
                          "qknorm_tp_comm_destroy", "qknorm_tp_comm_errors",
                          "qknorm_layerwise_tp_p2p"}
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", qbuild.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (qknorm_\w+)$", out, re.M))
    assert set(names) <= exported


def test_version_and_status_strings(lib):
    assert lib.qknorm_version() == 105
    for code in (OK, NULL, SHAPE, ALIGN, NSHARDS, UNSUP, CUDA, EPS, -8):
        s = lib.qknorm_status_string(code).decode()
        assert s and s != "unknown status"
    assert lib.qknorm_status_string(42).decode() == "unknown status"
    assert lib.qknorm_last_cuda_error() == 0
    # Only the argument check runs without a GPU.
    assert lib.qknorm_wait_timeouts(None) == NULL


def ph(lib, qkv=P, dtype=BF16, T=4, Hq=16, Hk=2, D=128, stride=None, gq=G1, gk=G2, eps=1e-6):
    stride = (Hq + 2 * Hk) * D if stride is None else stride
    return lib.qknorm_per_head(qkv, dtype, T, Hq, Hk, D, stride, gq, gk, eps, None)


def lw(lib, qkv=P, dtype=BF16, T=4, Hq=32, Hk=8, D=128, stride=None, gq=G1, gk=G2, eps=1e-6,
       n=1):
    stride = (Hq + 2 * Hk) * D if stride is None else stride
    return lib.qknorm_layerwise(qkv, dtype, T, Hq, Hk, D, stride, gq, gk, eps, n, None)


@pytest.mark.parametrize("fn", [ph, lw])
def test_validation(lib, fn):
    assert fn(lib, dtype=4) == UNSUP
    assert fn(lib, dtype=-1) == UNSUP
    assert fn(lib, D=96) == UNSUP
    assert fn(lib, D=32) == UNSUP
    assert fn(lib, Hq=0, Hk=0) == SHAPE
    assert fn(lib, Hq=-1) == SHAPE
    assert fn(lib, T=-1) == SHAPE
    W = (16 + 4) * 128 if fn is ph else (32 + 16) * 128
    assert fn(lib, stride=W - 8) == SHAPE
    assert fn(lib, eps=-1.0) == EPS
    assert fn(lib, eps=float("nan")) == EPS
    assert fn(lib, eps=math.inf) == EPS
    assert fn(lib, T=0, qkv=None, gq=None, gk=None) == OK  # empty: no launch, no pointers
    assert fn(lib, qkv=None) == NULL
    assert fn(lib, gq=None) == NULL
    assert fn(lib, gk=None) == NULL
    assert fn(lib, qkv=P + 8) == ALIGN
    assert fn(lib, gq=G1 + 4) == ALIGN
    assert fn(lib, gk=G2 + 4) == ALIGN
    assert fn(lib, stride=W + 4) == ALIGN  # 8 bytes of bf16: rows lose 16-byte alignment
    assert fn(lib, dtype=FP32, stride=W + 2) == ALIGN
    assert fn(lib, dtype=FP16, stride=W + 4) == ALIGN
    assert fn(lib, dtype=FP8, stride=W + 8) == ALIGN  # 8 bytes of e4m3 per row
    for dt in (FP16, FP8):  # accepted dtypes reach the pointer checks
        assert fn(lib, dtype=dt, qkv=P + 8) == ALIGN
    assert lib.qknorm_last_cuda_error() == 0


def test_gamma_k_optional_without_k_heads(lib):
    # Hk == 0: gamma_k may be NULL; the call then reaches the alignment check.
    assert ph(lib, Hk=0, gk=None, qkv=P + 8) == ALIGN
    assert lw(lib, Hk=0, gk=None, qkv=P + 8) == ALIGN
    assert ph(lib, Hq=0, Hk=2, gq=None, qkv=P + 8) == ALIGN


def test_layerwise_nshards(lib):
    for n in (0, 3, 5, 16, -1):
        assert lw(lib, n=n) == NSHARDS
    assert lw(lib, Hq=6, Hk=2, n=4) == NSHARDS
    assert lw(lib, Hq=8, Hk=2, n=4) == NSHARDS
    assert lw(lib, T=0, n=3) == NSHARDS  # checked even when there is nothing to do
    assert lw(lib, T=0, n=8, qkv=None) == OK
    assert lw(lib, n=8, qkv=P + 8) == ALIGN  # valid nshards, reaches later checks


def test_tensor_parallel_steps_validation(lib):
    W = (32 + 16) * 128
    part = lib.qknorm_layerwise_partials
    assert part(P, BF16, 4, 32, 8, 128, W, None, None) == NULL
    assert part(P, BF16, 4, 32, 8, 128, W, G1 + 4, None) == ALIGN
    assert part(P + 8, BF16, 4, 32, 8, 128, W, G1, None) == ALIGN
    assert part(P, BF16, 4, 32, 8, 96, W, G1, None) == UNSUP
    assert part(None, BF16, 0, 32, 8, 128, W, None, None) == OK  # T == 0: nothing to do
    app = lib.qknorm_layerwise_apply
    args = (BF16, 4, 32, 8, 128, W, G1, G2)
    assert app(P, *args, None, 4 * 4096, 4 * 1024, 1e-6, None) == NULL
    S = 0x300000  # 8-byte aligned; S + 4 is not
    assert app(P, *args, S + 4, 4 * 4096, 4 * 1024, 1e-6, None) == ALIGN
    assert app(P, *args, S, 4095, 1024, 1e-6, None) == SHAPE  # below this rank's Hq*D
    assert app(P, *args, S, 4096, 1023, 1e-6, None) == SHAPE
    assert app(P, *args, S, 1 << 25, 1024, 1e-6, None) == SHAPE
    assert app(P, *args, S, 4096, 1024, -1.0, None) == EPS
    assert app(P, BF16, 4, 32, 8, 128, W, None, G2, S, 4096, 1024, 1e-6, None) == NULL
    assert app(None, BF16, 0, 32, 8, 128, W, None, None, None, 4096, 1024, 1e-6, None) == OK
    assert lib.qknorm_last_cuda_error() == 0


def test_noalloc_validation(lib):
    f = lib.qknorm_layerwise_noalloc
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                  ctypes.c_void_p]
    f.restype = ctypes.c_int
    W = (32 + 16) * 128
    assert f(P, BF16, 65537, 32, 8, 128, W, G1, G2, 1e-6, None) == -8  # beyond the scratch
    assert lib.qknorm_status_string(-8).decode().startswith("T exceeds")
    assert f(None, BF16, 4, 32, 8, 128, W, G1, G2, 1e-6, None) == NULL
    assert f(P + 8, BF16, 4, 32, 8, 128, W, G1, G2, 1e-6, None) == ALIGN
    assert f(None, BF16, 0, 32, 8, 128, W, None, None, 1e-6, None) == OK
    assert lib.qknorm_last_cuda_error() == 0


def test_tp_lengths():
    assert qkn.tp_full_lengths(8, 2, 128, 4) == (4096, 1024)
    assert qkn.tp_allreduce_(None) == 1  # no process group: a single rank


def test_binding_rejects_host_tensors():
    import torch

    x = torch.zeros(4, 2560, dtype=torch.bfloat16)
    g = torch.ones(128)
    with pytest.raises(ValueError):
        qkn.qknorm_per_head(x, 16, 2, 128, g, g, 1e-6)
    with pytest.raises(ValueError):
        qkn.qknorm_layerwise(x, 16, 2, 128, g, g, 1e-6, nshards=2)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="not built"):
        qkn.load_library(str(tmp_path / "nope.so"))


def test_product_and_oracle_are_independent():
    root = os.path.dirname(qbuild.PKG)
    for d in ("attention_qk_norm_b200", "include"):
        for dirpath, _, files in os.walk(os.path.join(root, d)):
            for f in files:
                if f.endswith((".py", ".cu", ".h", ".cuh", ".cpp")):
                    text = open(os.path.join(dirpath, f)).read()
                    bad = re.search(r"^\s*(import|from)\s+oracle\b|\boracle\.\w+\(|qknorm_oracle",
                                    text, re.M)
                    assert not bad, (f, "product path reaches the oracle")
    for f in os.listdir(os.path.join(root, "oracle")):
        if f.endswith((".py", ".c", ".h")):
            text = open(os.path.join(root, "oracle", f)).read()
            assert "attention_qk_norm_b200" not in text and "qknorm.h" not in text, f
