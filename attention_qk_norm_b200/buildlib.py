"""Build ``libqknorm.so`` in-tree with nvcc for sm_100a.

The library links the CUDA runtime statically, so it loads on a host
without a GPU (argument validation needs no device) and does not depend on
the runtime version torch ships.
"""
from __future__ import annotations

import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
INCLUDE = os.path.join(ROOT, "include")
CSRC = os.path.join(PKG, "csrc")
SOURCES = [os.path.join(CSRC, "qknorm.cu")]
HEADERS = [os.path.join(INCLUDE, "qknorm.h")] + sorted(
    os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh"))
LIB_PATH = os.path.join(PKG, "libqknorm.so")
# The tensor-parallel exchange protocol built for the host (tests only).
TP_HOST_SOURCE = os.path.join(CSRC, "tp_exchange_host.cc")
TP_HOST_LIB = os.path.join(PKG, "libqknorm_tp_host.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
]


def nvcc() -> str:
    found = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(found):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libqknorm.so")
    return found


def code_only(text: str) -> str:
    """C/C++/CUDA source text without its comments and with each run of
    whitespace made one space: what the compiler reads."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":  # a string or character literal, copied whole
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_sources() -> list:
    """The files compiled into the kernels: the translation unit and the
    headers beside it."""
    return sorted(SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC)
                             if f.endswith((".cuh", ".h"))])


def kernel_source_sha256(read=None) -> str:
    """SHA-256 over the code of the library's CUDA sources (file names and
    their text without comments, in name order); recorded ncu counters are
    valid only for the code they were taken from.  ``read(path)`` returns a
    file's text (default: the file on disk)."""
    import hashlib

    read = read or (lambda p: open(p, encoding="utf-8").read())
    h = hashlib.sha256()
    for p in kernel_sources():
        h.update(os.path.basename(p).encode() + b"\0")
        h.update(code_only(read(p)).encode())
    return h.hexdigest()


def is_stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS)


def build(force: bool = False, extra_flags=(), out: str = LIB_PATH) -> str:
    """Compile the CUDA sources into ``out`` when stale (or always if forced)."""
    if not force and out == LIB_PATH and not is_stale():
        return out
    tmp = out + ".%d.tmp" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, *extra_flags, "-I", INCLUDE, *SOURCES, "-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build_tp_host(force: bool = False) -> str:
    """Compile the host build of the exchange protocol (tp_exchange.h) that
    the CPU tests run with one process per rank."""
    deps = [TP_HOST_SOURCE, os.path.join(CSRC, "tp_exchange.h")]
    if (not force and os.path.exists(TP_HOST_LIB)
            and all(os.path.getmtime(p) <= os.path.getmtime(TP_HOST_LIB) for p in deps)):
        return TP_HOST_LIB
    tmp = TP_HOST_LIB + ".%d.tmp" % os.getpid()
    gxx = shutil.which("g++") or "g++"
    subprocess.check_call([gxx, "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", "-I", CSRC,
                           TP_HOST_SOURCE, "-o", tmp])
    os.replace(tmp, TP_HOST_LIB)
    return TP_HOST_LIB


if __name__ == "__main__":
    print(build(force=True))
    print(build_tp_host(force=True))
