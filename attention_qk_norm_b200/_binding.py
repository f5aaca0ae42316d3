"""ctypes binding of libqknorm.so: argument marshalling only.

Every step of QK-Norm runs in the library's CUDA kernels; this module turns
torch tensors into pointers, sizes and a stream handle, calls the C entry
point of the same name, and raises ``QKNormError`` on a non-zero status.
There is no fallback: if the library is missing, loading fails loudly.
"""
from __future__ import annotations

import ctypes
import os
import threading

from .buildlib import LIB_PATH

QKN_BF16, QKN_FP32, QKN_FP16, QKN_FP8_E4M3 = 0, 1, 2, 3
STATUS = {
    0: "QKN_OK", -1: "QKN_ERR_NULL", -2: "QKN_ERR_SHAPE", -3: "QKN_ERR_ALIGN",
    -4: "QKN_ERR_NSHARDS", -5: "QKN_ERR_UNSUPPORTED", -6: "QKN_ERR_CUDA", -7: "QKN_ERR_EPS",
    -8: "QKN_ERR_TOO_LARGE",
}

_lock = threading.Lock()
_lib = None


class QKNormError(RuntimeError):
    """A non-zero qkn_status returned by libqknorm.so."""

    def __init__(self, fn: str, status: int, message: str, cuda_error: int = 0):
        self.status = status
        self.cuda_error = cuda_error
        extra = " (cudaError %d)" % cuda_error if status == -6 else ""
        super().__init__("%s: %s [%s]%s" % (fn, message, STATUS.get(status, status), extra))


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libqknorm.so and declare its prototypes (include/qknorm.h)."""
    global _lib
    with _lock:
        if _lib is not None and path == LIB_PATH:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                "libqknorm.so is not built at %s; run `python -m attention_qk_norm_b200.buildlib` "
                "(QK-Norm has no non-CUDA path)" % path)
        lib = ctypes.CDLL(path)
        vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        lib.qknorm_per_head.argtypes = [vp, i32, i64, i32, i32, i32, i64, vp, vp, f32, vp]
        lib.qknorm_per_head.restype = i32
        lib.qknorm_layerwise.argtypes = [vp, i32, i64, i32, i32, i32, i64, vp, vp, f32, i32, vp]
        lib.qknorm_layerwise.restype = i32
        lib.qknorm_layerwise_partials.argtypes = [vp, i32, i64, i32, i32, i32, i64, vp, vp]
        lib.qknorm_layerwise_partials.restype = i32
        lib.qknorm_layerwise_apply.argtypes = [vp, i32, i64, i32, i32, i32, i64, vp, vp, vp,
                                               i64, i64, f32, vp]
        lib.qknorm_layerwise_apply.restype = i32
        lib.qknorm_status_string.argtypes = [i32]
        lib.qknorm_status_string.restype = ctypes.c_char_p
        lib.qknorm_last_cuda_error.argtypes = []
        lib.qknorm_last_cuda_error.restype = i32
        lib.qknorm_version.argtypes = []
        lib.qknorm_version.restype = i32
        lib.qknorm_wait_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint)]
        lib.qknorm_wait_timeouts.restype = i32
        lib.qknorm_tp_comm_create.argtypes = [i32, i32, i64, ctypes.c_double,
                                              ctypes.POINTER(vp), vp]
        lib.qknorm_tp_comm_create.restype = i32
        lib.qknorm_tp_comm_connect.argtypes = [vp, vp]
        lib.qknorm_tp_comm_connect.restype = i32
        lib.qknorm_tp_comm_create_local.argtypes = [i32, i64, ctypes.c_double,
                                                    ctypes.POINTER(vp)]
        lib.qknorm_tp_comm_create_local.restype = i32
        lib.qknorm_tp_comm_destroy.argtypes = [vp]
        lib.qknorm_tp_comm_destroy.restype = i32
        lib.qknorm_tp_comm_errors.argtypes = [vp, ctypes.POINTER(ctypes.c_uint)]
        lib.qknorm_tp_comm_errors.restype = i32
        lib.qknorm_layerwise_tp_p2p.argtypes = [vp, vp, i32, i64, i32, i32, i32, i64, vp, vp, f32,
                                                vp]
        lib.qknorm_layerwise_tp_p2p.restype = i32
        if path == LIB_PATH:
            _lib = lib
        return lib


def status_string(status: int) -> str:
    return load_library().qknorm_status_string(int(status)).decode()


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        lib = load_library()
        raise QKNormError(fn, rc, lib.qknorm_status_string(rc).decode(),
                          lib.qknorm_last_cuda_error())


def _dtype_code(t) -> int:
    import torch

    codes = {torch.bfloat16: QKN_BF16, torch.float32: QKN_FP32, torch.float16: QKN_FP16,
             torch.float8_e4m3fn: QKN_FP8_E4M3}
    if t.dtype not in codes:
        raise TypeError("qkv must be bfloat16, float32, float16 or float8_e4m3fn, got %s"
                        % t.dtype)
    return codes[t.dtype]


def _rows(qkv, row_stride):
    if qkv.dim() != 2 or qkv.stride(1) != 1:
        raise ValueError("qkv must be a 2-D [T, row_stride] view with unit column stride")
    stride = qkv.stride(0) if row_stride is None else int(row_stride)
    return qkv.shape[0], stride


def _stream_ptr(qkv, stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream(qkv.device)
    return ctypes.c_void_p(int(stream.cuda_stream))


def _gamma_ptr(g, name):
    import torch

    if g is None:
        return None
    if g.dtype != torch.float32 or not g.is_contiguous():
        raise TypeError("%s must be a contiguous float32 tensor" % name)
    return ctypes.c_void_p(g.data_ptr())


def _device_check(qkv, *others):
    if not qkv.is_cuda:
        raise ValueError("qkv must be a CUDA tensor (QK-Norm runs only on the GPU)")
    for g in others:
        if g is not None and g.device != qkv.device:
            raise ValueError("gamma and sums must live on the same device as qkv")


def wait_timeouts() -> int:
    """In-kernel waits on the current device that gave up (qknorm_wait_timeouts)."""
    count = ctypes.c_uint(0)
    _check("qknorm_wait_timeouts", load_library().qknorm_wait_timeouts(ctypes.byref(count)))
    return int(count.value)


def qknorm_per_head(qkv, Hq, Hk, D, gamma_q, gamma_k, eps, row_stride=None, stream=None):
    """Per-head QK-Norm in place on ``qkv`` [T, row_stride] (see qknorm.h)."""
    _device_check(qkv, gamma_q, gamma_k)
    T, stride = _rows(qkv, row_stride)
    rc = load_library().qknorm_per_head(
        ctypes.c_void_p(qkv.data_ptr()), _dtype_code(qkv), T, Hq, Hk, D, stride,
        _gamma_ptr(gamma_q, "gamma_q"), _gamma_ptr(gamma_k, "gamma_k"), float(eps),
        _stream_ptr(qkv, stream))
    _check("qknorm_per_head", rc)
    return qkv


def qknorm_layerwise(qkv, Hq, Hk, D, gamma_q, gamma_k, eps, nshards=1, row_stride=None,
                     stream=None):
    """Layerwise (SwiftQK) QK-Norm in place on ``qkv`` [T, row_stride]."""
    _device_check(qkv, gamma_q, gamma_k)
    T, stride = _rows(qkv, row_stride)
    rc = load_library().qknorm_layerwise(
        ctypes.c_void_p(qkv.data_ptr()), _dtype_code(qkv), T, Hq, Hk, D, stride,
        _gamma_ptr(gamma_q, "gamma_q"), _gamma_ptr(gamma_k, "gamma_k"), float(eps),
        int(nshards), _stream_ptr(qkv, stream))
    _check("qknorm_layerwise", rc)
    return qkv


def qknorm_layerwise_partials(qkv, Hq, Hk, D, partials=None, row_stride=None, stream=None):
    """This rank's per-token fp32 sums of squares, ``[T, 2]`` (q, k) float32.

    ``qkv`` holds this rank's heads (Hq query, Hk key/value) in the fused
    layout; it is only read.  ``partials`` may be passed to reuse memory."""
    import torch

    _device_check(qkv)
    T, stride = _rows(qkv, row_stride)
    if partials is None:
        partials = torch.empty((T, 2), dtype=torch.float32, device=qkv.device)
    if partials.dtype != torch.float32 or not partials.is_contiguous() or partials.numel() < 2 * T:
        raise ValueError("partials must be a contiguous float32 tensor of 2*T elements")
    rc = load_library().qknorm_layerwise_partials(
        ctypes.c_void_p(qkv.data_ptr()), _dtype_code(qkv), T, Hq, Hk, D, stride,
        ctypes.c_void_p(partials.data_ptr()), _stream_ptr(qkv, stream))
    _check("qknorm_layerwise_partials", rc)
    return partials


def qknorm_layerwise_apply(qkv, Hq, Hk, D, gamma_q, gamma_k, sums, len_q, len_k, eps,
                           row_stride=None, stream=None):
    """Scale this rank's q / k columns in place by the inverse RMS that the
    summed partials ``sums`` ([T, 2] float32) and the full lengths give."""
    import torch

    _device_check(qkv, gamma_q, gamma_k, sums)
    T, stride = _rows(qkv, row_stride)
    if sums.dtype != torch.float32 or not sums.is_contiguous() or sums.numel() < 2 * T:
        raise ValueError("sums must be a contiguous float32 tensor of 2*T elements")
    rc = load_library().qknorm_layerwise_apply(
        ctypes.c_void_p(qkv.data_ptr()), _dtype_code(qkv), T, Hq, Hk, D, stride,
        _gamma_ptr(gamma_q, "gamma_q"), _gamma_ptr(gamma_k, "gamma_k"),
        ctypes.c_void_p(sums.data_ptr()), int(len_q), int(len_k), float(eps),
        _stream_ptr(qkv, stream))
    _check("qknorm_layerwise_apply", rc)
    return qkv


def tp_allreduce_(partials, group=None) -> int:
    """Sum ``partials`` over the ranks of ``group`` in place (one all-reduce;
    nothing without an initialised process group); returns the group size."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return 1
    world = dist.get_world_size(group)
    if world > 1:
        dist.all_reduce(partials, op=dist.ReduceOp.SUM, group=group)
    return world


def tp_full_lengths(Hq, Hk, D, world):
    """Full q / k vector lengths when every rank holds Hq and Hk heads."""
    return Hq * D * world, Hk * D * world


def tp_allgather_full(xq, xk, group=None):
    """All-gather this rank's q and k columns ([T, hq*D] and [T, hk*D]) over
    ``group``; returns (full q [T, world*hq*D], full k [T, world*hk*D], world,
    rank) with the ranks' columns in rank order.  Without an initialised
    process group it returns the inputs themselves, world 1 and rank 0."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return xq, xk, 1, 0
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    if world == 1:
        return xq, xk, 1, rank

    def gather(x):
        parts = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(parts, x.contiguous(), group=group)
        return torch.cat(parts, dim=1)

    return gather(xq), gather(xk), world, rank


def qknorm_layerwise_tp(qkv, Hq, Hk, D, gamma_q, gamma_k, eps, group=None, row_stride=None):
    """Layerwise QK-Norm across a tensor-parallel group, in place.

    Every rank of ``group`` (torch.distributed; a single process when it is
    not initialised) holds ``Hq`` query and ``Hk`` key/value heads of every
    token.  Steps: this rank's partial sums (qknorm_layerwise_partials), one
    all-reduce of the 2*T scalars over the group, and the scaling
    (qknorm_layerwise_apply) with the full vector lengths."""
    partials = qknorm_layerwise_partials(qkv, Hq, Hk, D, row_stride=row_stride)
    world = tp_allreduce_(partials, group)
    len_q, len_k = tp_full_lengths(Hq, Hk, D, world)
    return qknorm_layerwise_apply(qkv, Hq, Hk, D, gamma_q, gamma_k, partials, len_q, len_k, eps,
                                  row_stride=row_stride)


def qknorm_layerwise_tp_allgather(qkv, Hq, Hk, D, gamma_q_full, gamma_k_full, eps, group=None,
                                  row_stride=None):
    """The All-Gather baseline of tensor-parallel layerwise QK-Norm, in place:
    the standard exchange that SwiftQK's scalar all-reduce replaces.  Every
    rank of ``group`` gathers the q and k columns of all ranks (the full
    vectors of every token, (world-1)*T*(Hq+Hk)*D elements received per rank
    instead of 2*T scalars), normalises them with the full-length weights
    ``gamma_q_full`` [world*Hq*D] and ``gamma_k_full`` [world*Hk*D] in
    qknorm_layerwise, and keeps its own slice.  The result equals that of
    qknorm_layerwise_tp up to the fp32 summation order."""
    import torch

    _device_check(qkv, gamma_q_full, gamma_k_full)
    T, stride = _rows(qkv, row_stride)
    q0, k0, k1 = 0, Hq * D, (Hq + Hk) * D
    fq, fk, world, rank = tp_allgather_full(qkv[:, q0:k0], qkv[:, k0:k1], group)
    HQ, HK = world * Hq, world * Hk
    # A fused buffer of the full vectors; its V columns exist only to satisfy
    # the layout and are never read.
    full = torch.empty((T, (HQ + 2 * HK) * D), dtype=qkv.dtype, device=qkv.device)
    full[:, :HQ * D] = fq
    full[:, HQ * D:(HQ + HK) * D] = fk
    qknorm_layerwise(full, HQ, HK, D, gamma_q_full, gamma_k_full, eps)
    qkv[:, q0:k0] = full[:, rank * Hq * D:(rank + 1) * Hq * D]
    qkv[:, k0:k1] = full[:, HQ * D + rank * Hk * D:HQ * D + (rank + 1) * Hk * D]
    return qkv


# ------------------------------------------- in-kernel tensor-parallel exchange --
IPC_HANDLE_BYTES = 64


def exchange_handles(handle: bytes, group=None):
    """Every rank's IPC handle, in rank order (one all-gather of host objects
    over ``group``; just ``[handle]`` without an initialised process group)."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return [handle]
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, handle, group=group)
    return out


def _agree(ok: bool, group, what: str) -> None:
    """All-reduce (min) a success flag over ``group``; raise on every rank if
    any rank failed."""
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
    t = torch.tensor([1 if ok else 0], dtype=torch.int32, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MIN, group=group)
    if int(t.item()) == 0:
        raise RuntimeError(what)


class TPComm:
    """Communicator of ``qknorm_layerwise_tp_p2p`` (see include/qknorm.h):
    this rank's receive buffer and the other ranks' buffers mapped through
    CUDA IPC, or a whole group emulated on one device (``TPComm.local``).

    Create it on the device the rank runs on; ``close()`` (or garbage
    collection) frees it, after a barrier over the group so that no peer is
    still storing into this rank's buffer."""

    def __init__(self, ptr, world, rank, nlocal, group=None):
        self._ptr = ptr
        self.world, self.rank, self.nlocal, self.group = world, rank, nlocal, group

    @classmethod
    def local(cls, world: int, max_tokens: int, timeout_s: float = 2.0) -> "TPComm":
        """A group of ``world`` ranks on the current device, served by one
        launch per call."""
        ptr = ctypes.c_void_p()
        _check("qknorm_tp_comm_create_local", load_library().qknorm_tp_comm_create_local(
            int(world), int(max_tokens), float(timeout_s), ctypes.byref(ptr)))
        return cls(ptr, int(world), 0, int(world))

    @classmethod
    def from_group(cls, max_tokens: int, group=None, timeout_s: float = 2.0) -> "TPComm":
        """This process's rank of ``group`` (torch.distributed; one rank when it
        is not initialised): create, all-gather the IPC handles, connect."""
        import torch
        import torch.distributed as dist

        on = dist.is_available() and dist.is_initialized()
        world = dist.get_world_size(group) if on else 1
        rank = dist.get_rank(group) if on else 0
        lib = load_library()
        ptr = ctypes.c_void_p()
        handle = (ctypes.c_char * IPC_HANDLE_BYTES)()
        rc = lib.qknorm_tp_comm_create(world, rank, int(max_tokens), float(timeout_s),
                                       ctypes.byref(ptr), handle)
        if world > 1:
            # Every rank learns whether all created their buffer before any
            # collective that a failed rank would not join.
            _agree(rc == 0, group, "qknorm_tp_comm_create failed on some rank")
        _check("qknorm_tp_comm_create", rc)
        comm = cls(ptr, world, rank, 1, group)
        handles = exchange_handles(bytes(handle), group)
        if world > 1:
            torch.cuda.synchronize()
            rc = lib.qknorm_tp_comm_connect(ptr, b"".join(handles))
            _agree(rc == 0, group, "qknorm_tp_comm_connect failed on some rank")
        return comm

    def errors(self) -> int:
        """Waits of this communicator that gave up since it was created."""
        count = ctypes.c_uint(0)
        _check("qknorm_tp_comm_errors",
               load_library().qknorm_tp_comm_errors(self._ptr, ctypes.byref(count)))
        return int(count.value)

    def close(self):
        if self._ptr is None:
            return
        import torch

        torch.cuda.synchronize()
        if self.nlocal == 1 and self.world > 1:
            import torch.distributed as dist

            if dist.is_available() and dist.is_initialized():
                dist.barrier(self.group)
        load_library().qknorm_tp_comm_destroy(self._ptr)
        self._ptr = None

    def __del__(self):
        try:
            if self._ptr is not None and (self.nlocal > 1 or self.world == 1):
                load_library().qknorm_tp_comm_destroy(self._ptr)
                self._ptr = None
        except Exception:
            pass


def qknorm_layerwise_tp_p2p(comm: TPComm, qkv, Hq, Hk, D, gamma_q, gamma_k, eps, row_stride=None,
                            stream=None):
    """Tensor-parallel layerwise QK-Norm with the scalar exchange inside the
    kernel, in place.  ``qkv``, ``gamma_q`` and ``gamma_k`` are this rank's
    tensors, or lists with one entry per rank of a local communicator; each
    rank holds ``Hq`` query and ``Hk`` key/value heads of every token."""
    many = isinstance(qkv, (list, tuple))
    xs = list(qkv) if many else [qkv]
    gqs = list(gamma_q) if many else [gamma_q]
    gks = list(gamma_k) if many else [gamma_k]
    if not (len(xs) == len(gqs) == len(gks) == comm.nlocal):
        raise ValueError("pass one qkv / gamma_q / gamma_k per rank the communicator serves (%d)"
                         % comm.nlocal)
    T, stride = None, None
    for x, gq, gk in zip(xs, gqs, gks):
        _device_check(x, gq, gk)
        t, st = _rows(x, row_stride)
        if (T, stride) not in ((None, None), (t, st)):
            raise ValueError("every rank's buffer must have the same shape")
        T, stride = t, st
    vp = ctypes.c_void_p
    arr_x = (vp * comm.nlocal)(*[x.data_ptr() for x in xs])
    arr_q = (vp * comm.nlocal)(*[_gamma_ptr(g, "gamma_q") for g in gqs])
    arr_k = (vp * comm.nlocal)(*[_gamma_ptr(g, "gamma_k") for g in gks])
    rc = load_library().qknorm_layerwise_tp_p2p(
        comm._ptr, arr_x, _dtype_code(xs[0]), T, Hq, Hk, D, stride, arr_q, arr_k, float(eps),
        _stream_ptr(xs[0], stream))
    _check("qknorm_layerwise_tp_p2p", rc)
    return qkv
