"""QK-Norm on NVIDIA B200: per-head and layerwise (SwiftQK) RMSNorm of Q/K.

The compute lives in ``libqknorm.so`` (hand-written CUDA for sm_100a, C ABI
in ``include/qknorm.h``).  This package holds its build script, a thin
ctypes binding with the same entry-point names, and ``synth`` (seeded
synthetic inputs).  The library is loaded on first use, so importing the
package, or ``synth`` alone, needs neither the library nor a GPU.
"""
from ._binding import (  # noqa: F401
    QKN_BF16,
    QKN_FP8_E4M3,
    QKN_FP16,
    QKN_FP32,
    QKNormError,
    TPComm,
    exchange_handles,
    load_library,
    qknorm_layerwise,
    qknorm_layerwise_apply,
    qknorm_layerwise_partials,
    qknorm_layerwise_tp,
    qknorm_layerwise_tp_allgather,
    qknorm_layerwise_tp_p2p,
    qknorm_per_head,
    tp_allgather_full,
    tp_allreduce_,
    tp_full_lengths,
    status_string,
    wait_timeouts,
)
from .buildlib import LIB_PATH, build  # noqa: F401
