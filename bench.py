#!/usr/bin/env python
"""Benchmark of QK-Norm on B200: tokens/s and achieved HBM GB/s against T.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one call of the hot path over one batch: per-head QK-Norm of the
head_dim-128, 48-head, T=4096 bf16 workload (the shape of the sglang /
turbomind kernel table's largest row), in place, through the C ABI.  Steps
rotate over enough copies of the input that the set is more than four times
the L2 cache, so every step reads from HBM.  The K timed steps are replayed
from CUDA graphs of up to 100 steps, the first opening with the start event
and the last closing with the end event (event nodes inside the graphs, on
the launching stream); a barrier plus device synchronisation stands on both
sides of the timed region, and the time is the max over ranks.

Rank 0 prints one JSON line.  Besides the headline it carries the roofline
of the kernel, an end-to-end figure through host buffers, the CPU oracle as
a reported baseline, SM clocks sampled during the timed region, and a sweep
over T and over the other workloads (GQA fused layout, layerwise with 1..8
emulated shards, fp32 / head_dim 64..256 stress shapes).

With N > 1 (``--gpus N``, started here under torch.distributed.run when no
launcher set WORLD_SIZE, or under the caller's torchrun) every rank runs the
same per-GPU workload on its own GPU (weak scaling: tokens are independent,
so no collective touches the data; NCCL carries only the barrier and the max
of the timings).  The line's ``tp`` entry times tensor-parallel layerwise
QK-Norm with the layerwise workload's heads split over the N ranks: the
scalar all-reduce exchange against the All-Gather baseline, per layer call.
``--dry-run`` runs only the launch and the cross-rank steps, without a GPU.

``--impl reference`` times the float64 CPU oracle on the host cores instead
(rank 0 only), on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QK-Norm tokens/s and achieved HBM GB/s (fraction of B200 peak) vs T"
UNIT = "tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
GRAPH_STEPS = 100

HEADLINE = dict(kind="per_head", T=4096, Hq=48, Hk=0, D=128, dtype="bf16", eps=1e-6, nshards=1,
                seed=1001)
HEADLINE_NAME = ("per-head QK-Norm, head_dim 128, 48 heads, T=4096 tokens, bf16, Q-style "
                 "contiguous [T,48,128] (shape of the largest row of the sglang/turbomind "
                 "kernel table)")


# ---------------------------------------------------------------- helpers --
ELEM_BYTES = {"bf16": 2, "fp16": 2, "fp32": 4, "fp8_e4m3": 1}


def workload_bytes(w) -> int:
    """Algorithmic bytes of one call: read + write of Q and K once, gamma once."""
    es = ELEM_BYTES[w["dtype"]]
    qk = (w["Hq"] + w["Hk"]) * w["D"]
    if w["kind"] == "per_head":
        gamma = w["D"] * 4 * ((w["Hq"] > 0) + (w["Hk"] > 0))
    else:
        gamma = qk * 4
    return 2 * w["T"] * qk * es + gamma


def row_stride(w) -> int:
    return (w["Hq"] + 2 * w["Hk"]) * w["D"]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def traffic_record():
    """Committed ncu DRAM bytes per launch, valid only for the kernel sources
    they were taken from (buildlib.kernel_source_sha256)."""
    from attention_qk_norm_b200 import buildlib

    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        return rec if rec.get("source_sha256") == buildlib.kernel_source_sha256() else None
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.out = None

    def start(self, settle_s: float = 0.3):
        """Start sampling; returns at once, and ``settle_s`` seconds are left
        for nvidia-smi to come up (the caller keeps the GPU busy meanwhile)."""
        self.ready_at = time.perf_counter() + settle_s
        try:
            self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(max(0.15, self.ready_at - time.perf_counter()))
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.flush()
        with open(self.out.name) as f:
            rows = [r.split(",") for r in f.read().strip().splitlines() if r.strip()]
        os.unlink(self.out.name)
        rows = [[c.strip() for c in r] for r in rows if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            for name, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


def host_threads() -> int:
    """Host cores this process may run on (a launcher's OMP_NUM_THREADS=1 per
    rank does not shrink the CPU baseline)."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------- distributed --
def dist_init(use_gpu: bool = True):
    """Join the process group of a torchrun launch (NCCL with a GPU per rank,
    gloo on CPU); returns (rank, world size, local rank)."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        backend = "nccl" if use_gpu and torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local) if backend == "nccl" else None)
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def shard_units(total: int, world: int, rank: int):
    """Contiguous split of ``total`` independent units over ranks (for runs
    that divide one fixed job; the benchmark itself runs weak scaling)."""
    base, rem = divmod(total, world)
    start = rank * base + min(rank, rem)
    return start, start + base + (1 if rank < rem else 0)


# ---------------------------------------------------------------- GPU side --
class Workload:
    """Device buffers of one workload, rotated so their total exceeds 4x L2."""

    def __init__(self, w, device, l2_bytes, max_bytes=16 << 30):
        import torch
        from attention_qk_norm_b200 import synth

        self.w = w
        d = synth.make_case_torch(w["T"], w["Hq"], w["Hk"], w["D"], device=device,
                                  dtype=w["dtype"], seed=w["seed"], eps=w["eps"],
                                  layerwise=w["kind"] != "per_head",
                                  scale=w.get("scale"), zero_frac=w.get("zero_frac", 0.0),
                                  outlier_frac=w.get("outlier_frac", 0.0))
        self.gq, self.gk = d["gamma_q"], d["gamma_k"]
        one = d["qkv"].numel() * d["qkv"].element_size()
        n = max(2, math.ceil(4 * l2_bytes / max(1, one)))
        n = max(1, min(n, max_bytes // max(1, one)))
        self.bufs = [d["qkv"]] + [d["qkv"].clone() for _ in range(n - 1)]
        self.buffer_bytes = one
        self.host_in = None
        self.i = 0
        torch.cuda.synchronize()

    def launch(self, buf=None):
        import attention_qk_norm_b200 as qkn

        w = self.w
        if buf is None:
            buf = self.bufs[self.i % len(self.bufs)]
            self.i += 1
        if w["kind"] == "per_head":
            qkn.qknorm_per_head(buf, w["Hq"], w["Hk"], w["D"], self.gq, self.gk, w["eps"])
        elif w["kind"] == "layerwise_tp":
            # The two rank-local tensor-parallel steps of one rank (no peers,
            # so the all-reduce between them is empty).
            if getattr(self, "partials", None) is None:
                import torch

                self.partials = torch.empty((w["T"], 2), dtype=torch.float32, device=buf.device)
            qkn.qknorm_layerwise_partials(buf, w["Hq"], w["Hk"], w["D"], partials=self.partials)
            qkn.qknorm_layerwise_apply(buf, w["Hq"], w["Hk"], w["D"], self.gq, self.gk,
                                       self.partials, w["Hq"] * w["D"], w["Hk"] * w["D"], w["eps"])
        else:
            qkn.qknorm_layerwise(buf, w["Hq"], w["Hk"], w["D"], self.gq, self.gk, w["eps"],
                                 nshards=w["nshards"])

    def graph(self, steps: int):
        import torch

        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(steps):
                self.launch()
        return g

    def free(self):
        self.bufs = []


def time_graph_us(wl, reps=5, min_ms=20.0):
    """Median per-launch time (µs) over `reps` timed groups of graph replays."""
    import torch

    g = wl.graph(GRAPH_STEPS)
    g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    g.replay()
    e.record()
    e.synchronize()
    per = max(s.elapsed_time(e), 1e-3)
    n = max(1, int(math.ceil(min_ms / per)))
    samples = []
    for _ in range(reps):
        s.record()
        for _ in range(n):
            g.replay()
        e.record()
        e.synchronize()
        samples.append(s.elapsed_time(e) * 1e3 / (n * GRAPH_STEPS))
    del g
    return statistics.median(samples)


def point(w, us, hbm_peak):
    b = workload_bytes(w)
    gbs = b / (us * 1e-6) / 1e9
    return {"T": w["T"], "us": round(us, 3), "tokens_per_s": round(w["T"] / (us * 1e-6), 1),
            "gbs": round(gbs, 1), "frac_measured": round(gbs / hbm_peak, 4),
            "frac_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 4), "bytes": b}


def extra_workloads():
    from attention_qk_norm_b200 import synth

    out = []
    for T in synth.SWEEP_T:
        out.append(("sweep H=48", dict(HEADLINE, T=T, seed=2000 + T)))
    for H in (16, 32):
        out.append(("sweep H=%d" % H, dict(HEADLINE, Hq=H, T=4096, seed=2100 + H)))
    for T in synth.GQA_T:
        out.append(("gqa fused 32q/8kv", dict(kind="per_head", T=T, Hq=32, Hk=8, D=128,
                                              dtype="bf16", eps=1e-6, nshards=1,
                                              scale="lognormal", seed=2200 + T)))
    for n in synth.LAYERWISE_NSHARDS:
        for T in synth.LAYERWISE_T:
            out.append(("layerwise n=%d" % n, dict(kind="layerwise", T=T, Hq=32, Hk=8, D=128,
                                                    dtype="bf16", eps=1e-6, nshards=n,
                                                    seed=2300 + T)))
    for T in (4096, 8192):
        out.append(("layerwise tp steps, 1 rank", dict(kind="layerwise_tp", T=T, Hq=32, Hk=8,
                                                       D=128, dtype="bf16", eps=1e-6, nshards=1,
                                                       seed=2700 + T)))
    for dt in (synth.FP16, synth.FP8):
        out.append(("gqa fused 32q/8kv %s" % dt, dict(kind="per_head", T=16384, Hq=32, Hk=8,
                                                      D=128, dtype=dt, eps=1e-6, nshards=1,
                                                      scale="lognormal", seed=2500)))
        out.append(("layerwise n=8 %s" % dt, dict(kind="layerwise", T=8192, Hq=32, Hk=8, D=128,
                                                  dtype=dt, eps=1e-6, nshards=8, seed=2600)))
    for dt in synth.STRESS_DTYPES:
        for D in synth.STRESS_D:
            for kind in ("per_head", "layerwise"):
                out.append(("stress %s %s D=%d" % (kind, dt, D),
                            dict(kind=kind, T=32768, Hq=64, Hk=8, D=D, dtype=dt, eps=1e-6,
                                 nshards=8 if kind == "layerwise" else 1, scale="stress",
                                 zero_frac=0.01, outlier_frac=0.01, seed=2400 + D)))
    return out


def run_extras(device, l2, hbm_peak):
    import torch

    res = []
    for name, w in extra_workloads():
        wl = Workload(w, device, l2, max_bytes=8 << 30)
        for _ in range(3):
            wl.launch()
        us = time_graph_us(wl)
        p = point(w, us, hbm_peak)
        p["workload"] = name
        res.append(p)
        wl.free()
        del wl
        torch.cuda.empty_cache()
    return res


# The layerwise workload's heads (32 query, 8 key/value, head_dim 128, bf16),
# split by head over the ranks of a tensor-parallel group.
TP_GLOBAL = dict(Hq=32, Hk=8, D=128, dtype="bf16", eps=1e-6)


def time_eager_us(fn, bufs, world, iters=50, warm=5):
    """Mean µs per call of ``fn(buf)`` over ``iters`` calls launched eagerly
    (no graph: the calls hold collectives), rotating ``bufs``; CUDA events on
    the current stream, max over ranks."""
    import torch

    for i in range(warm):
        fn(bufs[i % len(bufs)])
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(iters):
        fn(bufs[i % len(bufs)])
    e.record()
    torch.cuda.synchronize()
    return max_over_ranks(s.elapsed_time(e) * 1e3 / iters, world)


def run_tp(device, l2, world, rank, T_list=(1, 16, 256, 4096, 8192)):
    """Tensor-parallel layerwise QK-Norm, the layerwise workload's heads split
    over the ``world`` ranks: per layer call, the scalar exchange
    (``qknorm_layerwise_tp``: partials, one all-reduce of 2T floats, scaling)
    against the All-Gather baseline (``qknorm_layerwise_tp_allgather``)."""
    import torch
    import attention_qk_norm_b200 as qkn
    from attention_qk_norm_b200 import synth

    G = TP_GLOBAL
    if G["Hq"] % world or G["Hk"] % world:
        return {"world": world, "skipped": "the group size must divide 32 query and 8 key heads"}
    hq, hk, D, eps = G["Hq"] // world, G["Hk"] // world, G["D"], G["eps"]
    gen = torch.Generator(device=device)
    gen.manual_seed(2900)  # the same full-length weights on every rank
    gq_full = 1.0 + 0.1 * torch.randn(G["Hq"] * D, generator=gen, device=device)
    gk_full = 1.0 + 0.1 * torch.randn(G["Hk"] * D, generator=gen, device=device)
    gq = gq_full[rank * hq * D:(rank + 1) * hq * D].contiguous()
    gk = gk_full[rank * hk * D:(rank + 1) * hk * D].contiguous()
    # The in-kernel exchange over the same group (peer stores through CUDA
    # IPC); any failure is reported, not raised, so the line still prints.
    comm, p2p_error = None, None
    try:
        comm = qkn.TPComm.from_group(max_tokens=max(T_list), timeout_s=10.0)
    except Exception as ex:  # every rank raises together (TPComm.from_group)
        p2p_error = str(ex)[:200]
    points = []
    for T in T_list:
        d = synth.make_case_torch(T, hq, hk, D, device=device, layerwise=True,
                                  seed=2800 + T + 31 * rank)
        one = d["qkv"].numel() * d["qkv"].element_size()
        n = max(2, min(64, math.ceil(4 * l2 / max(1, one))))
        bufs = [d["qkv"]] + [d["qkv"].clone() for _ in range(n - 1)]
        ar = time_eager_us(lambda b: qkn.qknorm_layerwise_tp(b, hq, hk, D, gq, gk, eps), bufs,
                           world)
        ag = time_eager_us(lambda b: qkn.qknorm_layerwise_tp_allgather(b, hq, hk, D, gq_full,
                                                                       gk_full, eps),
                           bufs, world)
        pt = {"T": T, "scalar_allreduce_us": round(ar, 3), "allgather_us": round(ag, 3),
              "allreduce_vs_allgather": round(ar / ag, 4)}
        if comm is not None:
            p2p = time_eager_us(
                lambda b: qkn.qknorm_layerwise_tp_p2p(comm, b, hq, hk, D, gq, gk, eps), bufs,
                world)
            pt["in_kernel_p2p_us"] = round(p2p, 3)
            pt["p2p_vs_allgather"] = round(p2p / ag, 4)
            # The same calls replayed from a CUDA graph (no collective library
            # on this path, so it captures): the device time of a layer call.
            barrier(world)
            p2p_g = time_graph_fn_us(
                lambda i: qkn.qknorm_layerwise_tp_p2p(comm, bufs[i], hq, hk, D, gq, gk, eps),
                len(bufs))
            pt["in_kernel_p2p_graph_us"] = round(max_over_ranks(p2p_g, world), 3)
        points.append(pt)
        del bufs, d
        torch.cuda.empty_cache()
    out = {"world": world, "heads_per_rank": {"q": hq, "kv": hk}, "head_dim": D,
           "dtype": G["dtype"],
           "workload": "layerwise QK-Norm of 32 query / 8 key heads x 128 split by head over "
                       "%d rank(s), one layer call per step" % world,
           "timing": "eager calls through the Python binding (the exchanges hold NCCL "
                     "collectives), CUDA events, mean of 50, max over ranks; the in-kernel "
                     "exchange also from CUDA graphs of 50 calls (median of 5 replays)",
           "points": points}
    if comm is not None:
        torch.cuda.synchronize()
        out["in_kernel_p2p_waits_given_up"] = int(max_over_ranks(float(comm.errors()), world))
        comm.close()
    else:
        out["in_kernel_p2p_error"] = p2p_error
    out["emulated_group"] = run_tp_emulated(device, l2, world)
    return out


def run_tp_emulated(device, l2, world, ranks=8, T_list=(1, 16, 256, 4096, 8192)):
    """An 8-rank group emulated on this GPU: every rank's buffer and receive
    buffer here, all ranks served by one cooperative launch of the in-kernel
    exchange, against the fused single-GPU kernel with nshards = 8 over the
    whole vectors (no exchange at all).  Graphs of 50 launches, CUDA events,
    max over ranks."""
    import torch
    import attention_qk_norm_b200 as qkn
    from attention_qk_norm_b200 import synth

    G = TP_GLOBAL
    hq, hk, D, eps = G["Hq"] // ranks, G["Hk"] // ranks, G["D"], G["eps"]
    comm = qkn.TPComm.local(ranks, max_tokens=max(T_list), timeout_s=10.0)
    points = []
    for T in T_list:
        d = synth.make_case_torch(T, G["Hq"], G["Hk"], D, device=device, layerwise=True,
                                  seed=3100 + T)
        W = (hq + 2 * hk) * D
        one = d["qkv"].numel() * d["qkv"].element_size()
        n = max(2, min(32, math.ceil(4 * l2 / max(1, one))))
        full = [d["qkv"].clone() for _ in range(n)]
        parts = [[d["qkv"][:, :W].clone() for _ in range(ranks)] for _ in range(n)]
        gqs = [d["gamma_q"][r * hq * D:(r + 1) * hq * D].contiguous() for r in range(ranks)]
        gks = [d["gamma_k"][r * hk * D:(r + 1) * hk * D].contiguous() for r in range(ranks)]
        p2p = time_graph_fn_us(
            lambda i: qkn.qknorm_layerwise_tp_p2p(comm, parts[i], hq, hk, D, gqs, gks, eps), n)
        fused = time_graph_fn_us(
            lambda i: qkn.qknorm_layerwise(full[i], G["Hq"], G["Hk"], D, d["gamma_q"],
                                           d["gamma_k"], eps, nshards=ranks), n)
        points.append({"T": T, "in_kernel_p2p_group_us": round(max_over_ranks(p2p, world), 3),
                       "fused_nshards8_us": round(max_over_ranks(fused, world), 3)})
        del full, parts, d
        torch.cuda.empty_cache()
    torch.cuda.synchronize()
    errors = comm.errors()
    comm.close()
    return {"ranks": ranks, "heads_per_rank": {"q": hq, "kv": hk}, "waits_given_up": errors,
            "points": points}


def time_graph_fn_us(fn, nbufs, steps=50, reps=5):
    """Median µs per call of ``fn(i)`` (i rotating over ``nbufs`` buffers)
    replayed from a CUDA graph of ``steps`` calls."""
    import torch

    i = [0]

    def launch():
        fn(i[0] % nbufs)
        i[0] += 1

    for _ in range(3):
        launch()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(steps):
            launch()
    g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    out = []
    for _ in range(reps):
        s.record()
        g.replay()
        e.record()
        e.synchronize()
        out.append(s.elapsed_time(e) * 1e3 / steps)
    del g
    return statistics.median(out)


def e2e(w, device, steps, lanes=2):
    """Same metric through host buffers: per step a pinned-host -> device copy
    of the input, the C-ABI call, and a device -> pinned-host copy of the
    normalised buffer, all inside the timed region.  Steps alternate over
    `lanes` streams, each with its own device and host output buffer, so the
    upload of one step overlaps the download of the previous one (the host
    link is full duplex); within a lane the three operations stay ordered."""
    import torch
    from attention_qk_norm_b200 import synth

    d = synth.make_case_torch(w["T"], w["Hq"], w["Hk"], w["D"], device="cpu", dtype=w["dtype"],
                              seed=w["seed"], eps=w["eps"])
    host_in = d["qkv"].pin_memory()
    host_out = [torch.empty_like(host_in).pin_memory() for _ in range(lanes)]
    devs = [torch.empty_like(host_in, device=device) for _ in range(lanes)]
    streams = [torch.cuda.Stream(device) for _ in range(lanes)]
    gq = d["gamma_q"].to(device)
    wl = Workload.__new__(Workload)
    wl.w, wl.gq, wl.gk = w, gq, None
    main = torch.cuda.current_stream(device)

    def run(n, start_event):
        for st in streams:
            st.wait_event(start_event)
        for i in range(n):
            k = i % lanes
            with torch.cuda.stream(streams[k]):
                devs[k].copy_(host_in, non_blocking=True)
                wl.launch(devs[k])
                host_out[k].copy_(devs[k], non_blocking=True)
        for st in streams:
            done = torch.cuda.Event()
            done.record(st)
            main.wait_event(done)

    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(main)
    run(3, s)
    torch.cuda.synchronize()
    s.record(main)
    run(steps, s)
    e.record(main)
    e.synchronize()
    ms = s.elapsed_time(e)
    nbytes = host_in.numel() * host_in.element_size()
    return ms, nbytes


def cpu_baseline(w, budget_s=10.0):
    """The float64 oracle on the host cores, over whole copies of the
    workload's input, for about `budget_s` seconds (at least one pass)."""
    import oracle
    from attention_qk_norm_b200 import synth

    c = synth.make_case(w["T"], w["Hq"], w["Hk"], w["D"], dtype=w["dtype"], seed=w["seed"],
                        eps=w["eps"])
    threads = host_threads()
    t0 = time.perf_counter()
    passes = 0
    while True:
        oracle.per_head(c.qkv, c.dtype, c.T, c.Hq, c.Hk, c.D, c.row_stride, c.gamma_q,
                        c.gamma_k, c.eps, nthreads=threads)
        passes += 1
        el = time.perf_counter() - t0
        if el >= budget_s or (passes >= 1 and el * (passes + 1) / passes > 3 * budget_s):
            break
    # One host thread, on the first tokens only (bounded to a second or two).
    n1 = min(c.T, 1024)
    t1 = time.perf_counter()
    oracle.per_head(c.qkv[:n1], c.dtype, n1, c.Hq, c.Hk, c.D, c.row_stride, c.gamma_q, c.gamma_k,
                    c.eps, nthreads=1)
    el1 = time.perf_counter() - t1
    return {"value": round(passes * c.T / el, 1), "unit": UNIT, "cores": threads,
            "kind": "oracle",
            "sample": "%d full pass(es) of the %d-token workload (%.1f s)" % (passes, c.T, el),
            "value_1_thread": round(n1 / el1, 1),
            "sample_1_thread": "the first %d tokens on one host thread (%.2f s)" % (n1, el1)}


# -------------------------------------------------------------- main arms --
def run_ours(args):
    import torch

    rank, world, local = dist_init()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    props = torch.cuda.get_device_properties(device)
    l2 = int(getattr(props, "L2_cache_size", 126 << 20))
    hbm_peak, peak_kind = peaks()
    w = dict(HEADLINE)
    wl = Workload(w, device, l2)
    # The K timed steps as graphs of up to GRAPH_STEPS launches: the first
    # graph opens with the start event and the last one closes with the end
    # event (event nodes inside the graphs), so the timed region is the K
    # launches on the device, without the host's graph-launch latency.
    s = torch.cuda.Event(enable_timing=True, external=True)
    e = torch.cuda.Event(enable_timing=True, external=True)
    sizes = [GRAPH_STEPS] * (args.steps // GRAPH_STEPS)
    if args.steps % GRAPH_STEPS:
        sizes.append(args.steps % GRAPH_STEPS)
    timed = []  # (graph, replays)
    for j, n in enumerate(sizes):
        first, last = j == 0, j == len(sizes) - 1
        if not first and not last and timed and timed[-1][2]:
            timed[-1][1] += 1  # another replay of the plain middle graph
            continue
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            if first:
                s.record()
            for _ in range(n):
                wl.launch()
            if last:
                e.record()
        timed.append([g, 1, not first and not last])
    # Replay every graph once: a graph's first replay uploads it to the
    # device, which must not land inside the timed region.
    for g, _, _ in timed:
        g.replay()
    torch.cuda.synchronize()

    # The clock sampler starts first; while it comes up the GPU replays a
    # warm-up graph (untimed), so that it does not idle, and drop its clocks,
    # right before the timed region.  Then the W warm-up steps.
    sampler = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[0])
                           if world == 1 else local)
    g_warm = wl.graph(GRAPH_STEPS)
    if rank == 0:
        sampler.start()
    settle_until = time.perf_counter() + 0.3
    while time.perf_counter() < settle_until:
        g_warm.replay()
        torch.cuda.synchronize()
    del g_warm
    barrier(world)
    for _ in range(args.warmup):
        wl.launch()
    barrier(world)
    torch.cuda.synchronize()
    for g, replays, _ in timed:
        for _ in range(replays):
            g.replay()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if rank == 0 else None
    ms_local = s.elapsed_time(e)
    ms = max_over_ranks(ms_local, world)
    del timed

    steps = args.steps
    tokens = w["T"] * steps * world
    value = tokens / (ms * 1e-3)
    per_launch_us = ms_local * 1e3 / steps
    b = workload_bytes(w)
    achieved = b / (per_launch_us * 1e-6) / 1e9
    tr = traffic_record()

    e2e_ms, e2e_bytes = e2e(w, device, args.e2e_steps)
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e_val = w["T"] * args.e2e_steps * world / (e2e_ms * 1e-3)

    l2_note = ("rotating %d in-place buffers of %.1f MB (%.0f MB > 4x L2 %.0f MB)"
               % (len(wl.bufs), wl.buffer_bytes / 1e6, wl.buffer_bytes * len(wl.bufs) / 1e6,
                  l2 / 1e6))
    extras = tp = None
    if not args.no_extras:
        wl.free()
        torch.cuda.empty_cache()
        extras = run_extras(device, l2, hbm_peak)
        tp = run_tp(device, l2, world, rank)
    barrier(world)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms / steps, 6),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": HEADLINE_NAME, "T": w["T"], "heads": w["Hq"],
                       "head_dim": w["D"], "kernel": "qknorm_per_head",
                       "l2": l2_note,
                       "launch": "CUDA graphs of %d launches" % GRAPH_STEPS,
                       "parallelism": "dp%d (tokens independent, no collective)" % world},
            "gpu_launches": steps,
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1),
                         "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(achieved / hbm_peak, 4),
                         "peak_kind": peak_kind,
                         "frac_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
                         "algorithmic_bytes_per_launch": b,
                         "traffic": tr["dram_bytes_per_launch"] if tr else None},
            "e2e": {"value": round(e2e_val, 1), "unit": UNIT,
                    "h2d_bytes_per_step": e2e_bytes, "d2h_bytes_per_step": e2e_bytes,
                    "steps": args.e2e_steps, "streams": 2},
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, args.cpu_budget)
        if extras is not None:
            line["sweep"] = extras
        if tp is not None:
            line["tp"] = tp
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def run_reference(args):
    """The float64 CPU oracle on the workload's tokens, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle
    from attention_qk_norm_b200 import synth

    w = HEADLINE
    c = synth.make_case(w["T"], w["Hq"], w["Hk"], w["D"], dtype=w["dtype"], seed=w["seed"],
                        eps=w["eps"])
    threads = host_threads()

    def step(n_tok, start):
        rows = [(start + i) % c.T for i in range(n_tok)]
        x = c.qkv[rows]
        oracle.per_head(x, c.dtype, n_tok, c.Hq, c.Hk, c.D, c.row_stride, c.gamma_q, c.gamma_k,
                        c.eps, nthreads=threads)

    t0 = time.perf_counter()
    step(256, 0)
    per_tok = (time.perf_counter() - t0) / 256
    budget = 120.0  # seconds for warm-up plus timed steps
    n_tok = int(max(1, min(c.T, budget / max(1, args.steps + args.warmup) / max(per_tok, 1e-9))))
    for i in range(args.warmup):
        step(n_tok, i * n_tok)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(n_tok, (args.warmup + i) * n_tok)
    el = time.perf_counter() - t0
    value = args.steps * n_tok / el
    sample = ("%d of the %d tokens per step (float64 oracle, %d threads)"
              % (n_tok, c.T, threads))
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": HEADLINE_NAME, "T": w["T"], "heads": w["Hq"],
                       "head_dim": w["D"]},
            "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


PROFILE_CASES = {
    "per_head": dict(HEADLINE),
    "per_head_h16": dict(HEADLINE, Hq=16),
    "per_head_h32": dict(HEADLINE, Hq=32),
    "gqa": dict(kind="per_head", T=16384, Hq=32, Hk=8, D=128, dtype="bf16", eps=1e-6, nshards=1,
                scale="lognormal", seed=1002),
    "layerwise": dict(kind="layerwise", T=8192, Hq=32, Hk=8, D=128, dtype="bf16", eps=1e-6,
                      nshards=8, seed=1003),
    "per_head_fp8": dict(kind="per_head", T=32768, Hq=32, Hk=8, D=128, dtype="fp8_e4m3",
                         eps=1e-6, nshards=1, scale="lognormal", seed=1002),
    "layerwise_wide": dict(kind="layerwise", T=8192, Hq=64, Hk=8, D=128, dtype="bf16", eps=1e-6,
                           nshards=8, scale="stress", zero_frac=0.01, outlier_frac=0.01,
                           seed=1004),
    "layerwise_fp8": dict(kind="layerwise", T=32768, Hq=32, Hk=8, D=128, dtype="fp8_e4m3",
                          eps=1e-6, nshards=8, seed=1006),
    # The in-kernel tensor-parallel exchange, an 8-rank group emulated on one
    # GPU (one cooperative launch serves all ranks).
    "tp_group": dict(kind="tp_group", T=4096, Hq=32, Hk=8, D=128, dtype="bf16", eps=1e-6,
                     nshards=8, seed=1007),
    # One rank holding every head: the exchange kernel as a rank on its own
    # GPU launches it (programmatic dependent launch, not cooperative).
    "tp_rank": dict(kind="tp_group", T=8192, Hq=32, Hk=8, D=128, dtype="bf16", eps=1e-6,
                    nshards=1, seed=1008),
    # 128 heads of 256: too wide for one block, so 2-block clusters exchange
    # head partials through distributed shared memory.
    "layerwise_cluster": dict(kind="layerwise", T=4096, Hq=112, Hk=16, D=256, dtype="bf16",
                              eps=1e-6, nshards=8, scale="stress", zero_frac=0.01,
                              outlier_frac=0.01, seed=1005),
}


def run_profile(args):
    """A few plain launches of one workload, for a profiler to capture: no
    graphs, no timing, no sweep.  ``--profile-T`` overrides the token count.
    Launches rotate over copies of the input totalling more than 4x L2, as in
    the timed runs, so a capture without cache flushes sees steady-state DRAM
    traffic."""
    import torch

    w = dict(PROFILE_CASES[args.profile])
    if args.profile_T:
        w["T"] = args.profile_T
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    props = torch.cuda.get_device_properties(device)
    if w["kind"] == "tp_group":
        import attention_qk_norm_b200 as qkn
        from attention_qk_norm_b200 import synth

        n = w["nshards"]
        hq, hk, D = w["Hq"] // n, w["Hk"] // n, w["D"]
        d = synth.make_case_torch(w["T"], w["Hq"], w["Hk"], D, device=device, layerwise=True,
                                  seed=w["seed"])
        W = (hq + 2 * hk) * D
        reps = max(2, math.ceil(4 * props.L2_cache_size / (d["qkv"].numel() * 2)))
        parts = [[d["qkv"][:, :W].clone() for _ in range(n)] for _ in range(reps)]
        gqs = [d["gamma_q"][r * hq * D:(r + 1) * hq * D].contiguous() for r in range(n)]
        gks = [d["gamma_k"][r * hk * D:(r + 1) * hk * D].contiguous() for r in range(n)]
        comm = qkn.TPComm.local(n, max_tokens=w["T"])
        for i in range(args.warmup + args.steps):
            qkn.qknorm_layerwise_tp_p2p(comm, parts[i % reps], hq, hk, D, gqs, gks, w["eps"])
        torch.cuda.synchronize()
        comm.close()
        print(json.dumps({"profile": args.profile, "T": w["T"], "ranks": n,
                          "launches": args.warmup + args.steps,
                          "bytes_per_launch": workload_bytes(dict(w, kind="layerwise"))}))
        return
    wl = Workload(w, device, l2_bytes=int(getattr(props, "L2_cache_size", 126 << 20)),
                  max_bytes=4 << 30)
    for _ in range(args.warmup + args.steps):
        wl.launch()
    torch.cuda.synchronize()
    print(json.dumps({"profile": args.profile, "T": w["T"], "launches": args.warmup + args.steps,
                      "bytes_per_launch": workload_bytes(w)}))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-extras", action="store_true", help="skip the T / workload sweep")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=sorted(PROFILE_CASES),
                    help="only launch one workload's kernel (for ncu captures)")
    ap.add_argument("--profile-T", type=int, default=0)
    ap.add_argument("--dry-run", action="store_true",
                    help="check the rank launch and the cross-rank timing steps (barrier, max "
                         "over ranks) without touching a GPU; rank 0 prints one JSON line")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    if args.steps < 1:
        ap.error("--steps must be >= 1")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is not None and int(env_world) != args.gpus:
        ap.error("--gpus %d disagrees with WORLD_SIZE=%s set by the launcher"
                 % (args.gpus, env_world))
    if env_world is None and args.gpus > 1:
        # One process per GPU: start the N ranks here under torch.distributed.run.
        if not args.dry_run:
            import torch

            have = torch.cuda.device_count()
            if have < args.gpus:
                ap.error("--gpus %d but only %d CUDA device(s) visible" % (args.gpus, have))
        return self_launch(args.gpus, sys.argv[1:] if argv is None else list(argv))
    if args.dry_run:
        run_dry(args)
    elif args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)
    return 0


def free_port() -> int:
    import socket

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def self_launch(n: int, argv) -> int:
    """Run this script as ``n`` ranks on this node under torch.distributed.run
    (rendezvous on 127.0.0.1) with the same arguments; returns its exit code."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", str(n), "--master-addr", "127.0.0.1",
           "--master-port", str(free_port()), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def run_dry(args):
    """The launch and cross-rank steps of a run, with no GPU work: every rank
    joins the process group (gloo without CUDA), counts the ranks with a sum,
    meets at the barrier and takes the max over ranks of a per-rank figure."""
    rank, world, _ = dist_init(use_gpu=False)
    count = world
    if world > 1:
        import torch
        import torch.distributed as dist

        t = torch.ones(1, dtype=torch.float64)
        dist.all_reduce(t)
        count = int(t.item())
    barrier(world)
    ms = max_over_ranks(1.0 + rank, world)
    barrier(world)
    if rank == 0:
        print(json.dumps({"dry_run": True, "impl": args.impl, "n_gpus": world,
                          "ranks_counted": count, "max_over_ranks": ms, "steps": args.steps,
                          "warmup": args.warmup}), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
