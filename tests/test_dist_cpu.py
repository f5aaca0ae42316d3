"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

QK-Norm tokens are independent, so ranks need no collective on the data
path; the only cross-rank steps are the barrier around the timed region
and the max over ranks of the elapsed time.  These run here as gloo ranks.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    r, w, _ = bench.dist_init()
    assert (r, w) == (rank, world) and dist.get_backend() == "gloo"
    bench.barrier(w)
    local_ms = 10.0 + 5.0 * rank
    got = bench.max_over_ranks(local_ms, w)
    lo, hi = bench.shard_units(1001, w, r)
    q.put((rank, got, lo, hi))
    bench.barrier(w)
    dist.destroy_process_group()


def _tp_worker(rank, world, port, q):
    """Each rank sums squares over its head shard of the same tokens; one
    all-reduce must give the full-vector sums, and the full lengths must be
    the local ones times the group size."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import numpy as np
    import torch
    import torch.distributed as dist

    import attention_qk_norm_b200 as qkn

    dist.init_process_group("gloo", rank=rank, world_size=world)
    T, Hq, Hk, D = 5, 8, 4, 16
    rng = np.random.default_rng(0)
    x = rng.standard_normal((T, (Hq + Hk) * D))
    xq, xk = x[:, :Hq * D], x[:, Hq * D:]
    hq, hk = Hq // world, Hk // world
    mine_q = xq[:, rank * hq * D:(rank + 1) * hq * D]
    mine_k = xk[:, rank * hk * D:(rank + 1) * hk * D]
    partials = torch.tensor(np.stack([(mine_q ** 2).sum(1), (mine_k ** 2).sum(1)], 1))
    got = qkn.tp_allreduce_(partials)
    full = np.stack([(xq ** 2).sum(1), (xk ** 2).sum(1)], 1)
    q.put((rank, got, bool(np.allclose(partials.numpy(), full, rtol=1e-12)),
           qkn.tp_full_lengths(hq, hk, D, got)))
    dist.destroy_process_group()


def _allgather_worker(rank, world, port, q):
    """The All-Gather baseline's exchange: each rank holds its head shard of
    every token's q and k; the gather must return the full vectors in head
    order on every rank."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import numpy as np
    import torch
    import torch.distributed as dist

    import attention_qk_norm_b200 as qkn

    dist.init_process_group("gloo", rank=rank, world_size=world)
    T, Hq, Hk, D = 5, 8, 4, 16
    x = torch.tensor(np.random.default_rng(1).standard_normal((T, (Hq + Hk) * D)))
    xq, xk = x[:, :Hq * D], x[:, Hq * D:]
    hq, hk = Hq // world, Hk // world
    mine_q = xq[:, rank * hq * D:(rank + 1) * hq * D]
    mine_k = xk[:, rank * hk * D:(rank + 1) * hk * D]
    fq, fk, w, r = qkn.tp_allgather_full(mine_q, mine_k)
    q.put((rank, w, r, bool(torch.equal(fq, xq)), bool(torch.equal(fk, xk))))
    dist.destroy_process_group()


def test_tensor_parallel_allgather_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_allgather_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(0, world, 0, True, True), (1, world, 1, True, True)]


def test_tensor_parallel_allreduce_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_tp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, ok, lens in out:
        assert got == world and ok and lens == (8 * 16, 4 * 16)


def test_two_gloo_ranks_barrier_and_max():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [15.0, 15.0]  # max over ranks, seen by every rank
    spans = [(o[2], o[3]) for o in out]
    assert spans == [(0, 501), (501, 1001)]


@pytest.mark.parametrize("total,world", [(0, 2), (7, 3), (4096, 8), (5, 8)])
def test_shard_units_partition(total, world):
    spans = [bench.shard_units(total, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == total
    for (a, b), (c, d) in zip(spans, spans[1:]):
        assert b == c
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def test_algorithmic_bytes():
    w = dict(bench.HEADLINE)
    assert bench.workload_bytes(w) == 2 * 4096 * 48 * 128 * 2 + 128 * 4
    lw = dict(kind="layerwise", T=8192, Hq=32, Hk=8, D=128, dtype="bf16")
    assert bench.workload_bytes(lw) == 2 * 8192 * 40 * 128 * 2 + 40 * 128 * 4


def _bench(args, env_extra=None):
    import subprocess
    import sys

    env = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, bench.__file__, *args], capture_output=True,
                          text=True, env=env, timeout=300)


def test_bench_gpus_flag_launches_that_many_ranks():
    """``bench.py --gpus 2`` without a launcher starts two ranks itself; the
    line reports both (gloo on CPU, --dry-run)."""
    import json

    r = _bench(["--gpus", "2", "--dry-run", "--steps", "4", "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    assert lines[0]["n_gpus"] == 2 and lines[0]["ranks_counted"] == 2
    assert lines[0]["max_over_ranks"] == 2.0  # rank 1's figure, seen by rank 0


def test_bench_gpus_flag_must_match_the_launcher():
    r = _bench(["--gpus", "2", "--dry-run"], {"WORLD_SIZE": "3", "RANK": "0"})
    assert r.returncode != 0 and "disagrees" in r.stderr


def _handles_worker(rank, world, port, q):
    """Every rank contributes a distinct 64-byte handle; every rank must get
    all of them in rank order (what qknorm_tp_comm_connect expects)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import attention_qk_norm_b200 as qkn

    dist.init_process_group("gloo", rank=rank, world_size=world)
    mine = bytes([rank + 1]) * qkn._binding.IPC_HANDLE_BYTES
    got = qkn.exchange_handles(mine)
    q.put((rank, [h[0] for h in got], all(len(h) == 64 for h in got)))
    dist.destroy_process_group()


def test_ipc_handles_gathered_in_rank_order_gloo():
    world = 4
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_handles_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(r, [1, 2, 3, 4], True) for r in range(world)]
