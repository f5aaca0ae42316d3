"""The in-kernel exchange of tensor-parallel layerwise QK-Norm on CPU ranks.

qknorm_layerwise_tp_p2p's exchange (attention_qk_norm_b200/csrc/tp_exchange.h:
one 64-bit {fp32 sum, call tag} word per rank, token and vector, stored into
every rank's receive buffer and polled there with a time limit; two buffer
halves used by alternate calls; a fixed pairwise rank tree) is built here for
the host and run with one process per rank, the receive buffers living in
shared host memory.  Each process plays its rank's kernel with several
"blocks" (threads).  The tests check what the protocol must guarantee:

* every rank gets the same bits, equal to the fixed rank tree of the ranks'
  sums, over consecutive calls that reuse both halves of the buffers, with
  different token counts, while ranks run at different speeds (one rank can
  be a call ahead of the others);
* a rank that stops taking part makes the others' waits give up within the
  time limit, counted, instead of hanging.

The SwiftQK review asks for exactly these two properties (major_comments[0]
on deadlock, major_comments[2] on the ordering of flag and payload).
"""
import ctypes
import time

import numpy as np
import pytest
import torch.multiprocessing as mp

from attention_qk_norm_b200 import buildlib


def _lib():
    lib = ctypes.CDLL(buildlib.build_tp_host())
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.qkn_tp_host_rank_call.argtypes = [vp, i32, i32, i64, ctypes.c_uint64, i64, i32, vp, vp,
                                          vp, vp, ctypes.c_double, i64, ctypes.c_double]
    lib.qkn_tp_host_rank_call.restype = i32
    lib.qkn_tp_host_buffer_words.argtypes = [i64, i32]
    lib.qkn_tp_host_buffer_words.restype = ctypes.c_uint64
    return lib


def _sums(call, rank, T):
    rng = np.random.default_rng(1000 * call + rank)
    return (rng.random(T, dtype=np.float32) * 100.0, rng.random(T, dtype=np.float32) * 7.0)


def _tree(values):
    """The kernel's rank combine (lane 0 of an xor butterfly), in float32."""
    world = len(values)
    v = [np.float32(x) for x in values] + [np.float32(0)] * (8 - world)
    d = 1
    while d < world:
        v = [np.float32(v[r] + v[r ^ d]) for r in range(8)]
        d <<= 1
    return v[0]


def _rank(shm_name, world, rank, max_tokens, Ts, blocks, timeout_s, stop_at, skew, start, q):
    from multiprocessing import shared_memory

    shm = shared_memory.SharedMemory(name=shm_name)
    try:
        lib = _lib()
        words = lib.qkn_tp_host_buffer_words(max_tokens, world)
        buf = np.ndarray((world, words), dtype=np.uint64, buffer=shm.buf)
        ptrs = (ctypes.c_void_p * world)(*[buf[r].ctypes.data for r in range(world)])
        out = []
        start.wait(timeout=120)  # every rank is up (process start-up takes seconds)
        for call, T in enumerate(Ts):
            if call == stop_at:
                break
            sq, sk = _sums(call, rank, T)
            oq, ok = np.zeros(T, np.float32), np.zeros(T, np.float32)
            t0 = time.monotonic()
            gave = lib.qkn_tp_host_rank_call(
                ptrs, world, rank, max_tokens, call, T, blocks, sq.ctypes.data, sk.ctypes.data,
                oq.ctypes.data, ok.ctypes.data, timeout_s, skew[0], skew[1])
            out.append((gave, oq.tobytes(), ok.tobytes(), time.monotonic() - t0))
        del buf
        q.put((rank, out))
    finally:
        shm.close()


def _run_group(world, Ts, blocks=3, timeout_s=20.0, stop=None, skews=None, max_tokens=64):
    from multiprocessing import shared_memory

    words = _lib().qkn_tp_host_buffer_words(max_tokens, world)
    shm = shared_memory.SharedMemory(create=True, size=int(world * words * 8))
    try:
        np.ndarray((world, words), dtype=np.uint64, buffer=shm.buf)[:] = 0
        ctx = mp.get_context("spawn")
        q = ctx.Queue()
        start = ctx.Barrier(world)
        procs = []
        for r in range(world):
            stop_at = stop.get(r, -1) if stop else -1
            skew = skews.get(r, (0, 0.0)) if skews else (0, 0.0)
            procs.append(ctx.Process(target=_rank, args=(shm.name, world, r, max_tokens, Ts,
                                                         blocks, timeout_s, stop_at, skew,
                                                         start, q)))
        for p in procs:
            p.start()
        res = dict(q.get(timeout=300) for _ in range(world))
        for p in procs:
            p.join(timeout=60)
            assert p.exitcode == 0
        return res
    finally:
        shm.close()
        shm.unlink()


@pytest.mark.parametrize("world", (1, 2, 4, 8))
def test_every_rank_gets_the_rank_tree_over_many_calls(world):
    Ts = (50, 20, 64, 1, 37, 64)  # six calls: both halves of every buffer, three times each
    # Ranks at different speeds: rank 0 runs ahead, the last rank pauses often.
    skews = {world - 1: (7, 0.002)} if world > 1 else None
    res = _run_group(world, Ts, skews=skews)
    for call, T in enumerate(Ts):
        want_q = np.array([_tree([_sums(call, r, T)[0][t] for r in range(world)])
                           for t in range(T)], dtype=np.float32)
        want_k = np.array([_tree([_sums(call, r, T)[1][t] for r in range(world)])
                           for t in range(T)], dtype=np.float32)
        for r in range(world):
            gave, oq, ok, _ = res[r][call]
            assert gave == 0, "rank %d call %d: a wait gave up" % (r, call)
            assert np.frombuffer(oq, np.float32).tobytes() == want_q.tobytes(), (r, call)
            assert np.frombuffer(ok, np.float32).tobytes() == want_k.tobytes(), (r, call)


def test_rank_tree_is_the_pairwise_order():
    """The combine is ((s0+s1)+(s2+s3))+((s4+s5)+(s6+s7)): values chosen so that
    any other order rounds differently in float32."""
    s = [np.float32(x) for x in (1e8, 1.0, -1e8, 1.0, 3.0, 2 ** -20, 5.0, 7.0)]
    want = np.float32(np.float32(np.float32(s[0] + s[1]) + np.float32(s[2] + s[3])) +
                      np.float32(np.float32(s[4] + s[5]) + np.float32(s[6] + s[7])))
    assert _tree(s) == want
    assert _tree(s) != np.float32(sum(np.float64(x) for x in s))


def test_a_rank_that_stops_makes_the_others_give_up_not_hang():
    world, timeout_s = 4, 0.5
    Ts = (40, 40, 40)
    res = _run_group(world, Ts, timeout_s=timeout_s, stop={3: 1})  # rank 3 skips calls 1, 2
    assert len(res[3]) == 1 and res[3][0][0] == 0
    for r in range(3):
        assert res[r][0][0] == 0  # call 0: everyone took part
        for call in (1, 2):
            gave, _, _, secs = res[r][call]
            assert gave >= 1, "rank %d call %d should have given up" % (r, call)
            # one time limit per block at most, the first give-up ends the others
            assert secs < 3 * 3 * timeout_s + 5.0
