"""GPU parity of qknorm_layerwise_tp_p2p: tensor-parallel layerwise QK-Norm with
the scalar exchange inside the kernel (SwiftQK's design), for a group of
ranks emulated on one GPU (TPComm.local: every rank's receive buffer on this
device, all ranks served by one cooperative launch whose blocks of one token
wait for one another).

Each rank holds its contiguous share of the query heads and of the key/value
heads (split by head); the reassembled outputs are compared element by
element with the float64 oracle of the whole vectors.  Where the fused
single-GPU kernel takes the same launch shape (decode sizes and the long
input), the result must also be bit-identical to qknorm_layerwise with
nshards = world: the ranks' sums are the shard subtrees of its fixed tree
and the rank combine is the rest of that tree.
"""
import numpy as np
import pytest
import torch

import attention_qk_norm_b200 as qkn
from attention_qk_norm_b200 import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _rank_case(c, n, r):
    """Rank r's fused buffer (its Q heads, its K heads, its V heads) and weights."""
    hq, hk, D = c.Hq // n, c.Hk // n, c.D
    q = np.arange(r * hq * D, (r + 1) * hq * D)
    k = c.Hq * D + np.arange(r * hk * D, (r + 1) * hk * D)
    v = (c.Hq + c.Hk) * D + np.arange(r * hk * D, (r + 1) * hk * D)
    cols = np.concatenate([q, k, v])
    gk = None if c.gamma_k is None else c.gamma_k[r * hk * D:(r + 1) * hk * D]
    sub = synth.Case(np.ascontiguousarray(c.qkv[:, cols]), c.gamma_q[r * hq * D:(r + 1) * hq * D],
                     gk, c.T, hq, hk, D, (hq + 2 * hk) * D, c.dtype, c.eps, True)
    return cols, sub


def run_group(c, n, comm=None, calls=1):
    """Run the emulated group on case c; returns the reassembled stored output."""
    own = comm is None
    comm = comm or qkn.TPComm.local(n, max_tokens=max(1, c.T))
    subs = [_rank_case(c, n, r) for r in range(n)]
    ups = [gu.to_device(sub) for _, sub in subs]
    for _ in range(calls):
        for (cols, sub), (buf, _, _) in zip(subs, ups):  # fresh input every call
            buf.copy_(gu.to_device(sub)[0])
        qkn.qknorm_layerwise_tp_p2p(comm, [u[0] for u in ups], c.Hq // n, c.Hk // n, c.D,
                                    [u[1] for u in ups], [u[2] for u in ups], c.eps)
    torch.cuda.synchronize()
    assert comm.errors() == 0, "a wait of the exchange gave up"
    out = c.qkv.copy()
    for (cols, sub), (buf, _, _) in zip(subs, ups):
        out[:, cols] = gu.stored_bits(buf)
    if own:
        comm.close()
    return out


@pytest.mark.parametrize("Hq,Hk,D,dtype", [(32, 8, 128, synth.BF16), (64, 8, 256, synth.FP32),
                                           (32, 8, 64, synth.FP8), (16, 8, 128, synth.FP16)])
@pytest.mark.parametrize("n", (1, 2, 4, 8))
@pytest.mark.parametrize("T", (1, 123, 1000))
def test_group_on_one_gpu_matches_oracle(Hq, Hk, D, dtype, n, T):
    c = synth.make_case(T, Hq, Hk, D, dtype=dtype, seed=500 + T + n + D, layerwise=True,
                        scale="stress", zero_frac=0.02, outlier_frac=0.02)
    out = run_group(c, n)
    want = gu.oracle_out(c, "layerwise", c.qkv, c.T)
    gu.check(out, want, c.qkv, dtype, (Hq + Hk) * D, "p2p n=%d T=%d %s" % (n, T, dtype))


@pytest.mark.parametrize("n", (1, 2, 4, 8))
@pytest.mark.parametrize("T", (1, 100, 8192))
def test_group_is_bit_identical_to_the_fused_kernel(n, T):
    """32 query / 8 key heads of 128 (the layerwise workload): at decode sizes
    and at T = 8192 both kernels give every thread two vectors of a head, so
    the rank sums are exactly the fused kernel's shard subtrees."""
    c = synth.make_case(T, seed=synth.LAYERWISE_SEED + 17 * n + T, **synth.LAYERWISE)
    out = run_group(c, n)
    full, gq, gk = gu.to_device(c)
    qkn.qknorm_layerwise(full, c.Hq, c.Hk, c.D, gq, gk, c.eps, nshards=n)
    torch.cuda.synchronize()
    assert np.array_equal(out, gu.stored_bits(full))
    if T == 8192:  # and the oracle at the full size, every element
        want = gu.oracle_out(c, "layerwise", c.qkv, c.T)
        gu.check(out, want, c.qkv, c.dtype, (c.Hq + c.Hk) * c.D, "p2p n=%d T=8192" % n)


def test_one_communicator_over_many_calls():
    """Consecutive calls alternate between the two halves of every receive
    buffer with growing tags; a call with fewer tokens than the last leaves
    stale slots behind that the next call must not take for fresh ones."""
    n = 4
    comm = qkn.TPComm.local(n, max_tokens=300)
    for i, T in enumerate((300, 7, 300, 1, 150, 300)):
        c = synth.make_case(T, 32, 8, 128, seed=900 + i, layerwise=True, scale="lognormal")
        out = run_group(c, n, comm=comm)
        want = gu.oracle_out(c, "layerwise", c.qkv, c.T)
        gu.check(out, want, c.qkv, c.dtype, 40 * 128, "call %d" % i)
    assert comm.errors() == 0
    comm.close()


def test_rejected_calls_launch_nothing():
    comm = qkn.TPComm.local(2, max_tokens=8)
    c = synth.make_case(9, 32, 8, 128, seed=3, layerwise=True)
    _, sub = _rank_case(c, 2, 0)
    bufs = [gu.to_device(_rank_case(c, 2, r)[1]) for r in range(2)]
    before = [b[0].clone() for b in bufs]
    with pytest.raises(qkn.QKNormError) as e:  # T = 9 > max_tokens = 8
        qkn.qknorm_layerwise_tp_p2p(comm, [b[0] for b in bufs], 16, 4, 128, [b[1] for b in bufs],
                                    [b[2] for b in bufs], 1e-6)
    assert e.value.status == -8
    with pytest.raises(ValueError):  # one buffer for a two-rank local group
        qkn.qknorm_layerwise_tp_p2p(comm, bufs[0][0], 16, 4, 128, bufs[0][1], bufs[0][2], 1e-6)
    torch.cuda.synchronize()
    for b, a in zip(bufs, before):
        assert torch.equal(b[0].view(torch.int16), a.view(torch.int16))
    comm.close()


def test_a_rank_of_its_own_group():
    """A one-rank group created through the multi-process path (no process
    group): the exchange with itself gives the fused kernel's bits."""
    c = synth.make_case(77, 32, 8, 128, seed=41, layerwise=True)
    comm = qkn.TPComm.from_group(max_tokens=128)
    x, gq, gk = gu.to_device(c)
    qkn.qknorm_layerwise_tp_p2p(comm, x, 32, 8, 128, gq, gk, c.eps)
    y, gq2, gk2 = gu.to_device(c)
    qkn.qknorm_layerwise(y, 32, 8, 128, gq2, gk2, c.eps)
    torch.cuda.synchronize()
    assert comm.errors() == 0
    assert np.array_equal(gu.stored_bits(x), gu.stored_bits(y))
    comm.close()


def test_group_calls_replayed_from_a_cuda_graph():
    """Two calls captured in one CUDA graph and the graph replayed three times,
    fresh inputs copied into the buffers before each replay: every replay
    must match the oracle (inputs and weights are copied into the captured
    tensors).  Each launch takes a new sequence number (and so
    a new tag) from device memory; a tag frozen at capture would let a replay
    take the previous replay's sums for fresh ones."""
    n, T = 4, 300
    comm = qkn.TPComm.local(n, max_tokens=T)
    cases = [synth.make_case(T, 32, 8, 128, seed=700 + i, layerwise=True, scale="lognormal")
             for i in range(4)]
    ups = [gu.to_device(_rank_case(cases[0], n, r)[1]) for r in range(n)]
    xs, gqs, gks = [u[0] for u in ups], [u[1] for u in ups], [u[2] for u in ups]
    second = [x.clone() for x in xs]  # the second captured call works on its own buffers
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up call outside the capture
        qkn.qknorm_layerwise_tp_p2p(comm, xs, 8, 2, 128, gqs, gks, 1e-6)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        qkn.qknorm_layerwise_tp_p2p(comm, xs, 8, 2, 128, gqs, gks, 1e-6)
        qkn.qknorm_layerwise_tp_p2p(comm, second, 8, 2, 128, gqs, gks, 1e-6)
    for c in cases[1:]:
        for r, (x, y) in enumerate(zip(xs, second)):
            fresh, fq, fk = gu.to_device(_rank_case(c, n, r)[1])
            x.copy_(fresh)
            y.copy_(fresh)
            gqs[r].copy_(fq)  # each case draws its own weights
            gks[r].copy_(fk)
        g.replay()
        torch.cuda.synchronize()
        want = gu.oracle_out(c, "layerwise", c.qkv, c.T)
        for bufs in (xs, second):
            out = c.qkv.copy()
            for r, buf in enumerate(bufs):
                out[:, _rank_case(c, n, r)[0]] = gu.stored_bits(buf)
            gu.check(out, want, c.qkv, c.dtype, 40 * 128, "graph replay")
    assert comm.errors() == 0
    del g
    comm.close()


def _random_groups(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        dtype = [synth.BF16, synth.FP16, synth.FP32, synth.FP8][int(rng.integers(4))]
        D = int(rng.choice([64, 128, 256]))
        world = int(rng.choice([2, 4, 8]))
        hq = int(rng.integers(0, 5))
        hk = int(rng.integers(0 if hq else 1, 3))
        T = int(rng.choice([1, 5, 149, 333]))
        out.append(dict(dtype=dtype, D=D, world=world, Hq=hq * world, Hk=hk * world, T=T,
                        seed=seed + i))
    return out


@pytest.mark.parametrize("cfg", _random_groups(16, 6000), ids=lambda c: "%s-D%d-%dq%dk-w%d-T%d" % (
    c["dtype"], c["D"], c["Hq"], c["Hk"], c["world"], c["T"]))
def test_random_groups(cfg):
    """Seeded random groups of the in-kernel exchange: storage type, head_dim,
    group size, heads per rank (either kind may be absent) and T; every
    element against the oracle of the whole vectors."""
    c = synth.make_case(cfg["T"], cfg["Hq"], cfg["Hk"], cfg["D"], dtype=cfg["dtype"],
                        seed=cfg["seed"], layerwise=True, scale="stress", zero_frac=0.02,
                        outlier_frac=0.02)
    out = run_group(c, cfg["world"])
    want = gu.oracle_out(c, "layerwise", c.qkv, c.T)
    gu.check(out, want, c.qkv, c.dtype, (c.Hq + c.Hk) * c.D, "random group %s" % cfg)
