"""GPU parity: libqknorm.so (through its C ABI) against the float64 oracle.

Every case draws the same seeded input for both sides.  Sizes the oracle
finishes in seconds are compared element by element over the whole buffer
(several tiles plus ragged tails); the full-size workloads are compared on
sampled tokens (random ones, the first and last, and every all-zero or
outlier row found), which the oracle computes one token at a time.
Tolerances are in ``tests/gpu_util.py``.
"""
import numpy as np
import pytest
import torch

import attention_qk_norm_b200 as qkn
from attention_qk_norm_b200 import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

GUARD = 3
GUARD_VALUE = -7.25


def run(kind, qkv, c, gq, gk, nshards=1, stream=None):
    if kind == "per_head":
        qkn.qknorm_per_head(qkv, c.Hq, c.Hk, c.D, gq, gk, c.eps, row_stride=c.row_stride,
                            stream=stream)
    else:
        qkn.qknorm_layerwise(qkv, c.Hq, c.Hk, c.D, gq, gk, c.eps, nshards=nshards,
                             row_stride=c.row_stride, stream=stream)


def full_parity(case, kind, nshards=1, what=""):
    full, gq, gk = gu.to_device(case, extra_rows=GUARD)
    run(kind, full[: case.T], case, gq, gk, nshards)
    torch.cuda.synchronize()
    out = gu.stored_bits(full)
    want = gu.oracle_out(case, kind, case.qkv, case.T)
    qk = (case.Hq + case.Hk) * case.D
    err = gu.check(out[: case.T], want, case.qkv, case.dtype, qk, what)
    guard = out[case.T:]
    ref = gu.stored_bits(torch.full((1,), GUARD_VALUE, dtype=full.dtype))[0]
    assert np.all(guard == ref), "%s: wrote past the last row" % what
    return out[: case.T], err


# ------------------------------------------------------------------ configs --
def test_smoke_config():
    c = synth.make_case(**synth.SMOKE)
    full_parity(c, "per_head", what="smoke")


@pytest.mark.parametrize("H", synth.SWEEP_HEADS)
@pytest.mark.parametrize("T", synth.SWEEP_T + (3, 257, 1000))
def test_per_head_sweep(H, T):
    c = synth.sweep_case(H, T)
    assert c.Hk == 0 and c.row_stride == H * 128
    full_parity(c, "per_head", what="sweep H=%d T=%d" % (H, T))


@pytest.mark.parametrize("T", (1, 64, 1024, 4096, 3001))
def test_gqa_fused(T):
    c = synth.make_case(T, seed=synth.GQA_SEED + T, **synth.GQA)
    assert c.row_stride == 6144
    full_parity(c, "per_head", what="gqa T=%d" % T)


@pytest.mark.parametrize("T", (1, 16, 256, 4096, 1000))
def test_layerwise(T):
    c = synth.make_case(T, seed=synth.LAYERWISE_SEED + T, **synth.LAYERWISE)
    outs = [full_parity(c, "layerwise", n, what="layerwise T=%d n=%d" % (T, n))[0]
            for n in synth.LAYERWISE_NSHARDS]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0]), "layerwise output depends on nshards"


@pytest.mark.parametrize("dtype", (synth.BF16, synth.FP16))
def test_layerwise_config_largest_T_every_element(dtype):
    """The layerwise workload at its largest T (8192), which takes the long-input
    launch shape (two vectors per thread, 320-thread blocks, staging ring):
    every element against the oracle for nshards 1 and 8, the same bits for
    both."""
    T = synth.LAYERWISE_T[-1]
    c = synth.make_case(T, seed=synth.LAYERWISE_SEED + T, **dict(synth.LAYERWISE, dtype=dtype))
    outs = [full_parity(c, "layerwise", n, what="layerwise %s T=%d n=%d" % (dtype, T, n))[0]
            for n in (1, 8)]
    assert np.array_equal(outs[0], outs[1]), "layerwise output depends on nshards"


@pytest.mark.parametrize("D", synth.STRESS_D)
def test_stress_layerwise_bf16_long_every_element(D):
    """Stress layerwise (64 query / 8 key heads, lognormal scales over 1e-3..1e3,
    zero and outlier rows) at 7200 tokens, long enough for the long-input
    shape at every head_dim (single blocks at 64 and 128, 2-block clusters at
    256): every element against the oracle, nshards 1 and 8 bit-identical."""
    kw = dict(synth.STRESS, T=7200)
    c = synth.make_case(D=D, dtype=synth.BF16, eps=1e-6, seed=synth.STRESS_SEED + 7 * D,
                        layerwise=True, **kw)
    outs = [full_parity(c, "layerwise", n, what="stress layerwise long D=%d n=%d" % (D, n))[0]
            for n in (1, 8)]
    assert np.array_equal(outs[0], outs[1])


@pytest.mark.parametrize("dtype", synth.STRESS_DTYPES)
@pytest.mark.parametrize("D", synth.STRESS_D)
@pytest.mark.parametrize("eps", synth.STRESS_EPS)
def test_stress_small(dtype, D, eps):
    kw = dict(synth.STRESS, T=1037)
    c = synth.make_case(D=D, dtype=dtype, eps=eps, seed=synth.STRESS_SEED + D, **kw)
    full_parity(c, "per_head", what="stress per-head %s D=%d" % (dtype, D))
    lw = synth.make_case(D=D, dtype=dtype, eps=eps, seed=synth.STRESS_SEED + D, layerwise=True,
                         **kw)
    a, _ = full_parity(lw, "layerwise", 8, what="stress layerwise %s D=%d" % (dtype, D))
    b, _ = full_parity(lw, "layerwise", 1, what="stress layerwise %s D=%d" % (dtype, D))
    assert np.array_equal(a, b)


# --------------------------------------------------- full sizes, sampled --
def sampled_parity(d, kind, nshards_list=(1,), n_random=256, seed=0):
    qkv = d["qkv"]
    c = gu.Sampled(d)
    qk = (c.Hq + c.Hk) * c.D
    idx = gu.sample_tokens(qkv, qk, n_random, seed)
    x_s = gu.stored_bits(qkv[idx])
    want = gu.oracle_out(c, kind, x_s, int(idx.numel()))
    first = None
    for n in nshards_list:
        buf = qkv.clone() if len(nshards_list) > 1 else qkv
        run(kind, buf, c, d["gamma_q"], d["gamma_k"], n)
        torch.cuda.synchronize()
        gu.check(gu.stored_bits(buf[idx]), want, x_s, c.dtype, qk, "%s n=%d" % (kind, n))
        bits = buf.view(torch.uint8) if buf.dtype == torch.float8_e4m3fn else (
            buf.view(torch.int16) if buf.element_size() == 2 else buf.view(torch.int32))
        if first is None:
            first = bits
        else:
            assert torch.equal(bits, first), "output depends on nshards"
        del buf


def test_sweep_full_size_h48_t4096_sampled():
    d = synth.make_case_torch(4096, 48, 0, 128, device="cuda", seed=7, eps=1e-6)
    sampled_parity(d, "per_head")


def test_gqa_full_size_sampled():
    T = synth.GQA_T[-1]
    d = synth.make_case_torch(T, device="cuda", seed=synth.GQA_SEED, **synth.GQA)
    sampled_parity(d, "per_head")


def test_layerwise_full_size_sampled():
    T = synth.LAYERWISE_T[-1]
    d = synth.make_case_torch(T, device="cuda", seed=synth.LAYERWISE_SEED, **synth.LAYERWISE)
    sampled_parity(d, "layerwise", synth.LAYERWISE_NSHARDS)


@pytest.mark.parametrize("dtype", synth.STRESS_DTYPES)
@pytest.mark.parametrize("D", synth.STRESS_D)
@pytest.mark.parametrize("eps", synth.STRESS_EPS)
def test_stress_full_size_sampled(dtype, D, eps):
    d = synth.make_case_torch(D=D, dtype=dtype, eps=eps, device="cuda",
                              seed=synth.STRESS_SEED + D, **synth.STRESS)
    sampled_parity(d, "per_head", seed=D)
    del d
    d = synth.make_case_torch(D=D, dtype=dtype, eps=eps, device="cuda", layerwise=True,
                              seed=synth.STRESS_SEED + D, **synth.STRESS)
    sampled_parity(d, "layerwise", (1, 8), n_random=128, seed=D)
    del d
    torch.cuda.empty_cache()


# --------------------------------------------------------------- edge cases --
def test_empty_input_is_a_no_op():
    x = torch.empty((0, 2560), dtype=torch.bfloat16, device="cuda")
    g = torch.ones(128, device="cuda")
    qkn.qknorm_per_head(x, 16, 2, 128, g, g, 1e-6)
    qkn.qknorm_layerwise(x, 16, 2, 128, torch.ones(2048, device="cuda"),
                         torch.ones(256, device="cuda"), 1e-6, nshards=2)


@pytest.mark.parametrize("dtype", (synth.BF16, synth.FP32))
@pytest.mark.parametrize("D", synth.STRESS_D)
def test_padded_rows_and_key_only(dtype, D):
    es = 2 if dtype == synth.BF16 else 4
    pad = 48 // es  # 48 bytes of padding keeps rows 16-byte aligned
    c = synth.make_case(37, 3, 2, D, dtype=dtype, seed=11, row_stride=(3 + 4) * D + pad)
    full_parity(c, "per_head", what="padded")
    c = synth.make_case(9, 0, 3, D, dtype=dtype, seed=12)
    full_parity(c, "per_head", what="key heads only")
    c = synth.make_case(9, 2, 2, D, dtype=dtype, seed=13, row_stride=6 * D + pad,
                        layerwise=True)
    full_parity(c, "layerwise", 2, what="layerwise padded")


@pytest.mark.parametrize("Hq,Hk,ns", [(40, 8, (1, 2, 4, 8)), (24, 4, (1, 2, 4)), (3, 1, (1,)),
                                      (6, 2, (1, 2)), (64, 8, (1, 8)), (1, 0, (1,))])
def test_layerwise_head_counts(Hq, Hk, ns):
    c = synth.make_case(23, Hq, Hk, 128, seed=Hq * 10 + Hk, layerwise=True)
    outs = [full_parity(c, "layerwise", n, what="Hq=%d Hk=%d n=%d" % (Hq, Hk, n))[0] for n in ns]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


@pytest.mark.parametrize("dtype", (synth.BF16, synth.FP32))
@pytest.mark.parametrize("D", synth.STRESS_D)
@pytest.mark.parametrize("Hq,Hk,ns", [(64, 8, (1, 8)), (32, 4, (1, 4)), (30, 5, (1, 5))])
def test_layerwise_wide_tokens(dtype, D, Hq, Hk, ns):
    """Wide tokens: one block of up to 576 threads, or heads split over a
    thread-block cluster where a block would need more (72 or 36 heads at
    head_dim 256), or an odd head count (35) that no cluster size divides."""
    ns = tuple(n for n in ns if n in (1, 2, 4, 8))
    c = synth.make_case(45, Hq, Hk, D, dtype=dtype, seed=Hq + D, layerwise=True, scale="stress",
                        zero_frac=0.05, outlier_frac=0.05)
    outs = [full_parity(c, "layerwise", n, what="wide %s D=%d n=%d" % (dtype, D, n))[0]
            for n in ns]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


@pytest.mark.parametrize("Hq,Hk,D,dtype,ns", [
    (112, 16, 256, synth.BF16, (1, 2, 8)),  # 2-block clusters of 512 threads
    (144, 16, 256, synth.FP16, (1, 8)),     # 4-block clusters
    (256, 64, 256, synth.BF16, (1, 4)),     # 8-block clusters
    (64, 16, 256, synth.FP32, (1, 8)),      # 2-block clusters, fp32
    (112, 16, 256, synth.FP8, (1, 4)),      # 2-block clusters, FP8
])
def test_layerwise_cluster_split(Hq, Hk, D, dtype, ns):
    """Tokens too wide for one block of 576 threads with gamma in registers:
    the heads are split over a cluster of 2, 4 or 8 blocks, which pass head
    partials to one another through distributed shared memory.  700 tokens
    give every cluster several tokens, so both partials buffers and several
    phases of their barriers are used.  Outputs are identical for every
    nshards."""
    c = synth.make_case(700, Hq, Hk, D, dtype=dtype, seed=Hq + Hk + D, layerwise=True,
                        scale="stress", zero_frac=0.05, outlier_frac=0.05)
    outs = [full_parity(c, "layerwise", n, what="cluster %s %d/%d n=%d" % (dtype, Hq, Hk, n))[0]
            for n in ns]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


@pytest.mark.parametrize("T", (1, 5, 37))
@pytest.mark.parametrize("Hq,Hk,D,dtype", [(32, 8, 128, synth.BF16), (32, 8, 128, synth.FP8),
                                           (112, 16, 256, synth.BF16), (256, 64, 256, synth.BF16)])
def test_layerwise_decode_sizes(T, Hq, Hk, D, dtype):
    """Decode-size inputs, at most one block per SM: the fused kernel loads each
    token straight into registers (no staging ring), in single blocks or in
    2- and 8-block clusters.  Every element against the oracle, the same bits
    for every nshards, and for one rank the same bits as the two
    tensor-parallel steps, which stage through the ring."""
    c = synth.make_case(T, Hq, Hk, D, dtype=dtype, seed=90 + T + Hq, layerwise=True,
                        scale="lognormal")
    outs = [full_parity(c, "layerwise", n, what="decode T=%d n=%d" % (T, n))[0] for n in (1, 8)]
    assert np.array_equal(outs[0], outs[1])
    x, gq, gk = gu.to_device(c)
    sums = qkn.qknorm_layerwise_partials(x, Hq, Hk, D)
    qkn.qknorm_layerwise_apply(x, Hq, Hk, D, gq, gk, sums, Hq * D, Hk * D, c.eps)
    torch.cuda.synchronize()
    assert np.array_equal(gu.stored_bits(x), outs[0])


@pytest.mark.parametrize("dtype,T,Hq,Hk,D,ns", [
    (synth.FP8, 4000, 64, 8, 128, (1, 8)),   # overlap; 8 query warps, 64-head tree
    (synth.FP8, 3000, 8, 4, 128, (1, 4)),    # key warp padded past its 4 heads
    (synth.FP8, 500, 0, 16, 128, (1, 8)),    # key heads only
    (synth.FP8, 500, 16, 0, 64, (1, 8)),     # query heads only, 16 heads per warp
    (synth.FP8, 2000, 32, 8, 256, (1, 8)),   # 4 heads per warp
    (synth.FP8, 300, 4, 4, 128, (1, 4)),     # a warp holds both kinds: head partials
    (synth.FP8, 300, 12, 4, 128, (1, 4)),    # 12 is no power of two: head partials
    (synth.FP8, 300, 128, 8, 128, (1, 8)),   # 16 query warps: head partials
    (synth.BF16, 64, 32, 8, 128, (1, 8)),    # decode size, direct schedule
    (synth.BF16, 1000, 32, 8, 128, (1, 8)),  # short input, twice the vectors per thread
    (synth.BF16, 1000, 16, 16, 64, (1, 8)),
    (synth.FP32, 500, 32, 8, 128, (1, 8)),
])
def test_layerwise_warp_tree(dtype, T, Hq, Hk, D, ns):
    """Shapes on both sides of the warp tree's conditions (FP8 launches and
    short inputs; each vector a power of two of heads up to 64, whole warps
    per vector, at most 8 warps per vector).  Every element against the
    oracle, the same bits for every nshards, and the same bits as the two
    tensor-parallel steps, whose partials step always sums head partials
    in warp_sumsq's order at the same vectors per thread."""
    c = synth.make_case(T, Hq, Hk, D, dtype=dtype, seed=400 + T + Hq + D, layerwise=True,
                        scale="stress", zero_frac=0.02, outlier_frac=0.02)
    outs = [full_parity(c, "layerwise", n, what="warp tree %s %d/%d n=%d" % (dtype, Hq, Hk, n))[0]
            for n in ns]
    assert np.array_equal(outs[0], outs[1])
    x, gq, gk = gu.to_device(c)
    sums = qkn.qknorm_layerwise_partials(x, Hq, Hk, D)
    qkn.qknorm_layerwise_apply(x, Hq, Hk, D, gq, gk, sums, Hq * D, Hk * D, c.eps)
    torch.cuda.synchronize()
    assert np.array_equal(gu.stored_bits(x), outs[0])


@pytest.mark.parametrize("dtype", (synth.BF16, synth.FP8))
def test_layerwise_gamma_through_l1(dtype):
    """129 heads of 256 (odd, so no cluster split): gamma cannot stay in
    registers within 1024 threads, so the kernel reads it through L1."""
    c = synth.make_case(37, 121, 8, 256, dtype=dtype, seed=61, layerwise=True, scale="stress",
                        zero_frac=0.05, outlier_frac=0.05)
    full_parity(c, "layerwise", 1, what="gamma through L1 %s" % dtype)


@pytest.mark.parametrize("dtype", (synth.FP16, synth.FP8))
@pytest.mark.parametrize("D", synth.STRESS_D)
def test_low_precision_per_head(dtype, D):
    c = synth.make_case(333, 32, 8, D, dtype=dtype, seed=50 + D, scale="stress",
                        zero_frac=0.02, outlier_frac=0.02)
    full_parity(c, "per_head", what="%s per-head gqa D=%d" % (dtype, D))
    c = synth.make_case(257, 48, 0, D, dtype=dtype, seed=51 + D)
    full_parity(c, "per_head", what="%s per-head sweep D=%d" % (dtype, D))


@pytest.mark.parametrize("dtype", (synth.FP16, synth.FP8))
@pytest.mark.parametrize("D", synth.STRESS_D)
@pytest.mark.parametrize("Hq,Hk", [(32, 8), (64, 8)])
def test_low_precision_layerwise(dtype, D, Hq, Hk):
    c = synth.make_case(211, Hq, Hk, D, dtype=dtype, seed=60 + D + Hq, layerwise=True,
                        scale="lognormal")
    outs = [full_parity(c, "layerwise", n, what="%s layerwise D=%d n=%d" % (dtype, D, n))[0]
            for n in (1, 8)]
    assert np.array_equal(outs[0], outs[1])


@pytest.mark.parametrize("dtype,T,Hq,Hk,D", [(synth.FP8, 8192, 32, 8, 128),
                                              (synth.FP32, 4096, 64, 8, 64)])
def test_layerwise_overlap_every_element(dtype, T, Hq, Hk, D):
    """Inputs long enough for the launch rule to pick the overlap variant (x*gamma
    formed before the combine): every element against the oracle, and the
    same bits for every nshards."""
    c = synth.make_case(T, Hq, Hk, D, dtype=dtype, seed=72 + D, layerwise=True, scale="stress",
                        zero_frac=0.01, outlier_frac=0.01)
    outs = [full_parity(c, "layerwise", n, what="overlap %s n=%d" % (dtype, n))[0] for n in (1, 8)]
    assert np.array_equal(outs[0], outs[1])


@pytest.mark.parametrize("dtype", (synth.FP16, synth.FP8))
def test_low_precision_full_size_sampled(dtype):
    d = synth.make_case_torch(16384, device="cuda", seed=70, **dict(synth.GQA, dtype=dtype))
    sampled_parity(d, "per_head")
    del d
    d = synth.make_case_torch(8192, device="cuda", seed=71, **dict(synth.LAYERWISE, dtype=dtype))
    sampled_parity(d, "layerwise", (1, 8))


def test_zero_eps_on_nonzero_rows():
    c = synth.make_case(64, 4, 2, 128, seed=21, eps=0.0)
    full_parity(c, "per_head", what="eps=0")
    c = synth.make_case(64, 4, 2, 128, seed=22, eps=0.0, layerwise=True)
    full_parity(c, "layerwise", 2, what="eps=0 layerwise")


def test_side_stream_and_repeatability():
    c = synth.make_case(777, 32, 8, 128, seed=31, scale="lognormal")
    a, gq, gk = gu.to_device(c)
    b = a.clone()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        run("per_head", a, c, gq, gk, stream=s)
    s.synchronize()
    run("per_head", b, c, gq, gk)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_errors_leave_buffer_untouched():
    c = synth.make_case(8, 16, 2, 128, seed=41)
    full, gq, gk = gu.to_device(c)
    before = full.clone()
    with pytest.raises(qkn.QKNormError) as e:
        # a view that starts 8 bytes into the buffer: misaligned base pointer
        qkn.qknorm_per_head(full[:, 4:], 16, 2, 128, gq, gk, 1e-6, row_stride=2560)
    assert e.value.status == -3
    with pytest.raises(qkn.QKNormError) as e:
        qkn.qknorm_layerwise(full, 16, 2, 128, gq, gk, 1e-6, nshards=4)
    assert e.value.status == -4
    # 137 fp32 heads of 256: an odd head count rules out a cluster split, and
    # two staged tokens in one block would need 274 KiB of shared memory
    wide = torch.zeros((1, (129 + 16) * 256), dtype=torch.float32, device="cuda")
    g = torch.ones(129 * 256, device="cuda")
    with pytest.raises(qkn.QKNormError) as e:
        qkn.qknorm_layerwise(wide, 129, 8, 256, g, g, 1e-6)
    assert e.value.status == -5
    torch.cuda.synchronize()
    assert torch.equal(full.view(torch.int16), before.view(torch.int16))


# ------------------------------------------- tensor-parallel layerwise steps --
def _rank_columns(c, n, r):
    """Global columns of rank r's fused buffer when heads are split in n
    contiguous groups (its Q heads, then its K heads, then its V heads)."""
    hq, hk, D = c.Hq // n, c.Hk // n, c.D
    q = np.arange(r * hq * D, (r + 1) * hq * D)
    k = c.Hq * D + np.arange(r * hk * D, (r + 1) * hk * D)
    v = (c.Hq + c.Hk) * D + np.arange(r * hk * D, (r + 1) * hk * D)
    return np.concatenate([q, k, v]), hq, hk


@pytest.mark.parametrize("Hq,Hk,D,dtype", [(32, 8, 128, synth.BF16), (64, 8, 256, synth.FP32),
                                           (32, 8, 64, synth.FP8), (16, 8, 128, synth.FP16),
                                           (112, 16, 256, synth.BF16)])
@pytest.mark.parametrize("n", (1, 2, 4, 8))
def test_tensor_parallel_steps_emulated(Hq, Hk, D, dtype, n):
    """n ranks emulated one after another on one GPU: each rank's partial sums,
    their sum (standing in for the all-reduce), each rank's scaling; the
    reassembled result must match the float64 oracle of the whole vectors."""
    c = synth.make_case(123, Hq, Hk, D, dtype=dtype, seed=80 + n + D, layerwise=True,
                        scale="lognormal")
    W = (Hq + 2 * Hk) * D
    locals_, sums = [], None
    for r in range(n):
        cols, hq, hk = _rank_columns(c, n, r)
        sub = synth.Case(np.ascontiguousarray(c.qkv[:, cols]),
                         c.gamma_q[r * hq * D:(r + 1) * hq * D],
                         c.gamma_k[r * hk * D:(r + 1) * hk * D], c.T, hq, hk, D,
                         (hq + 2 * hk) * D, dtype, c.eps, True)
        buf, gq, gk = gu.to_device(sub)
        part = qkn.qknorm_layerwise_partials(buf, hq, hk, D)
        sums = part.clone() if sums is None else sums + part
        locals_.append((cols, sub, buf, gq, gk))
    out = c.qkv.copy()
    for cols, sub, buf, gq, gk in locals_:
        qkn.qknorm_layerwise_apply(buf, sub.Hq, sub.Hk, D, gq, gk, sums, Hq * D, Hk * D, c.eps)
        torch.cuda.synchronize()
        out[:, cols] = gu.stored_bits(buf)
    want = gu.oracle_out(c, "layerwise", c.qkv, c.T)
    gu.check(out, want, c.qkv, dtype, (Hq + Hk) * D, "tp n=%d" % n)
    assert out.shape[1] == W
    if n == 1:  # a single rank is exactly the fused kernel
        full, gq, gk = gu.to_device(c)
        qkn.qknorm_layerwise(full, Hq, Hk, D, gq, gk, c.eps)
        torch.cuda.synchronize()
        assert np.array_equal(gu.stored_bits(full), out)
        x, gq, gk = gu.to_device(c)
        qkn.qknorm_layerwise_tp(x, Hq, Hk, D, gq, gk, c.eps)  # no process group: one rank
        torch.cuda.synchronize()
        assert np.array_equal(gu.stored_bits(x), out)


@pytest.mark.parametrize("Hq,Hk,D,dtype", [(32, 8, 128, synth.BF16), (64, 8, 64, synth.FP32)])
def test_tensor_parallel_allgather_baseline_one_rank(Hq, Hk, D, dtype):
    """The All-Gather baseline with a single rank (no process group): the
    gathered vectors are this rank's own, so the result is exactly the fused
    kernel's, and V is untouched."""
    c = synth.make_case(211, Hq, Hk, D, dtype=dtype, seed=95, layerwise=True, scale="lognormal")
    x, gq, gk = gu.to_device(c)
    qkn.qknorm_layerwise_tp_allgather(x, Hq, Hk, D, gq, gk, c.eps)
    y, gq2, gk2 = gu.to_device(c)
    qkn.qknorm_layerwise(y, Hq, Hk, D, gq2, gk2, c.eps)
    torch.cuda.synchronize()
    assert np.array_equal(gu.stored_bits(x), gu.stored_bits(y))
    want = gu.oracle_out(c, "layerwise", c.qkv, c.T)
    gu.check(gu.stored_bits(x), want, c.qkv, dtype, (Hq + Hk) * D, "all-gather baseline")


def test_tensor_parallel_partials_leave_buffer_untouched():
    c = synth.make_case(77, 32, 8, 128, seed=90, layerwise=True)
    buf, _, _ = gu.to_device(c)
    part = qkn.qknorm_layerwise_partials(buf, 32, 8, 128)
    torch.cuda.synchronize()
    assert np.array_equal(gu.stored_bits(buf), c.qkv)
    x = gu.as_f64(c.qkv, c.dtype)
    want = np.stack([(x[:, :4096] ** 2).sum(1), (x[:, 4096:5120] ** 2).sum(1)], 1)
    got = part.cpu().numpy().astype(np.float64)
    assert np.allclose(got, want, rtol=1e-5, atol=0)


def test_no_in_kernel_wait_gave_up():
    """The cluster exchange waits of every launch above completed: none ran into
    its time limit (which would have left wrong results behind)."""
    torch.cuda.synchronize()
    assert qkn.wait_timeouts() == 0


def test_calls_capture_into_a_cuda_graph():
    """Decode-style use: a graph of per-head, layerwise and tensor-parallel
    step calls, captured once and replayed on new inputs copied into the same
    buffers, gives exactly the outputs of the same calls made eagerly (the
    library neither allocates, synchronises nor reads device data on the host
    inside a call)."""
    Hq, Hk, D, T = 32, 8, 128, 3
    cases = [synth.make_case(T, Hq, Hk, D, seed=s, layerwise=True) for s in (301, 302)]
    x, gq, gk = gu.to_device(cases[0])      # per-head buffer
    y, lq, lk = gu.to_device(cases[0])      # layerwise buffer (same data, other weights use)
    z, _, _ = gu.to_device(cases[0])        # tensor-parallel steps buffer
    gq_h, gk_h = gq[:D].contiguous(), gk[:D].contiguous()
    part = torch.empty((T, 2), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm the launch-shape caches outside the capture
        qkn.qknorm_per_head(x, Hq, Hk, D, gq_h, gk_h, 1e-6)
        qkn.qknorm_layerwise(y, Hq, Hk, D, lq, lk, 1e-6, nshards=4)
        qkn.qknorm_layerwise_partials(z, Hq, Hk, D, partials=part)
        qkn.qknorm_layerwise_apply(z, Hq, Hk, D, lq, lk, part, Hq * D, Hk * D, 1e-6)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        qkn.qknorm_per_head(x, Hq, Hk, D, gq_h, gk_h, 1e-6)
        qkn.qknorm_layerwise(y, Hq, Hk, D, lq, lk, 1e-6, nshards=4)
        qkn.qknorm_layerwise_partials(z, Hq, Hk, D, partials=part)
        qkn.qknorm_layerwise_apply(z, Hq, Hk, D, lq, lk, part, Hq * D, Hk * D, 1e-6)
    for c in cases:
        src, _, _ = gu.to_device(c)
        for buf in (x, y, z):
            buf.copy_(src)
        g.replay()
        torch.cuda.synchronize()
        ex, _, _ = gu.to_device(c)
        ey, _, _ = gu.to_device(c)
        qkn.qknorm_per_head(ex, Hq, Hk, D, gq_h, gk_h, 1e-6)
        qkn.qknorm_layerwise(ey, Hq, Hk, D, lq, lk, 1e-6, nshards=4)
        torch.cuda.synchronize()
        assert np.array_equal(gu.stored_bits(x), gu.stored_bits(ex))
        assert np.array_equal(gu.stored_bits(y), gu.stored_bits(ey))
        assert np.array_equal(gu.stored_bits(z), gu.stored_bits(ey))  # one rank: the fused result


# ------------------------------------------------------------- random shapes --
def _random_shapes(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        dtype = [synth.BF16, synth.FP16, synth.FP32, synth.FP8][int(rng.integers(4))]
        D = int(rng.choice([64, 128, 256]))
        ns = int(rng.choice([1, 2, 4, 8]))
        Hq = int(rng.integers(0, 11)) * ns
        Hk = int(rng.integers(0 if Hq else 1, 5)) * ns
        es = {synth.BF16: 2, synth.FP16: 2, synth.FP32: 4, synth.FP8: 1}[dtype]
        pad = int(rng.integers(0, 4)) * (16 // es)  # keeps rows 16-byte aligned
        T = int(rng.choice([1, 2, 3, 17, 149, 150, 333, 777]))
        eps = float(rng.choice([0.0, 1e-6, 1e-5, 1e-2]))
        out.append(dict(dtype=dtype, D=D, ns=ns, Hq=Hq, Hk=Hk, pad=pad, T=T, eps=eps, seed=seed + i))
    return out


@pytest.mark.parametrize("cfg", _random_shapes(40, 4000), ids=lambda c: "%s-D%d-%dq%dk-n%d-T%d" % (
    c["dtype"], c["D"], c["Hq"], c["Hk"], c["ns"], c["T"]))
def test_random_shapes(cfg):
    """Seeded random shapes through both variants: storage type, head_dim, head
    counts (multiples of nshards, either kind may be absent), row padding,
    token counts around the decode / short / long launch-shape boundaries,
    and eps (0 only where no row is all zero).  Every element against the
    oracle; layerwise identical for nshards 1 and cfg's nshards."""
    c = cfg
    stride = (c["Hq"] + 2 * c["Hk"]) * c["D"] + c["pad"]
    kw = dict(dtype=c["dtype"], seed=c["seed"], eps=c["eps"], row_stride=stride,
              scale=None if c["eps"] == 0.0 else "stress")
    ph = synth.make_case(c["T"], c["Hq"], c["Hk"], c["D"], **kw)
    full_parity(ph, "per_head", what="random per-head %s" % c)
    lw = synth.make_case(c["T"], c["Hq"], c["Hk"], c["D"], layerwise=True, **kw)
    try:
        a, _ = full_parity(lw, "layerwise", c["ns"], what="random layerwise %s" % c)
    except qkn.QKNormError as e:  # a token too wide for any launch shape
        assert e.status == -5, e
        return
    b, _ = full_parity(lw, "layerwise", 1, what="random layerwise n=1 %s" % c)
    assert np.array_equal(a, b), "layerwise output depends on nshards"
