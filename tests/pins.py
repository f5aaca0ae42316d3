"""Checks that pin the float64 oracle to facts outside itself.

Every ``pin_*`` function takes an oracle object (methods ``per_head``,
``layerwise``, ``layerwise_sharded`` with the signatures of
``oracle.Oracle``) and raises ``AssertionError`` when the oracle disagrees
with:

* hand-derived closed forms (``tests/golden/closed_forms.json``);
* invariants the RMSNorm definition implies (SwiftQK review,
  ``core_discovery``): unit RMS of the un-weighted output, invariance under
  ``x -> c*x, eps -> c^2*eps``, odd symmetry, permutation equivariance;
* the epsilon branch (all-zero rows give zeros; one spike gives
  ``sqrt(L) * g``);
* a library routine: with ``eps = 0``, ``y = x * g * sqrt(L) / ||x||_2``
  using ``numpy.linalg.norm``;
* brute force with plain Python loops on tiny fused buffers;
* the scalar-statistics decomposition (SwiftQK abstract and review
  ``key_machinery``): sharded partial sums plus a scalar combine equal the
  unsharded norm.

``tests/test_oracle_pins.py`` runs them on the committed oracle and
``tests/test_oracle_mutants.py`` shows each planted mistake fails one.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "closed_forms.json")
FP32 = "fp32"
BF16 = "bf16"


def _close(a, b, rel=1e-12, abs_=1e-300, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    err = np.abs(a - b)
    bound = rel * np.maximum(np.abs(a), np.abs(b)) + abs_
    bad = ~(err <= bound)
    assert not bad.any(), "%s: max err %g at %s" % (what, err.max(), np.argwhere(bad)[:4].tolist())


def _eval(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"sqrt": math.sqrt}))


def _rand(rng, T, stride):
    return rng.standard_normal((T, stride)).astype(np.float32)


def _gam(rng, n):
    return (1.0 + 0.25 * rng.standard_normal(n)).astype(np.float32)


# --------------------------------------------------------------------------
def pin_closed_forms(o):
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        x = np.asarray(c["x"], dtype=np.float32)
        gk = None if c["gamma_k"] is None else np.asarray(c["gamma_k"], dtype=np.float32)
        gq = np.asarray(c["gamma_q"], dtype=np.float32)
        args = (x, FP32, c["T"], c["Hq"], c["Hk"], c["D"], c["row_stride"], gq, gk, c["eps"])
        want = np.array([_eval(e) for e in c["expect"]])
        if c["kind"] == "per_head":
            outs = [o.per_head(*args)]
        elif c["kind"] == "layerwise":
            outs = [o.layerwise(*args)]
        else:
            outs = [o.layerwise_sharded(*args, n) for n in c["nshards"]]
        for y in outs:
            _close(y.ravel(), want, rel=1e-14, abs_=0.0, what=c["name"])


def pin_bf16_widening(o):
    # 0x4040 = 3.0, 0x4080 = 4.0, 0xC000 = -2.0, 0x3F80 = 1.0 as bfloat16 bits.
    x = np.array([0x4040, 0x4080, 0xC000, 0x3F80], dtype=np.uint16)
    y = o.per_head(x, BF16, 1, 2, 0, 2, 4, np.ones(2, np.float32), None, 0.0)
    _close(y.ravel(), [3 / math.sqrt(12.5), 4 / math.sqrt(12.5), -2 / math.sqrt(2.5),
                       1 / math.sqrt(2.5)], rel=1e-14, abs_=0.0, what="bf16 widening")


def pin_low_precision_widening(o):
    """fp16 bits and FP8 E4M3 codes reach the oracle as their exact values:
    a one-head row with eps = 0 and the value 2^k at one spot maps to
    sqrt(D) * g there, so a wrong decode of that spot would show; every code
    is also checked through the oracle's input path against torch's decode."""
    import torch

    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    finite = ~np.isnan(ref)
    D = 256
    x = codes.reshape(1, D)
    x = np.where(finite.reshape(1, D), x, np.uint8(0))  # replace the NaN codes by +0
    got = o.per_head(x, "fp8_e4m3", 1, 1, 0, D, D, np.ones(D, np.float32), None, 0.0)
    want = np.where(finite, ref, 0.0)
    _close(got.ravel(), want * math.sqrt(D) / np.linalg.norm(want), rel=1e-14, abs_=0.0,
           what="e4m3 widening")
    h = np.array([0x3C00, 0xC000, 0x0001, 0x7BFF], dtype=np.uint16)  # 1, -2, 2^-24, 65504
    y = o.per_head(h, "fp16", 1, 1, 0, 4, 4, np.ones(4, np.float32), None, 0.0)
    v = np.array([1.0, -2.0, 2.0 ** -24, 65504.0])
    _close(y.ravel(), v * 2.0 / np.linalg.norm(v), rel=1e-14, abs_=0.0, what="fp16 widening")


def pin_unit_rms(o):
    rng = np.random.default_rng(11)
    T, Hq, Hk, D = 5, 3, 2, 16
    stride = (Hq + 2 * Hk) * D
    x = _rand(rng, T, stride)
    xd = x.astype(np.float64)
    ones_d, ones_q, ones_k = (np.ones(n, np.float32) for n in (D, Hq * D, Hk * D))
    for eps in (0.0, 0.3):
        y = o.per_head(x, FP32, T, Hq, Hk, D, stride, ones_d, ones_d, eps)
        for t in range(T):
            for h in range(Hq + Hk):
                sl = slice(h * D, (h + 1) * D)
                m = np.mean(xd[t, sl] ** 2)
                _close(np.mean(y[t, sl] ** 2), m / (m + eps), what="per-head unit rms")
        y = o.layerwise(x, FP32, T, Hq, Hk, D, stride, ones_q, ones_k, eps)
        for t in range(T):
            for sl in (slice(0, Hq * D), slice(Hq * D, (Hq + Hk) * D)):
                m = np.mean(xd[t, sl] ** 2)
                _close(np.mean(y[t, sl] ** 2), m / (m + eps), what="layerwise unit rms")


def pin_scale_invariance(o):
    rng = np.random.default_rng(12)
    T, Hq, Hk, D = 4, 2, 1, 8
    stride = (Hq + 2 * Hk) * D
    x = _rand(rng, T, stride)
    gq, gk = _gam(rng, D), _gam(rng, D)
    lq, lk = _gam(rng, Hq * D), _gam(rng, Hk * D)
    qk = (Hq + Hk) * D
    for eps in (0.0, 0.7):
        base_ph = o.per_head(x, FP32, T, Hq, Hk, D, stride, gq, gk, eps)
        base_lw = o.layerwise(x, FP32, T, Hq, Hk, D, stride, lq, lk, eps)
        for c in (2.0 ** -9, 4.0, 2.0 ** 7):  # powers of two: c*x is exact in fp32
            xs = (x * np.float32(c)).astype(np.float32)
            ph = o.per_head(xs, FP32, T, Hq, Hk, D, stride, gq, gk, eps * c * c)
            lw = o.layerwise(xs, FP32, T, Hq, Hk, D, stride, lq, lk, eps * c * c)
            _close(ph[:, :qk], base_ph[:, :qk], what="per-head scale invariance")
            _close(lw[:, :qk], base_lw[:, :qk], what="layerwise scale invariance")


def pin_eps_branch(o):
    rng = np.random.default_rng(13)
    T, Hq, Hk, D = 3, 2, 2, 8
    stride = (Hq + 2 * Hk) * D
    qk = (Hq + Hk) * D
    x = np.zeros((T, stride), np.float32)
    x[:, qk:] = 7.0
    gq, gk = _gam(rng, D), _gam(rng, D)
    for eps in (1e-6, 1e-5):
        y = o.per_head(x, FP32, T, Hq, Hk, D, stride, gq, gk, eps)
        assert np.all(y[:, :qk] == 0.0) and np.all(y[:, qk:] == 7.0), "zero rows"
        y = o.layerwise(x, FP32, T, Hq, Hk, D, stride, _gam(rng, Hq * D), _gam(rng, Hk * D), eps)
        assert np.all(y[:, :qk] == 0.0) and np.all(y[:, qk:] == 7.0), "zero rows"
    # one spike a at column j of a length-L row, eps = 0: |y_j| = sqrt(L) * |g_j|.
    x = np.zeros((1, stride), np.float32)
    x[0, 3] = -5.0
    x[0, Hq * D + D + 2] = 0.125
    y = o.per_head(x, FP32, 1, Hq, Hk, D, stride, gq, gk, 0.0)
    _close(y[0, 3], -math.sqrt(D) * float(gq[3]), what="per-head spike")
    _close(y[0, Hq * D + D + 2], math.sqrt(D) * float(gk[2]), what="per-head spike K")
    lq, lk = _gam(rng, Hq * D), _gam(rng, Hk * D)
    y = o.layerwise(x, FP32, 1, Hq, Hk, D, stride, lq, lk, 0.0)
    _close(y[0, 3], -math.sqrt(Hq * D) * float(lq[3]), what="layerwise spike")
    _close(y[0, Hq * D + D + 2], math.sqrt(Hk * D) * float(lk[D + 2]), what="layerwise spike K")


def pin_library_norm(o):
    rng = np.random.default_rng(14)
    T, Hq, Hk, D = 6, 4, 2, 16
    stride = (Hq + 2 * Hk) * D + 8
    x = _rand(rng, T, stride)
    xd = x.astype(np.float64)
    gq, gk = _gam(rng, D), _gam(rng, D)
    y = o.per_head(x, FP32, T, Hq, Hk, D, stride, gq, gk, 0.0)
    for t in range(T):
        for h in range(Hq + Hk):
            sl = slice(h * D, (h + 1) * D)
            g = (gq if h < Hq else gk).astype(np.float64)
            want = xd[t, sl] * g * math.sqrt(D) / np.linalg.norm(xd[t, sl])
            _close(y[t, sl], want, rel=1e-13, what="per-head vs numpy norm")
    lq, lk = _gam(rng, Hq * D), _gam(rng, Hk * D)
    y = o.layerwise(x, FP32, T, Hq, Hk, D, stride, lq, lk, 0.0)
    for t in range(T):
        for sl, g in ((slice(0, Hq * D), lq), (slice(Hq * D, (Hq + Hk) * D), lk)):
            L = sl.stop - sl.start
            want = xd[t, sl] * g.astype(np.float64) * math.sqrt(L) / np.linalg.norm(xd[t, sl])
            _close(y[t, sl], want, rel=1e-13, what="layerwise vs numpy norm")


def _brute(x, T, Hq, Hk, D, stride, gq, gk, eps, layerwise):
    """Plain Python loops over a flat list; math.fsum for the sums."""
    flat = [float(v) for v in np.asarray(x, dtype=np.float64).ravel()]
    out = list(flat)
    rows = []
    for t in range(T):
        if layerwise:
            rows.append((t * stride, Hq * D, [float(g) for g in gq]))
            if Hk:
                rows.append((t * stride + Hq * D, Hk * D, [float(g) for g in gk]))
        else:
            for h in range(Hq + Hk):
                g = gq if h < Hq else gk
                rows.append((t * stride + h * D, D, [float(v) for v in g]))
    for start, L, g in rows:
        vals = flat[start:start + L]
        denom = math.sqrt(math.fsum(v * v for v in vals) / L + eps)
        for j in range(L):
            out[start + j] = vals[j] * g[j] / denom
    return np.array(out).reshape(T, stride)


def pin_brute_force(o):
    rng = np.random.default_rng(15)
    for (T, Hq, Hk, D, pad) in ((3, 3, 2, 4, 3), (2, 1, 1, 8, 0), (4, 2, 0, 4, 1), (1, 4, 2, 2, 5)):
        stride = (Hq + 2 * Hk) * D + pad
        x = _rand(rng, T, stride)
        for eps in (0.0, 0.2):
            gq, gk = _gam(rng, D), (_gam(rng, D) if Hk else None)
            y = o.per_head(x, FP32, T, Hq, Hk, D, stride, gq, gk, eps)
            _close(y, _brute(x, T, Hq, Hk, D, stride, gq, gk, eps, False), rel=1e-13,
                   abs_=1e-300, what="per-head brute force")
            lq, lk = _gam(rng, Hq * D), (_gam(rng, Hk * D) if Hk else None)
            y = o.layerwise(x, FP32, T, Hq, Hk, D, stride, lq, lk, eps)
            _close(y, _brute(x, T, Hq, Hk, D, stride, lq, lk, eps, True), rel=1e-13,
                   abs_=1e-300, what="layerwise brute force")


def pin_sharding(o):
    rng = np.random.default_rng(16)
    for (Hq, Hk, D) in ((8, 8, 1), (8, 8, 2), (16, 8, 1), (8, 0, 2)):
        T = 3
        stride = (Hq + 2 * Hk) * D + 2
        x = _rand(rng, T, stride)
        lq, lk = _gam(rng, Hq * D), (_gam(rng, Hk * D) if Hk else None)
        for eps in (0.0, 1e-6, 0.5):
            ref = o.layerwise(x, FP32, T, Hq, Hk, D, stride, lq, lk, eps)
            for n in (1, 2, 4, 8):
                y = o.layerwise_sharded(x, FP32, T, Hq, Hk, D, stride, lq, lk, eps, n)
                _close(y, ref, rel=1e-12, what="sharded n=%d" % n)
    x = _rand(rng, 1, 24)
    for bad in (0, 3):
        try:
            o.layerwise_sharded(x, FP32, 1, 4, 2, 2, 24, _gam(rng, 8), _gam(rng, 4), 0.0, bad)
        except ValueError:
            continue
        raise AssertionError("nshards=%d accepted" % bad)


def pin_per_head_equals_layerwise_one_head(o):
    rng = np.random.default_rng(17)
    T, D = 5, 32
    stride = 3 * D + 4
    x = _rand(rng, T, stride)
    gq, gk = _gam(rng, D), _gam(rng, D)
    for eps in (0.0, 1e-3):
        a = o.per_head(x, FP32, T, 1, 1, D, stride, gq, gk, eps)
        b = o.layerwise(x, FP32, T, 1, 1, D, stride, gq, gk, eps)
        _close(a, b, rel=0.0, abs_=0.0, what="one head: per-head == layerwise")


def pin_symmetries(o):
    rng = np.random.default_rng(18)
    T, Hq, Hk, D = 3, 2, 2, 8
    stride = (Hq + 2 * Hk) * D
    x = _rand(rng, T, stride)
    lq, lk = _gam(rng, Hq * D), _gam(rng, Hk * D)
    gq, gk = _gam(rng, D), _gam(rng, D)
    qk = (Hq + Hk) * D
    for eps in (0.0, 0.1):
        a = o.per_head(x, FP32, T, Hq, Hk, D, stride, gq, gk, eps)
        b = o.per_head(-x, FP32, T, Hq, Hk, D, stride, gq, gk, eps)
        _close(b[:, :qk], -a[:, :qk], rel=0.0, abs_=0.0, what="odd symmetry")
        a = o.layerwise(x, FP32, T, Hq, Hk, D, stride, lq, lk, eps)
        perm = rng.permutation(Hq * D)
        xp = x.copy()
        xp[:, :Hq * D] = x[:, perm]
        b = o.layerwise(xp, FP32, T, Hq, Hk, D, stride, lq[perm], lk, eps)
        _close(b[:, :Hq * D], a[:, perm], rel=1e-13, what="permutation equivariance")


def pin_gamma_and_layout(o):
    rng = np.random.default_rng(19)
    T, Hq, Hk, D = 4, 3, 2, 8
    stride = (Hq + 2 * Hk) * D + 5
    qk = (Hq + Hk) * D
    x = _rand(rng, T, stride)
    gq = _gam(rng, D)
    a = o.per_head(x, FP32, T, Hq, Hk, D, stride, gq, gq, 0.01)
    b = o.per_head(x, FP32, T, Hq, Hk, D, stride, gq, (2 * gq).astype(np.float32), 0.01)
    _close(b[:, :Hq * D], a[:, :Hq * D], rel=0.0, abs_=0.0, what="Q uses gamma_q")
    _close(b[:, Hq * D:qk], 2 * a[:, Hq * D:qk], rel=1e-15, what="K uses gamma_k")
    assert np.array_equal(a[:, qk:], x[:, qk:].astype(np.float64)), "V/padding copied"
    lq, lk = _gam(rng, Hq * D), _gam(rng, Hk * D)
    c = o.layerwise(x, FP32, T, Hq, Hk, D, stride, lq, lk, 0.01)
    assert np.array_equal(c[:, qk:], x[:, qk:].astype(np.float64)), "V/padding copied"


ALL_PINS = [
    pin_closed_forms,
    pin_bf16_widening,
    pin_low_precision_widening,
    pin_unit_rms,
    pin_scale_invariance,
    pin_eps_branch,
    pin_library_norm,
    pin_brute_force,
    pin_sharding,
    pin_per_head_equals_layerwise_one_head,
    pin_symmetries,
    pin_gamma_and_layout,
]
