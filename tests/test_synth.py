"""Seeded input generator: determinism, storage rounding, workload recipe."""
import numpy as np
import torch

from attention_qk_norm_b200 import synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 100,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0, 0.0, 65504.0],
                                 dtype=np.float32)])
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_seeded_and_shaped():
    a = synth.make_case(8, 4, 2, 64, seed=3, row_stride=520)
    b = synth.make_case(8, 4, 2, 64, seed=3, row_stride=520)
    assert a.qkv.shape == (8, 520) and a.qkv.dtype == np.uint16
    assert np.array_equal(a.qkv, b.qkv) and np.array_equal(a.gamma_q, b.gamma_q)
    assert a.gamma_q.shape == (64,) and a.gamma_k.shape == (64,)
    c = synth.make_case(8, 4, 2, 64, seed=3, layerwise=True, dtype=synth.FP32)
    assert c.qkv.dtype == np.float32 and c.gamma_q.shape == (256,) and c.gamma_k.shape == (128,)


def test_stress_rows():
    T, Hq, Hk, D = 400, 4, 2, 16
    c = synth.make_case(T, Hq, Hk, D, seed=1, dtype=synth.FP32, scale="stress",
                        zero_frac=0.01, outlier_frac=0.01)
    qk = c.qkv[:, :(Hq + Hk) * D]
    zero_rows = np.where(~qk.any(axis=1))[0]
    assert zero_rows.size == 4
    assert np.count_nonzero(np.abs(qk) == 1e4) == 4
    assert c.qkv[:, (Hq + Hk) * D:].any()  # V keeps random values


def test_torch_generator_recipe():
    d = synth.make_case_torch(300, 4, 2, 16, device="cpu", seed=2, scale="stress",
                              zero_frac=0.01, outlier_frac=0.01)
    qk = d["qkv"][:, :96].float()
    assert int((qk == 0).all(dim=1).sum()) == 3
    assert int((qk.abs() > 9000).sum()) == 3  # 1e4 rounds to 9984 in bf16
    assert d["qkv"].dtype == torch.bfloat16 and d["gamma_q"].shape == (16,)
