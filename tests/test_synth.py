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


def test_fp16_and_e4m3_rounding_match_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(50000).astype(np.float32) * 40,
                        rng.standard_normal(5000).astype(np.float32) * 1e-3,
                        np.array([448, 460, 463.9, -464 + 1e-3, 2 ** -9 * 0.5, 2 ** -9 * 1.5,
                                  2 ** -10 * 3, 0.0, -0.0, 65504.0], dtype=np.float32)])
    ref16 = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.f32_to_fp16_bits(x), ref16)
    finite = np.abs(x) < 464  # torch turns larger magnitudes into NaN; ours saturate
    ref8 = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(synth.f32_to_e4m3_bits(x)[finite], ref8[finite])
    assert np.all(synth.f32_to_e4m3_bits(np.array([500.0, -1e4], np.float32)) == [0x7E, 0xFE])


def test_low_precision_cases():
    c = synth.make_case(5, 4, 2, 64, dtype=synth.FP8, seed=2, scale="stress", outlier_frac=0.2)
    assert c.qkv.dtype == np.uint8 and c.qkv.shape == (5, 512)
    assert int(np.max(c.qkv & 0x7F)) <= 0x7E  # finite codes only
    c = synth.make_case(5, 4, 2, 64, dtype=synth.FP16, seed=2)
    assert c.qkv.dtype == np.uint16
    d = synth.make_case_torch(64, 4, 2, 64, device="cpu", dtype=synth.FP8, seed=3,
                              scale="stress", outlier_frac=0.05)
    assert d["qkv"].dtype == torch.float8_e4m3fn
    assert not torch.isnan(d["qkv"].float()).any()
