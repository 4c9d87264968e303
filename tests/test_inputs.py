"""The seeded input generator: deterministic, the stated distributions, exact bf16 rounding."""

import numpy as np
import torch

import flashnorm_inputs as I


def test_deterministic_and_keyed_by_seed():
    a = I.activations(8, 64, 123)
    b = I.activations(8, 64, 123)
    c = I.activations(8, 64, 124)
    assert a.dtype == np.uint16 and a.shape == (8, 64)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)
    # different tensors of the same seed draw from different streams
    assert not np.array_equal(I.gain(64, 5), I.gain(64, 5, tag="g2"))


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    f = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(I.f32_to_bf16_bits(f), ref)


def test_distributions():
    d = 4096
    g = I.bf16_bits_to_f32(I.gain(d, 1))
    assert g.min() >= 0.5 and g.max() <= 1.5 and abs(g.mean() - 1.0) < 0.02
    w = I.bf16_bits_to_f32(I.weight(d, 256, 1)).astype(np.float64)
    assert abs(w.std() * np.sqrt(d) - 1.0) < 0.01 and abs(w.mean()) < 1e-3
    x = I.bf16_bits_to_f32(I.activations(2000, 256, 1)).astype(np.float64)
    rms = np.sqrt(np.mean(x * x, axis=1))
    # per-row scale is log-uniform on [0.1, 10]: log10(rms) roughly uniform on [-1, 1]
    lr = np.log10(rms)
    assert lr.min() > -1.2 and lr.max() < 1.2
    assert abs(np.mean(lr)) < 0.06 and abs(np.std(lr) - 2 / np.sqrt(12)) < 0.05


def test_workloads_table():
    wl = I.WORKLOADS["smollm2_ffn_m8192"]
    assert wl.kind == "glu" and wl.w_cols == 3072 and wl.flops == 2 * 8192 * 576 * 3072
    assert I.WORKLOADS["mla_latent_m2048"].head_dim == 512
    small = I.WORKLOADS["smollm2_qkv_m64"].draw()
    assert small["x"].shape == (64, 576) and small["w"].shape == (576, 960) and small["g"].shape == (576,)
