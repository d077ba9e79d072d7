"""The seeded input recipe (CPU): the generators are deterministic per seed,
have the documented shapes and dtypes, and draw the documented
distributions (weights N(mean, std); activations N(0, 1) with 1% of the
channels x20; BitNet activations z * (1 + Laplace(0, 0.5)) per channel)."""
import math

import numpy as np
import torch

import synthetic


def test_deterministic_per_seed_and_distinct_across_seeds():
    for fn in (lambda s: synthetic.weights(64, 256, s), lambda s: synthetic.activations(8, 512, s),
               lambda s: synthetic.laplace_channel_activations(8, 512, s)):
        a, b, c = fn(3), fn(3), fn(4)
        assert torch.equal(a, b) and not torch.equal(a, c)


def test_weights_moments():
    W32 = synthetic.weights(512, 1024, seed=1, mean=0.001, std=0.02)
    assert W32.dtype == torch.float32 and W32.shape == (512, 1024)
    W = W32.double()
    assert abs(W.mean().item() - 0.001) < 5e-5 and abs(W.std().item() - 0.02) < 2e-4


def test_activation_outlier_channels():
    K = 4096
    xb = synthetic.activations(256, K, seed=2)
    assert xb.dtype == torch.bfloat16 and xb.shape == (256, K)
    x = xb.float()
    rms = x.pow(2).mean(dim=0).sqrt()
    out = rms > 5.0  # x20 channels have rms ~20, the others ~1
    assert out.sum().item() == round(0.01 * K)
    assert abs(rms[out].mean().item() - 20.0) < 1.5 and abs(rms[~out].mean().item() - 1.0) < 0.05
    # the same channels are outliers for every token
    assert torch.all((x[:, out].abs().max(dim=0).values > 5.0))


def test_laplace_channel_scales():
    K = 8192
    x = synthetic.laplace_channel_activations(2048, K, seed=4).double().numpy()
    c = np.sqrt((x ** 2).mean(axis=0))  # per-channel |1 + Laplace(0, 0.5)| (z has unit variance)
    # E|1 + L| for L ~ Laplace(0, b=0.5): the scale's median is 1 and its spread matches b
    assert abs(np.median(c) - 1.0) < 0.05
    lap_abs_dev = np.median(np.abs(c - 1.0))  # median |L| = b ln 2 for the part with 1 + L > 0
    assert abs(lap_abs_dev - 0.5 * math.log(2.0)) < 0.05


def test_bf16_bits_round_trip():
    x = synthetic.activations(4, 256, seed=5)
    bits = synthetic.bf16_bits(x)
    back = torch.from_numpy((bits.astype(np.uint32) << 16).view(np.float32))
    assert bits.dtype == np.uint16 and torch.equal(back, x.float())
