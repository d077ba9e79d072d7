"""Seeded synthetic inputs for the binarized linear layers.

This module only draws random numbers: it holds none of the layers'
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.
All draws use a CPU ``torch.Generator`` unless a device is named, so the
same seed gives the same tensors on every machine.

Workloads (shapes of the 130M / 1.3B / 7B models the FBI-LLM and BitNet
pages describe; value distributions are this library's choice since the
pages publish no data):

* weights   W ~ N(mean, std), fp32, row-major [N out, K in]
* decode / prefill activations x ~ N(0, 1) in bf16, with a seeded 1% of
  the K channels scaled by 20 for every token (outlier channels)
* BitNet activations x_mk = z_mk * c_k, z ~ N(0,1), c_k = 1 + Laplace(0, 0.5)
  drawn once per channel, rounded to bf16
"""
from __future__ import annotations

import torch


def _gen(seed: int, device: str | torch.device = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weights(N: int, K: int, seed: int, mean: float = 0.0, std: float = 0.02,
            device: str | torch.device = "cpu") -> torch.Tensor:
    """fp32 [N, K] with entries ~ N(mean, std)."""
    g = _gen(seed, device)
    w = torch.randn((N, K), generator=g, dtype=torch.float32, device=device)
    return w.mul_(std).add_(mean)


def activations(M: int, K: int, seed: int, outlier_frac: float = 0.01, outlier_scale: float = 20.0,
                device: str | torch.device = "cpu") -> torch.Tensor:
    """bf16 [M, K], N(0,1) with ``outlier_frac`` of the channels scaled by ``outlier_scale``."""
    g = _gen(seed + 7919, device)
    x = torch.randn((M, K), generator=g, dtype=torch.float32, device=device)
    n_out = int(round(outlier_frac * K))
    if n_out > 0:
        idx = torch.randperm(K, generator=g, device=device)[:n_out]
        x[:, idx] *= outlier_scale
    return x.to(torch.bfloat16)


def laplace_channel_activations(M: int, K: int, seed: int, b: float = 0.5,
                                device: str | torch.device = "cpu") -> torch.Tensor:
    """bf16 [M, K]: z * (1 + Laplace(0, b)) with one Laplace draw per channel."""
    g = _gen(seed + 104729, device)
    z = torch.randn((M, K), generator=g, dtype=torch.float32, device=device)
    u = torch.rand((K,), generator=g, dtype=torch.float64, device=device) - 0.5
    # inverse CDF of the Laplace distribution
    lap = -b * torch.sign(u) * torch.log1p(-2.0 * u.abs())
    c = (1.0 + lap).to(torch.float32)
    return (z * c).to(torch.bfloat16)


def bf16_bits(x: torch.Tensor):
    """Raw 16-bit patterns of a bf16 tensor as a numpy uint16 array (CPU)."""
    assert x.dtype == torch.bfloat16
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


# The five workloads, by what they are. Sizes are (M tokens, K in, N out).
WORKLOADS = {
    "w1a8_single_4x256x256": dict(kind="w1a8", shapes=[(4, 256, 256)], seed=0,
                                  w_mean=0.0, x="gauss_plain"),
    "w1a16_decode_1x4096x4096": dict(kind="w1a16", shapes=[(1, 4096, 4096)], seed=2,
                                     w_mean=0.0, x="gauss_outlier"),
    "w1a16_prefill_2048x4096x11008": dict(kind="w1a16",
                                          shapes=[(2048, 4096, 11008), (2048, 11008, 4096)],
                                          seed=1, w_mean=0.0, x="gauss_outlier"),
    "w1a8_1p3b_512x2048x5632": dict(kind="w1a8", shapes=[(512, 2048, 5632), (512, 5632, 2048)],
                                    seed=4, w_mean=0.001, x="laplace_channel"),
}

# one 7B-shaped decoder layer: q, k, v, o, gate, up, down as (K in, N out)
LLAMA7B_LAYER = [(4096, 4096), (4096, 4096), (4096, 4096), (4096, 4096),
                 (4096, 11008), (4096, 11008), (11008, 4096)]
LLAMA7B_LAYERS = 32


def make_x(kind: str, M: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    if kind == "gauss_outlier":
        return activations(M, K, seed, device=device)
    if kind == "gauss_plain":
        return activations(M, K, seed, outlier_frac=0.0, device=device)
    if kind == "laplace_channel":
        return laplace_channel_activations(M, K, seed, device=device)
    raise ValueError(kind)


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = ["weights", "activations", "laplace_channel_activations", "bf16_bits", "WORKLOADS",
           "LLAMA7B_LAYER", "LLAMA7B_LAYERS", "make_x", "ceil_div"]
