"""bitlinear_w1a8_noalloc: BitLinear for callers that cannot allocate.

Some users of this library call the layer from places where they may not
allocate device memory: an operator inside a host framework that gets only
its inputs and outputs, or a serving loop whose memory is planned once and
which must not call cudaMalloc while it runs. For them the library keeps the
layer's scratch (int8 codes and per-token gamma) in a fixed array of its own.

These tests call that entry point through the C ABI and compare it with the
workspace-taking bitlinear_w1a8 on two calls in a row, within the W1A8
output tolerance the other parity tests use. This file is named so pytest
collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity import W1A8_ULPS, f32_ulp_diff


def test_noalloc_rejects_problems_beyond_its_scratch():
    import bit_linear_layers_b200 as bl
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    M, N, K = 2048, 128, 4096        # 8 MiB of codes > the 4 MiB scratch
    assert bl.workspace_bytes(bl.BL_OP_W1A8, M, N, K) > bl.W1A8_NOALLOC_SCRATCH_BYTES
    assert bl.lib.bitlinear_w1a8_noalloc(fake, fake, fake, fake, M, N, K, None) == bl.BL_ERR_SCRATCH_LIMIT
    assert "scratch" in bl.status_string(bl.BL_ERR_SCRATCH_LIMIT)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_linear_layers_b200 as bl
    from bit_linear_layers_b200 import synthetic

    dev = torch.device("cuda", 0)
    # first a tensor-core-sized problem that fills most of the scratch, then a
    # small one that reuses it: the second call must not see the first's data
    cases = [(512, 2048, 5632, 4), (12, 384, 1024, 5)]
    inputs, outs = [], []
    for M, N, K, seed in cases:
        assert bl.workspace_bytes(bl.BL_OP_W1A8, M, N, K) <= bl.W1A8_NOALLOC_SCRATCH_BYTES
        W = synthetic.weights(N, K, seed, mean=0.001).to(dev)
        packed, _, beta = bl.bin_pack(W, bl.BL_PACK_BITNET)
        x = synthetic.laplace_channel_activations(M, K, seed).to(dev)
        inputs.append((x, packed, beta))
    for x, packed, beta in inputs:  # two calls in a row
        outs.append(bl.bitlinear_w1a8_noalloc(x, packed, beta))
    for (x, packed, beta), y in zip(inputs, outs):
        y_ref = bl.bitlinear_w1a8(x, packed, beta)
        torch.cuda.synchronize()
        ulps = f32_ulp_diff(y.cpu().numpy(), y_ref.cpu().numpy())
        assert ulps.max() <= W1A8_ULPS, f"max {ulps.max()} ulp from bitlinear_w1a8"
        assert np.isfinite(y.cpu().numpy()).all()
    assert bl.device_error() == (0, 0)
