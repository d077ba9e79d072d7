"""bitlinear_w1a8_noalloc: BitLinear for callers that cannot allocate.

Some users of this library call the layer from places where they may not
allocate device memory: an operator inside a host framework that gets only
its inputs and outputs, or a serving loop whose memory is planned once and
which must not call cudaMalloc while it runs. For them the library keeps the
layer's scratch (int8 codes and per-token gamma) in a fixed array of its own.

These tests call that entry point through the C ABI on two calls in a row
and require its outputs to be bit-identical to the workspace-taking
bitlinear_w1a8 (both run the same kernels on the same codes, so any
difference would be stale or overwritten scratch), and check both against the
oracle: codes and gamma against its LN/quantisation, int32 accumulators
bit-exact against its integer product of the GPU's codes, outputs within the
2-ulp W1A8 tolerance. This file is named so pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity import TIE_BAND, W1A8_ULPS, f32_ulp_diff, gamma_rel_bound, sample_positions


def test_noalloc_rejects_problems_beyond_its_scratch():
    import bit_linear_layers_b200 as bl
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    M, N, K = 2048, 128, 4096        # 8 MiB of codes > the 4 MiB scratch
    assert bl.workspace_bytes(bl.BL_OP_W1A8, M, N, K) > bl.W1A8_NOALLOC_SCRATCH_BYTES
    assert bl.lib.bitlinear_w1a8_noalloc(fake, fake, fake, fake, M, N, K, None) == bl.BL_ERR_SCRATCH_LIMIT
    assert "scratch" in bl.status_string(bl.BL_ERR_SCRATCH_LIMIT)


def _check_against_oracle(oracle, x, packed, beta, y, xq, gamma, acc, full):
    """Codes, gamma, accumulators and outputs of one call against the oracle."""
    import synthetic
    M, K = x.shape
    N = packed.shape[0]
    xb = synthetic.bf16_bits(x.cpu())
    pk = packed.cpu().numpy().view(np.uint32)
    xq_g, gamma_g, acc_g, y_g = xq.cpu().numpy(), gamma.cpu().numpy(), acc.cpu().numpy(), y.cpu().numpy()
    xq_ref, gamma_ref, pre = oracle.ln_absmax_quant(xb, want_pre=True)
    diff = np.nonzero(xq_g != xq_ref)
    if diff[0].size:  # only at .5 ties, by one step
        p = pre[diff]
        assert np.all(np.abs(np.abs(p - np.floor(p)) - 0.5) <= TIE_BAND)
        assert np.all(np.abs(xq_g[diff].astype(int) - xq_ref[diff].astype(int)) == 1)
    rel = np.abs(gamma_g - gamma_ref) / np.maximum(np.abs(gamma_ref), 1e-300)
    assert np.all((rel <= gamma_rel_bound(K)) | (gamma_ref == gamma_g))
    if full:
        ms, js = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
        ms, js = ms.ravel(), js.ravel()
        acc_own = oracle.w1a8_acc(xq_g, pk, K).ravel()
        acc_ref = oracle.w1a8_acc(xq_ref, pk, K).ravel()
    else:
        ms, js = sample_positions(M, N, 3000, seed=M)
        acc_own = oracle.w1a8_acc_at(xq_g, pk, K, ms, js)
        acc_ref = oracle.w1a8_acc_at(xq_ref, pk, K, ms, js)
    assert np.array_equal(acc_g[ms, js].astype(np.int64), acc_own), "int32 accumulators not bit-exact"
    beta32 = float(beta.cpu().numpy()[0])
    y_ref = acc_ref.astype(np.float64) * beta32 * gamma_ref[ms] / 128.0
    ulps = f32_ulp_diff(y_g[ms, js], y_ref.astype(np.float32))
    assert ulps.max() <= W1A8_ULPS, f"max {ulps.max()} ulp from the oracle"


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls(oracle):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_linear_layers_b200 as bl
    import synthetic

    dev = torch.device("cuda", 0)
    # first a tensor-core-sized problem that fills most of the scratch, then a
    # small one that reuses it: the second call must not see the first's data
    cases = [(512, 2048, 5632, 4, False), (12, 384, 1024, 5, True)]
    inputs, outs = [], []
    for M, N, K, seed, _ in cases:
        assert bl.workspace_bytes(bl.BL_OP_W1A8, M, N, K) <= bl.W1A8_NOALLOC_SCRATCH_BYTES
        W = synthetic.weights(N, K, seed, mean=0.001).to(dev)
        packed, _, beta = bl.bin_pack(W, bl.BL_PACK_BITNET)
        x = synthetic.laplace_channel_activations(M, K, seed).to(dev)
        inputs.append((x, packed, beta))
    for x, packed, beta in inputs:  # two calls in a row
        outs.append(bl.bitlinear_w1a8_noalloc(x, packed, beta))
    torch.cuda.synchronize()
    outs = [y.clone() for y in outs]
    for (x, packed, beta), y, case in zip(inputs, outs, cases):
        y_ref = bl.bitlinear_w1a8(x, packed, beta)
        y_dbg, xq, gamma, acc = bl.bitlinear_w1a8_debug(x, packed, beta)
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref), "bitlinear_w1a8_noalloc differs from bitlinear_w1a8"
        assert torch.equal(y_dbg, y_ref)
        _check_against_oracle(oracle, x, packed, beta, y, xq, gamma, acc, full=case[4])
    assert bl.device_error() == (0, 0)
