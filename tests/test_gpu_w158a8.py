"""BitNet b1.58 (ternary weights, "BitNet b1.58" page, section 2, Eq.(9)-(11))
on the GPU against the oracle: bin_pack(BL_PACK_TERNARY) bit-exact, and
bitlinear_w158a8 at the same two levels as the W1A8 tests (codes and gamma
against the oracle's LN/quant, int32 accumulators bit-exact against the
oracle's ternary product of the GPU's own codes, fp32 outputs within 2 ulp)."""
import numpy as np
import pytest
import torch

from parity import W1A8_ULPS, f32_ulp_diff, guarded_empty, guards_intact, sample_positions
from test_gpu_w1a8 import _check_codes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bl():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_linear_layers_b200 as m
    return m


@pytest.mark.parametrize("N,K", [(1, 128), (3, 256), (257, 384), (1000, 1024), (4096, 4096)])
def test_pack_ternary(bl, oracle, N, K):
    import synthetic
    W = synthetic.weights(N, K, seed=N + K, mean=0.001)
    packed_ref, gamma_ref = oracle.pack_ternary(W.numpy())
    packed, buf, sent = guarded_empty((N, K // 16), torch.int32, "cuda")
    got, beta = bl.bin_pack(W.cuda(), bl.BL_PACK_TERNARY, packed=packed)
    torch.cuda.synchronize()
    assert guards_intact(buf, packed.numel(), sentinel=sent)
    assert np.array_equal(got.cpu().numpy().view(np.uint32), packed_ref), "ternary planes differ"
    assert f32_ulp_diff(beta.cpu().numpy(), np.array([gamma_ref], np.float32)).max() <= 1
    # every value class occurs at this scale (W ~ N(0.001, 0.02): about 38% zeros)
    planes = packed_ref.reshape(N, -1, 8)
    if N * K >= 4096:
        nz = np.unpackbits(planes[:, :, :4].view(np.uint8)).sum() + np.unpackbits(planes[:, :, 4:].view(np.uint8)).sum()
        assert 0 < nz < N * K


def _run(bl, oracle, M, N, K, seed, full=True):
    import synthetic
    W = synthetic.weights(N, K, seed, mean=0.001)
    x = synthetic.laplace_channel_activations(M, K, seed)
    packed, gamma_w = oracle.pack_ternary(W.numpy())
    beta32 = np.float32(gamma_w)
    xb = synthetic.bf16_bits(x)
    dp = torch.from_numpy(packed.view(np.int32)).cuda()
    dbeta = torch.tensor([beta32], dtype=torch.float32, device="cuda")
    y, xq, gamma, acc = bl.bitlinear_w158a8_debug(x.cuda(), dp, dbeta)
    y_plain = bl.bitlinear_w158a8(x.cuda(), dp, dbeta)
    torch.cuda.synchronize()
    assert torch.equal(y, y_plain), "debug and plain entry points disagree"
    xq_g, gamma_g, acc_g, y_g = xq.cpu().numpy(), gamma.cpu().numpy(), acc.cpu().numpy(), y.cpu().numpy()
    xq_ref, gamma_ref, n_tie = _check_codes(oracle, xb, xq_g, gamma_g)
    if full:
        ms, js = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
        ms, js = ms.ravel(), js.ravel()
        acc_own = oracle.w158a8_acc(xq_g, packed, K).ravel()
        acc_ref = oracle.w158a8_acc(xq_ref, packed, K).ravel() if n_tie else acc_own
    else:
        ms, js = sample_positions(M, N, 4000, seed=seed)
        acc_own = oracle.w158a8_acc_at(xq_g, packed, K, ms, js)
        acc_ref = oracle.w158a8_acc_at(xq_ref, packed, K, ms, js) if n_tie else acc_own
    assert np.array_equal(acc_g[ms, js].astype(np.int64), acc_own), "int32 accumulators not bit-exact"
    y_ref = acc_ref.astype(np.float64) * float(beta32) * gamma_ref[ms] / 128.0
    ulps = f32_ulp_diff(y_g[ms, js], y_ref.astype(np.float32))
    assert ulps.max() <= W1A8_ULPS, f"max {ulps.max()} ulp"
    return y_g, acc_g


# decode GEMV (M <= 16) and every tensor-core configuration: 32/64/128-token
# tiles split and unsplit, 128x256 tiles, ragged M and N
FULL = [(1, 128, 128), (4, 256, 256), (7, 200, 384), (16, 129, 256), (17, 300, 512),
        (48, 700, 384), (130, 257, 640), (300, 1000, 1024), (20, 20000, 128), (100, 20000, 128),
        (260, 9500, 128),
        # warp-MMA GEMV (ternary planes, slices crossing 128-k blocks) and the dp4a GEMV
        (1, 300, 2048), (5, 700, 5632), (16, 257, 12288), (9, 100, 1152)]


@pytest.mark.parametrize("M,N,K", FULL)
def test_w158a8_full(bl, oracle, M, N, K):
    _run(bl, oracle, M, N, K, seed=M * 13 + N + K)


@pytest.mark.parametrize("M,N,K", [(512, 5632, 2048), (512, 2048, 5632)])
def test_w158a8_1p3b_sampled(bl, oracle, M, N, K):
    _run(bl, oracle, M, N, K, seed=5, full=False)


@pytest.mark.parametrize("M,K", [(40, 640), (7, 768)])
def test_w158a8_unit_codes_give_plane_counts(bl, M, K):
    # codes all 1 (xq_in): acc_j = #(+1) - #(-1) of row j, from the planes
    # (7 tokens, K % 256 == 0: the warp-MMA GEMV; 40 tokens: the GEMM)
    import synthetic
    N = 700
    W = synthetic.weights(N, K, 9, mean=0.001, device="cuda")
    packed, beta = bl.bin_pack(W, bl.BL_PACK_TERNARY)
    xq = torch.ones((M, K), dtype=torch.int8, device="cuda")
    g = torch.ones(M, dtype=torch.float64, device="cuda")
    _, _, _, acc = bl.bitlinear_w158a8_debug(None, packed, beta, xq_in=xq, gamma_in=g)
    torch.cuda.synchronize()
    w = packed.cpu().numpy().view(np.uint32).reshape(N, -1, 8)
    plus = np.unpackbits(w[:, :, :4].copy().view(np.uint8), axis=None).reshape(N, -1).sum(axis=1)
    minus = np.unpackbits(w[:, :, 4:].copy().view(np.uint8), axis=None).reshape(N, -1).sum(axis=1)
    counts = plus.astype(np.int64) - minus.astype(np.int64)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), np.broadcast_to(counts, (M, N)))
    assert bl.device_error() == (0, 0)


def test_w158a8_end_to_end_pack_then_forward(bl, oracle):
    # bin_pack on the GPU feeding the forward, against the oracle's pack + forward
    import synthetic
    M, N, K = 64, 512, 1024
    W = synthetic.weights(N, K, 21, mean=0.001)
    x = synthetic.laplace_channel_activations(M, K, 21)
    packed, beta = bl.bin_pack(W.cuda(), bl.BL_PACK_TERNARY)
    y = bl.bitlinear_w158a8(x.cuda(), packed, beta)
    torch.cuda.synchronize()
    p_ref, g_ref = oracle.pack_ternary(W.numpy())
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_ref)
    y_ref, _, _, _ = oracle.w158a8(synthetic.bf16_bits(x), p_ref, float(np.float32(g_ref)), K)
    ulps = f32_ulp_diff(y.cpu().numpy(), y_ref.astype(np.float32))
    assert ulps.max() <= W1A8_ULPS + 1  # + the 1-ulp freedom of beta's fp32 rounding
