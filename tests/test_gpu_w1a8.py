"""bitlinear_w1a8 on the GPU against the oracle (tolerances in tests/parity.py).

Two levels: (1) the int8 codes and gamma against the oracle's LN/quant, and
the int32 accumulators bit-exact against the oracle's integer dot product of
the GPU's own codes; (2) the fp32 outputs within 2 ulp of the oracle's
fp64 forward from its own codes and gamma."""
import numpy as np
import pytest
import torch

from parity import (TIE_BAND, W1A8_ULPS, f32_ulp_diff, gamma_rel_bound, guarded_empty, guards_intact,
                    sample_positions)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bl():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_linear_layers_b200 as m
    return m


def _case(M, N, K, seed, kind="laplace_channel", w_mean=0.001):
    import synthetic
    W = synthetic.weights(N, K, seed, mean=w_mean)
    x = synthetic.make_x(kind, M, K, seed)
    return W, x


def _check_codes(oracle, xb, xq_gpu, gamma_gpu):
    xq_ref, gamma_ref, pre = oracle.ln_absmax_quant(xb, want_pre=True)
    diff = np.nonzero(xq_gpu != xq_ref)
    if diff[0].size:
        p = pre[diff]
        dist = np.abs(np.abs(p - np.floor(p)) - 0.5)
        assert np.all(dist <= TIE_BAND), f"{diff[0].size} codes differ away from a .5 tie"
        assert np.all(np.abs(xq_gpu[diff].astype(int) - xq_ref[diff].astype(int)) == 1)
    rel = np.abs(gamma_gpu - gamma_ref) / np.maximum(np.abs(gamma_ref), 1e-300)
    assert np.all((rel <= gamma_rel_bound(xb.shape[1])) | (gamma_ref == gamma_gpu)), rel.max()
    return xq_ref, gamma_ref, diff[0].size


def _run(bl, oracle, M, N, K, seed, kind="laplace_channel", w_mean=0.001, full=True):
    import synthetic
    W, x = _case(M, N, K, seed, kind, w_mean)
    packed, a_g, beta = oracle.pack_bitnet(W.numpy())
    beta32 = np.float32(beta)
    xb = synthetic.bf16_bits(x)
    dp = torch.from_numpy(packed.view(np.int32)).cuda()
    dbeta = torch.tensor([beta32], dtype=torch.float32, device="cuda")
    y, xq, gamma, acc = bl.bitlinear_w1a8_debug(x.cuda(), dp, dbeta)
    y_plain = bl.bitlinear_w1a8(x.cuda(), dp, dbeta)
    torch.cuda.synchronize()
    assert torch.equal(y, y_plain), "debug and plain entry points disagree"
    xq_g, gamma_g, acc_g, y_g = xq.cpu().numpy(), gamma.cpu().numpy(), acc.cpu().numpy(), y.cpu().numpy()
    xq_ref, gamma_ref, n_tie = _check_codes(oracle, xb, xq_g, gamma_g)
    if full:
        ms, js = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
        ms, js = ms.ravel(), js.ravel()
        acc_own = oracle.w1a8_acc(xq_g, packed, K).ravel()
        acc_ref = oracle.w1a8_acc(xq_ref, packed, K).ravel() if n_tie else acc_own
    else:
        ms, js = sample_positions(M, N, 4000, seed=seed)
        acc_own = oracle.w1a8_acc_at(xq_g, packed, K, ms, js)
        acc_ref = oracle.w1a8_acc_at(xq_ref, packed, K, ms, js) if n_tie else acc_own
    got_acc = acc_g[ms, js].astype(np.int64)
    assert np.array_equal(got_acc, acc_own), "int32 accumulators not bit-exact"
    # outputs: oracle's fp64 forward from its own codes and gamma
    y_ref = (acc_ref.astype(np.float64) * float(beta32) * gamma_ref[ms] / 128.0)
    ulps = f32_ulp_diff(y_g[ms, js], y_ref.astype(np.float32))
    assert ulps.max() <= W1A8_ULPS, f"max {ulps.max()} ulp"
    return y_g, xq_g, gamma_g, acc_g


FULL = [(4, 256, 256), (1, 128, 128), (7, 200, 384), (16, 129, 256), (17, 300, 512),
        (130, 257, 640), (300, 1000, 1024), (512, 640, 2048),
        # many tiles, ragged in M and N
        (260, 9500, 128),
        # 64-token tiles split along K; 32-, 64- and 128-token tiles with more tiles than SMs
        (48, 700, 384), (20, 20000, 128), (40, 20000, 128), (100, 20000, 128),
        # decode batches past the one-launch path: the warp-MMA GEMV (K % 256 == 0, 1..16 tokens, slices
        # of 8..48 words, ragged row clusters) and the dp4a GEMV (K % 256 != 0)
        (1, 300, 2048), (4, 1000, 5632), (8, 64, 2048), (13, 513, 4096), (16, 5632, 2048), (16, 257, 12288),
        (3, 100, 1152)]


@pytest.mark.parametrize("M,N,K", FULL)
def test_w1a8_full(bl, oracle, M, N, K):
    _run(bl, oracle, M, N, K, seed=M * 17 + N + K)


def test_w1a8_single_layer_config(bl, oracle):
    # M=4, K=N=256, W ~ N(0, 0.02) seed 0, x ~ N(0,1)
    _run(bl, oracle, 4, 256, 256, seed=0, kind="gauss_plain", w_mean=0.0)


@pytest.mark.parametrize("M,N,K", [(512, 5632, 2048), (512, 2048, 5632)])
def test_w1a8_1p3b_sampled(bl, oracle, M, N, K):
    _run(bl, oracle, M, N, K, seed=4, full=False)


def test_w1a8_constant_and_alternating_tokens(bl, oracle):
    M, N, K = 20, 384, 256
    import synthetic
    x = synthetic.make_x("gauss_plain", M, K, 3)
    x[0] = 2.5                                     # constant token: gamma = 0
    x[1] = torch.tensor([1.0, -1.0] * (K // 2))    # alternating: codes +-127
    W = synthetic.weights(N, K, 3, mean=0.001)
    packed, _, beta = oracle.pack_bitnet(W.numpy())
    dp = torch.from_numpy(packed.view(np.int32)).cuda()
    dbeta = torch.tensor([np.float32(beta)], device="cuda")
    for m_tokens in (4, M):  # small-M kernel and tensor-core GEMM
        y, xq, gamma, acc = bl.bitlinear_w1a8_debug(x[:m_tokens].cuda(), dp, dbeta)
        torch.cuda.synchronize()
        assert gamma[0].item() == 0.0 and torch.all(xq[0] == 0) and torch.all(y[0] == 0)
        assert xq[1].tolist() == [127 if k % 2 == 0 else -127 for k in range(K)]
        alt = np.array([1 if k % 2 == 0 else -1 for k in range(K)])
        bits = ((packed[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(N, -1)[:, :K]
        want = 127 * ((2 * bits.astype(np.int64) - 1) @ alt)
        assert np.array_equal(acc[1].cpu().numpy(), want)


def test_w1a8_unit_codes_give_popcount(bl):
    # with the quantisation bypassed and every code 1: acc_j = #pos - #neg
    # (3 and 11 tokens: the warp-MMA GEMV's 8- and 16-token tiles; 150: the GEMM)
    import synthetic
    for M in (3, 11, 150):
        N, K = 300, 512
        W = synthetic.weights(N, K, 8).cuda()
        packed, _, beta = bl.bin_pack(W, bl.BL_PACK_BITNET)
        shift = W.double().mean()
        pos = (W.double() - shift > 0).sum(dim=1).cpu().numpy().astype(np.int64)
        xq_in = torch.ones((M, K), dtype=torch.int8, device="cuda")
        g_in = torch.ones(M, dtype=torch.float64, device="cuda")
        y, xq, gamma, acc = bl.bitlinear_w1a8_debug(None, packed, beta, xq_in=xq_in, gamma_in=g_in)
        torch.cuda.synchronize()
        assert np.array_equal(acc.cpu().numpy(), np.broadcast_to(2 * pos - K, (M, N)))


def test_w1a8_guard_bands_and_error_word(bl, oracle):
    M, N, K = 140, 300, 384
    import synthetic
    W, x = _case(M, N, K, 6)
    packed, _, beta = oracle.pack_bitnet(W.numpy())
    dp = torch.from_numpy(packed.view(np.int32)).cuda()
    dbeta = torch.tensor([np.float32(beta)], device="cuda")
    y, ybuf, sent = guarded_empty((M, N), torch.float32, "cuda")
    bl.bitlinear_w1a8(x.cuda(), dp, dbeta, out=y)
    torch.cuda.synchronize()
    assert guards_intact(ybuf, y.numel(), sentinel=sent)
    assert bl.device_error() == (0, 0)


def test_w1a8_end_to_end_pack_then_forward(bl, oracle):
    M, N, K = 200, 512, 1024
    import synthetic
    W, x = _case(M, N, K, 12)
    packed_ref, _, beta_ref = oracle.pack_bitnet(W.numpy())
    gp, ga, gb = bl.bin_pack(W.cuda(), bl.BL_PACK_BITNET)
    y = bl.bitlinear_w1a8(x.cuda(), gp, gb)
    torch.cuda.synchronize()
    y_ref, _, _, _ = oracle.w1a8(synthetic.bf16_bits(x), packed_ref, float(np.float32(beta_ref)), K)
    ulps = f32_ulp_diff(y.cpu().numpy(), y_ref.astype(np.float32))
    assert ulps.max() <= W1A8_ULPS + 1  # + the 1-ulp freedom of beta's fp32 rounding
