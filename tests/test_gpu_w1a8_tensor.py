"""Per-tensor activation quantisers of the "BitNet b1.58" page, section 1, on
the GPU against the oracle: Eq.(5) with gamma taken over the whole LN output
of the matrix, and Eq.(6), which shifts by the matrix's smallest LN value and
codes into [0, 127]. Both with +-1 (BitNet) and ternary (b1.58) weights,
through bitlinear_w1a8_ex. Levels as in the per-token tests: codes and gamma
against the oracle's quantiser (codes may differ by one only at a .5 tie),
int32 accumulators bit-exact against the oracle's product of the GPU's own
codes, fp32 outputs within 2 ulp of the oracle's fp64 value."""
import numpy as np
import pytest
import torch

from parity import TIE_BAND, W1A8_ULPS, f32_ulp_diff, gamma_rel_bound, sample_positions

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bl():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_linear_layers_b200 as m
    return m


def _check_codes(oracle, xb, mode, xq_gpu, gamma_gpu):
    xq_ref, gamma_ref, eta, pre = oracle.ln_quant_tensor(xb, mode, want_pre=True)
    diff = np.nonzero(xq_gpu != xq_ref)
    if diff[0].size:
        p = pre[diff]
        dist = np.abs(np.abs(p - np.floor(p)) - 0.5)
        assert np.all(dist <= TIE_BAND), f"{diff[0].size} codes differ away from a .5 tie"
        assert np.all(np.abs(xq_gpu[diff].astype(int) - xq_ref[diff].astype(int)) == 1)
    assert np.all(gamma_gpu == gamma_gpu[0]), "gamma is not shared by every token"
    rel = abs(gamma_gpu[0] - gamma_ref[0]) / max(abs(gamma_ref[0]), 1e-300)
    assert rel <= gamma_rel_bound(xb.shape[1]) or gamma_gpu[0] == gamma_ref[0], rel
    lo = 0 if mode == 1 else -127
    assert xq_gpu.min() >= lo and xq_gpu.max() <= 127
    if mode == 1 and gamma_ref[0] != 0.0:
        assert xq_gpu.min() == 0 and xq_gpu.max() == 127  # eta maps to 0, the largest LN to Q_b
    return xq_ref, gamma_ref, diff[0].size


def _run(bl, oracle, M, N, K, seed, mode, ternary, full=True, x=None):
    import synthetic
    W = synthetic.weights(N, K, seed, mean=0.001)
    if x is None:
        x = synthetic.laplace_channel_activations(M, K, seed)
    if ternary:
        packed, beta = oracle.pack_ternary(W.numpy())
        acc_fn, acc_at = oracle.w158a8_acc, oracle.w158a8_acc_at
    else:
        packed, _, beta = oracle.pack_bitnet(W.numpy())
        acc_fn, acc_at = oracle.w1a8_acc, oracle.w1a8_acc_at
    beta32 = np.float32(beta)
    xb = synthetic.bf16_bits(x)
    flags = (bl.BL_W1A8_NONNEG if mode == 1 else bl.BL_W1A8_PER_TENSOR) | (bl.BL_W1A8_TERNARY if ternary else 0)
    dp = torch.from_numpy(packed.view(np.int32)).cuda()
    dbeta = torch.tensor([beta32], dtype=torch.float32, device="cuda")
    y, xq, gamma, acc = bl.bitlinear_w1a8_ex(x.cuda(), dp, dbeta, flags, debug=True)
    y_plain = bl.bitlinear_w1a8_ex(x.cuda(), dp, dbeta, flags)
    torch.cuda.synchronize()
    assert torch.equal(y, y_plain), "debug and plain calls disagree"
    xq_g, gamma_g, acc_g, y_g = xq.cpu().numpy(), gamma.cpu().numpy(), acc.cpu().numpy(), y.cpu().numpy()
    xq_ref, gamma_ref, n_tie = _check_codes(oracle, xb, mode, xq_g, gamma_g)
    if full:
        ms, js = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
        ms, js = ms.ravel(), js.ravel()
        acc_own = acc_fn(xq_g, packed, K).ravel()
        acc_ref = acc_fn(xq_ref, packed, K).ravel() if n_tie else acc_own
    else:
        ms, js = sample_positions(M, N, 4000, seed=seed)
        acc_own = acc_at(xq_g, packed, K, ms, js)
        acc_ref = acc_at(xq_ref, packed, K, ms, js) if n_tie else acc_own
    assert np.array_equal(acc_g[ms, js].astype(np.int64), acc_own), "int32 accumulators not bit-exact"
    # Eq.(7) as printed: y = acc * beta * gamma / Q_b, for Eq.(6) codes too
    y_ref = acc_ref.astype(np.float64) * float(beta32) * gamma_ref[ms] / 128.0
    ulps = f32_ulp_diff(y_g[ms, js], y_ref.astype(np.float32))
    assert ulps.max() <= W1A8_ULPS, f"max {ulps.max()} ulp"
    return xq_g


# decode GEMV (M <= 16), split and unsplit tensor-core tiles, ragged M and N
FULL = [(1, 128, 128), (5, 200, 384), (16, 129, 256), (48, 700, 384), (130, 257, 640), (300, 1000, 1024),
        (12, 300, 2048)]


@pytest.mark.parametrize("ternary", [False, True], ids=["pm1", "ternary"])
@pytest.mark.parametrize("mode", [0, 1], ids=["eq5_tensor", "eq6_nonneg"])
@pytest.mark.parametrize("M,N,K", FULL)
def test_tensor_quant_full(bl, oracle, M, N, K, mode, ternary):
    _run(bl, oracle, M, N, K, seed=M * 7 + N + K + mode, mode=mode, ternary=ternary)


@pytest.mark.parametrize("ternary", [False, True], ids=["pm1", "ternary"])
@pytest.mark.parametrize("mode", [0, 1], ids=["eq5_tensor", "eq6_nonneg"])
def test_tensor_quant_1p3b_shapes_sampled(bl, oracle, mode, ternary):
    """The 1.3B projection shapes the W1A8 bench times (512 tokens, 2048 -> 5632)."""
    _run(bl, oracle, 512, 5632, 2048, seed=11 + mode, mode=mode, ternary=ternary, full=False)


def test_per_tensor_gamma_differs_from_per_token(bl, oracle):
    """One token is a single spike, whose LN peak sqrt(K - 1) is the largest
    any token can have: it sets the shared gamma, so no other token reaches
    code 127 (under a per-token gamma every token does)."""
    import synthetic
    M, K = 4, 512
    x = synthetic.laplace_channel_activations(M, K, 3)
    x[1] = 0.0
    x[1, 7] = 1.0
    xq = _run(bl, oracle, M, 128, K, seed=5, mode=0, ternary=False, x=x)
    peaks = np.abs(xq.astype(int)).max(axis=1)
    assert peaks[1] == 127 and np.all(np.delete(peaks, 1) < 127), peaks


@pytest.mark.parametrize("mode", [0, 1], ids=["eq5_tensor", "eq6_nonneg"])
def test_constant_rows_give_zero(bl, mode):
    """A matrix of constant rows has LN == 0 everywhere: gamma = 0, every code
    and output 0 (no division by zero)."""
    M, N, K = 3, 128, 256
    x = torch.ones((M, K), dtype=torch.bfloat16, device="cuda") * torch.tensor([[1.0], [-2.0], [0.25]],
                                                                               dtype=torch.bfloat16, device="cuda")
    packed = torch.randint(-2**31, 2**31 - 1, (N, K // 32), dtype=torch.int32, device="cuda")
    beta = torch.tensor([0.02], dtype=torch.float32, device="cuda")
    flags = bl.BL_W1A8_NONNEG if mode else bl.BL_W1A8_PER_TENSOR
    y, xq, gamma, acc = bl.bitlinear_w1a8_ex(x, packed, beta, flags, debug=True)
    torch.cuda.synchronize()
    assert torch.count_nonzero(xq).item() == 0 and torch.count_nonzero(acc).item() == 0
    assert torch.count_nonzero(gamma).item() == 0 and torch.count_nonzero(y).item() == 0


def test_no_quant_flag_matches_plain_entry(bl):
    """Without a quantiser flag bitlinear_w1a8_ex is bitlinear_w1a8 / w158a8."""
    import synthetic
    M, N, K = 37, 300, 512
    x = synthetic.laplace_channel_activations(M, K, 9).cuda()
    packed = torch.randint(-2**31, 2**31 - 1, (N, K // 32), dtype=torch.int32, device="cuda")
    packed3 = torch.randint(-2**31, 2**31 - 1, (N, K // 16), dtype=torch.int32, device="cuda")
    beta = torch.tensor([0.02], dtype=torch.float32, device="cuda")
    assert torch.equal(bl.bitlinear_w1a8_ex(x, packed, beta, 0), bl.bitlinear_w1a8(x, packed, beta))
    assert torch.equal(bl.bitlinear_w1a8_ex(x, packed3, beta, bl.BL_W1A8_TERNARY),
                       bl.bitlinear_w158a8(x, packed3, beta))
