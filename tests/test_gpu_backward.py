"""bin_linear_w1a16_backward (the straight-through backward of FBI-linear)
on the GPU against the oracle, with the tolerances of tests/parity.py: the
whole of dx, dW and dalpha at sizes the oracle finishes in seconds (ragged M,
several tiles, the one-token and few-token forward paths that dx reuses),
sampled positions at the 7B MLP shape, and the argument checks."""
import numpy as np
import pytest
import torch

from parity import bf16_to_f64, ste_dalpha_bound, ste_dw_bound, ste_dx_bound

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bl():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_linear_layers_b200 as m
    return m


def _case(oracle, M, N, K, seed):
    import synthetic
    W = synthetic.weights(N, K, seed)
    x = synthetic.activations(M, K, seed)
    dy = synthetic.activations(M, N, seed + 7)
    packed, alpha = oracle.pack_fbi(W.numpy())
    return x, dy, packed, alpha


def _abs(bits):
    return np.abs((bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64))


def _check(got, ref, bound, what):
    err = np.abs(got - ref)
    bad = np.nonzero(err > bound)[0]
    assert bad.size == 0, f"{what}: {bad.size}/{err.size} outside; first {bad[0]}: got {got[bad[0]]} ref {ref[bad[0]]}"


FULL = [(1, 128, 128), (3, 256, 384), (17, 384, 256), (64, 128, 640), (100, 640, 512), (300, 256, 1024),
        (130, 1024, 256), (5, 384, 1152)]


@pytest.mark.parametrize("M,N,K", FULL)
def test_backward_full(bl, oracle, M, N, K):
    import synthetic
    x, dy, packed, alpha = _case(oracle, M, N, K, seed=M + N + K)
    xb, dyb = synthetic.bf16_bits(x), synthetic.bf16_bits(dy)
    dx_ref, dw_ref, da_ref = oracle.w1a16_backward(xb, packed, alpha, dyb, K)
    dp = torch.from_numpy(packed.view(np.int32)).cuda()
    da_dev = torch.from_numpy(alpha).cuda()
    dx, dw, da = bl.bin_linear_w1a16_backward(x.cuda(), dp, da_dev, dy.cuda())
    torch.cuda.synchronize()
    assert bl.device_error() == (0, 0)
    dya, xa = _abs(dyb), _abs(xb)
    ms, ks = np.meshgrid(np.arange(M), np.arange(K), indexing="ij")
    _check(bf16_to_f64(dx).ravel(), dx_ref.ravel(), ste_dx_bound(dya, alpha, dx_ref.ravel(), ms.ravel()), "dx")
    js, ks = np.meshgrid(np.arange(N), np.arange(K), indexing="ij")
    _check(dw.cpu().numpy().astype(np.float64).ravel(), dw_ref.ravel(),
           ste_dw_bound(dya, xa, alpha, dw_ref.ravel(), js.ravel(), ks.ravel()), "dw")
    _check(da.cpu().numpy().astype(np.float64), da_ref, ste_dalpha_bound(dya, xa, da_ref, np.arange(N)), "dalpha")


def test_backward_7b_mlp_sampled(bl, oracle):
    import synthetic
    M, N, K = 2048, 11008, 4096
    x, dy, packed, alpha = _case(oracle, M, N, K, seed=1)
    xb, dyb = synthetic.bf16_bits(x), synthetic.bf16_bits(dy)
    dp = torch.from_numpy(packed.view(np.int32)).cuda()
    dx, dw, da = bl.bin_linear_w1a16_backward(x.cuda(), dp, torch.from_numpy(alpha).cuda(), dy.cuda())
    torch.cuda.synchronize()
    assert bl.device_error() == (0, 0)
    rng = np.random.default_rng(5)
    dya, xa = _abs(dyb), _abs(xb)
    ms, ks = rng.integers(0, M, 1500), rng.integers(0, K, 1500)
    ref = oracle.w1a16_backward_at(xb, packed, alpha, dyb, K, "dx", ms, ks)
    _check(bf16_to_f64(dx)[ms, ks], ref, ste_dx_bound(dya, alpha, ref, ms), "dx")
    js, ks = rng.integers(0, N, 1500), rng.integers(0, K, 1500)
    ref = oracle.w1a16_backward_at(xb, packed, alpha, dyb, K, "dw", js, ks)
    _check(dw.cpu().numpy()[js, ks].astype(np.float64), ref, ste_dw_bound(dya, xa, alpha, ref, js, ks), "dw")
    js = rng.integers(0, N, 24)
    ref = oracle.w1a16_backward_at(xb, packed, alpha, dyb, K, "dalpha", js)
    _check(da.cpu().numpy()[js].astype(np.float64), ref, ste_dalpha_bound(dya, xa, ref, js), "dalpha")


def test_backward_parts_and_empty_batch(bl, oracle):
    import synthetic
    M, N, K = 40, 256, 256
    x, dy, packed, alpha = _case(oracle, M, N, K, seed=9)
    dp, da_dev = torch.from_numpy(packed.view(np.int32)).cuda(), torch.from_numpy(alpha).cuda()
    dx_all, dw_all, da_all = bl.bin_linear_w1a16_backward(x.cuda(), dp, da_dev, dy.cuda())
    dx_only, none_w, none_a = bl.bin_linear_w1a16_backward(x.cuda(), dp, da_dev, dy.cuda(), want_dw=False)
    none_x, dw_only, da_only = bl.bin_linear_w1a16_backward(x.cuda(), dp, da_dev, dy.cuda(), want_dx=False)
    torch.cuda.synchronize()
    assert none_w is None and none_a is None and none_x is None
    assert torch.equal(dx_all, dx_only) and torch.equal(dw_all, dw_only) and torch.equal(da_all, da_only)
    # no tokens: the weight and scale gradients are zero
    x0 = torch.empty((0, K), dtype=torch.bfloat16, device="cuda")
    dy0 = torch.empty((0, N), dtype=torch.bfloat16, device="cuda")
    _, dw0, da0 = bl.bin_linear_w1a16_backward(x0, dp, da_dev, dy0, want_dx=False,
                                               dw=torch.full((N, K), 7.0, device="cuda"),
                                               dalpha=torch.full((N,), 7.0, device="cuda"))
    torch.cuda.synchronize()
    assert torch.count_nonzero(dw0).item() == 0 and torch.count_nonzero(da0).item() == 0
    assert bl.device_error() == (0, 0)


def test_backward_shape_checks(bl):
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    dy = torch.zeros((4, 192), dtype=torch.bfloat16, device="cuda")
    p = torch.zeros((192, 8), dtype=torch.int32, device="cuda")
    a = torch.zeros(192, dtype=torch.float32, device="cuda")
    with pytest.raises(RuntimeError):
        bl.bin_linear_w1a16_backward(x, p, a, dy)  # N % 128 != 0
