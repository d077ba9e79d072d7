"""W1A1 XNOR/popcount products on the GPU ("BitNet-Transformers" page: 1-bit
operands reduce the product to XNOR / popcount) against the oracle's +-1 dot
products, which the oracle pins brute-force over small K. Integer results:
bit-exact."""
import numpy as np
import pytest
import torch

from parity import guarded_empty, guards_intact

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bl():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_linear_layers_b200 as m
    return m


def _rows(rng, R, K):
    return rng.integers(0, 2 ** 32, size=(R, K // 32), dtype=np.uint64).astype(np.uint32)


# one tile, ragged tiles in M and N, K of one, two and a partial 32-word chunk
@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (5, 7, 256), (64, 64, 128), (65, 130, 384),
                                   (200, 300, 1152), (256, 300, 2048), (3, 1000, 4096)])
def test_xnor_gemm(bl, oracle, M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    a, b = _rows(rng, M, K), _rows(rng, N, K)
    dot_ref = oracle.w1a1(a, b, K)
    out, buf, sent = guarded_empty((M, N), torch.int32, "cuda")
    bl.bin_xnor_gemm(torch.from_numpy(a.view(np.int32)).cuda(), torch.from_numpy(b.view(np.int32)).cuda(),
                     K, out=out)
    torch.cuda.synchronize()
    assert guards_intact(buf, out.numel(), sentinel=sent)
    assert np.array_equal(out.cpu().numpy().astype(np.int64), dot_ref)


def test_xnor_gemm_extremes_and_packed_activations(bl, oracle):
    # identical rows give +K, complementary rows -K; and activations packed by
    # bin_pack (sign of x, Sign(0) = -1) through the same path
    import synthetic
    K = 512
    rng = np.random.default_rng(3)
    a = _rows(rng, 4, K)
    b = np.concatenate([a, ~a], axis=0)
    got = bl.bin_xnor_gemm(torch.from_numpy(a.view(np.int32)).cuda(), torch.from_numpy(b.view(np.int32)).cuda(), K)
    torch.cuda.synchronize()
    g = got.cpu().numpy()
    assert np.all(np.diag(g[:, :4]) == K) and np.all(np.diag(g[:, 4:]) == -K)
    x = synthetic.activations(33, K, seed=5).float()
    W = synthetic.weights(70, K, seed=6)
    xa, _ = bl.bin_pack(x.cuda(), bl.BL_PACK_FBI)
    wb, _ = bl.bin_pack(W.cuda(), bl.BL_PACK_FBI)
    dot = bl.bin_xnor_gemm(xa, wb, K)
    torch.cuda.synchronize()
    xr, _ = oracle.pack_fbi(x.numpy())
    wr, _ = oracle.pack_fbi(W.numpy())
    assert np.array_equal(dot.cpu().numpy().astype(np.int64), oracle.w1a1(xr, wr, K))
    assert bl.device_error() == (0, 0)
