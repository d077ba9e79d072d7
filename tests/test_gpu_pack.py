"""bin_pack on the GPU against the oracle: packed signs bit-exact, scales
within 1 fp32 ulp (tolerances in tests/parity.py)."""
import numpy as np
import pytest
import torch

from parity import f32_ulp_diff, u32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bl():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_linear_layers_b200 as m
    return m


def _weights(N, K, seed, mean=0.0):
    import synthetic
    return synthetic.weights(N, K, seed, mean=mean)


@pytest.mark.parametrize("N,K", [(1, 128), (37, 256), (300, 4096), (4096, 4096), (5, 11008),
                                 (1000, 640), (11008, 384)])
def test_pack_fbi(bl, oracle, N, K):
    W = _weights(N, K, seed=N * 7 + K)
    W[0, :3] = 0.0  # Sign(0) = -1
    if N > 1:
        W[1, :2] = -0.0
    packed, alpha = bl.bin_pack(W.cuda(), bl.BL_PACK_FBI)
    torch.cuda.synchronize()
    ref_packed, ref_alpha = oracle.pack_fbi(W.numpy())
    assert np.array_equal(u32(packed), ref_packed)
    assert f32_ulp_diff(alpha.cpu().numpy(), ref_alpha).max() <= 1


@pytest.mark.parametrize("N,K,mean", [(4, 128, 0.001), (256, 256, 0.0), (2048, 5632, 0.001),
                                      (5632, 2048, 0.001), (33, 1024, -0.01)])
def test_pack_bitnet(bl, oracle, N, K, mean):
    W = _weights(N, K, seed=N + 3 * K, mean=mean)
    packed, alpha, beta = bl.bin_pack(W.cuda(), bl.BL_PACK_BITNET)
    torch.cuda.synchronize()
    ref_packed, ref_a, ref_b = oracle.pack_bitnet(W.numpy())
    got = u32(packed)
    mism = np.nonzero(got != ref_packed)
    assert mism[0].size == 0, f"{mism[0].size} words differ"
    assert f32_ulp_diff(alpha.cpu().numpy(), np.float32(ref_a)).max() <= 1
    assert f32_ulp_diff(beta.cpu().numpy(), np.float32(ref_b)).max() <= 1


def test_pack_bitnet_weight_equal_to_mean(bl, oracle):
    # every row has entries equal to the global mean: those must pack as -1
    W = torch.tensor([[1.0, 2.0, 3.0, 2.0] * 32, [2.0, 0.0, 4.0, 2.0] * 32], dtype=torch.float32)
    packed, alpha, beta = bl.bin_pack(W.cuda(), bl.BL_PACK_BITNET)
    ref_packed, ref_a, ref_b = oracle.pack_bitnet(W.numpy())
    assert ref_a == 2.0 and alpha.item() == 2.0
    assert np.array_equal(u32(packed), ref_packed)


def test_pack_guard_bands(bl):
    from parity import guarded_empty, guards_intact
    N, K = 129, 384
    W = _weights(N, K, 5).cuda()
    packed, pbuf, ps = guarded_empty((N, K // 32), torch.int32, "cuda")
    alpha, abuf, as_ = guarded_empty((N,), torch.float32, "cuda")
    bl.bin_pack(W, bl.BL_PACK_FBI, packed=packed, alpha=alpha)
    torch.cuda.synchronize()
    assert guards_intact(pbuf, packed.numel(), sentinel=ps)
    assert guards_intact(abuf, alpha.numel(), sentinel=as_)
    assert bl.device_error() == (0, 0)
