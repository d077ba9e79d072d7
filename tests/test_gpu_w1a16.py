"""bin_linear_w1a16 on the GPU against the oracle (tolerance in tests/parity.py):
full comparison at sizes the oracle finishes in seconds (several tiles,
ragged tails in M and N, multi-chunk K), sampled comparison at the 7B
prefill sizes, plus edge cases."""
import numpy as np
import pytest
import torch

from parity import bf16_to_f64, check_w1a16, guarded_empty, guards_intact, sample_positions

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bl():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_linear_layers_b200 as m
    return m


def _case(M, N, K, seed):
    import synthetic
    W = synthetic.weights(N, K, seed)
    x = synthetic.activations(M, K, seed)
    return W, x


def _oracle_inputs(oracle, W, x):
    import synthetic
    packed, alpha = oracle.pack_fbi(W.numpy())
    return packed, alpha, synthetic.bf16_bits(x)


def _to_dev(packed, alpha, x):
    return (torch.from_numpy(packed.view(np.int32)).cuda(), torch.from_numpy(alpha).cuda(), x.cuda())


FULL = [
    # single-token lookup-table GEMV: cluster splits C=8 (1 and 3 pages), C=4, C=1, short rows,
    # ragged row clusters, and K with no split (falls back to the predicated GEMV)
    (1, 128, 128), (1, 4096, 4096), (1, 1000, 11008), (1, 257, 2048), (1, 300, 640), (1, 513, 5632),
    (1, 4099, 384), (1, 77, 8320),
    # 2..4 tokens with K % 256 != 0: predicated-add GEMV
    (2, 300, 384), (4, 129, 640),
    # 2..16 tokens, K % 256 == 0: warp-MMA GEMV (8- and 16-token tiles, 16- and 48-word slices,
    # slices shorter than a word group, ragged row clusters)
    (2, 1000, 4096), (3, 129, 256), (4, 1000, 11008), (4, 4099, 512), (6, 384, 256), (8, 1000, 4096), (9, 129, 2048), (12, 4099, 512), (16, 300, 4096), (16, 257, 11008),
    (7, 200, 12288), (13, 128, 8192),
    # tcgen05 GEMM path
    (5, 384, 384), (16, 128, 128), (17, 200, 384), (129, 383, 640), (256, 512, 1024),
    (300, 1000, 1024), (1000, 1100, 512),
    # enough tiles for the 128-row x 256-token configuration, ragged in M and N
    (300, 9100, 256),
    # 64-token tiles split along K; 32-, 64- and 128-token tiles with more tiles than SMs
    (48, 1000, 512), (20, 20000, 128), (40, 20000, 256), (100, 20000, 256),
]


@pytest.mark.parametrize("M,N,K", FULL)
def test_w1a16_full(bl, oracle, M, N, K):
    W, x = _case(M, N, K, seed=M * 131 + N * 7 + K)
    packed, alpha, xb = _oracle_inputs(oracle, W, x)
    y_ref = oracle.w1a16(xb, packed, alpha, K)
    dp, da, dx = _to_dev(packed, alpha, x)
    y, ybuf, sent = guarded_empty((M, N), torch.bfloat16, "cuda")
    bl.bin_linear_w1a16(dx, dp, da, out=y)
    torch.cuda.synchronize()
    assert guards_intact(ybuf, y.numel(), sentinel=sent)
    ms, js = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    check_w1a16(bf16_to_f64(y).ravel(), y_ref.ravel(), alpha, xb, ms.ravel(), js.ravel(),
                what=f"{M}x{N}x{K}")
    assert bl.device_error() == (0, 0)


@pytest.mark.parametrize("M,N,K", [(2048, 11008, 4096), (2048, 4096, 11008)])
def test_w1a16_prefill_7b_sampled(bl, oracle, M, N, K):
    W, x = _case(M, N, K, seed=1)
    packed, alpha, xb = _oracle_inputs(oracle, W, x)
    dp, da, dx = _to_dev(packed, alpha, x)
    y = bl.bin_linear_w1a16(dx, dp, da)
    torch.cuda.synchronize()
    ms, js = sample_positions(M, N, 3000, seed=K)
    y_ref = oracle.w1a16_at(xb, packed, alpha, K, ms, js)
    yg = bf16_to_f64(y)[ms, js]
    check_w1a16(yg, y_ref, alpha, xb, ms, js, what=f"{M}x{N}x{K} sampled")


def test_w1a16_learned_alpha_any_sign(bl, oracle):
    # the forward takes any alpha (the page only initialises it from |W|)
    M, N, K = 3, 257, 512
    W, x = _case(M, N, K, seed=9)
    packed, _, xb = _oracle_inputs(oracle, W, x)
    alpha = np.random.default_rng(4).standard_normal(N).astype(np.float32)
    y_ref = oracle.w1a16(xb, packed, alpha, K)
    dp, da, dx = _to_dev(packed, alpha, x)
    for m_tokens in (3, 40):  # GEMV and GEMM paths
        xx = x if m_tokens == 3 else x.repeat(14, 1)[:m_tokens]
        xbb = xb if m_tokens == 3 else np.tile(xb, (14, 1))[:m_tokens]
        yr = y_ref if m_tokens == 3 else oracle.w1a16(xbb, packed, alpha, K)
        y = bl.bin_linear_w1a16(xx.cuda(), dp, da)
        torch.cuda.synchronize()
        ms, js = np.meshgrid(np.arange(m_tokens), np.arange(N), indexing="ij")
        check_w1a16(bf16_to_f64(y).ravel(), yr.ravel(), alpha, xbb, ms.ravel(), js.ravel())


def test_w1a16_all_ones_closed_form(bl):
    # y_j = alpha_j * (#pos - #neg), independent of the oracle
    N, K = 384, 1024
    import synthetic
    W = synthetic.weights(N, K, 11).cuda()
    packed, alpha = bl.bin_pack(W, bl.BL_PACK_FBI)
    pos = (W > 0).sum(dim=1).float()
    # one fp32 product, then bf16 rounding, as the layer's epilogue does
    want = (alpha * (2 * pos - K)).to(torch.bfloat16).double().cpu().numpy()
    for M in (1, 4, 200):
        x = torch.ones((M, K), dtype=torch.bfloat16, device="cuda")
        y = bf16_to_f64(bl.bin_linear_w1a16(x, packed, alpha))
        assert np.array_equal(y, np.broadcast_to(want, (M, N)))


def test_w1a16_end_to_end_pack_then_linear(bl, oracle):
    M, N, K = 64, 640, 2048
    W, x = _case(M, N, K, seed=21)
    packed, alpha, xb = _oracle_inputs(oracle, W, x)
    y_ref = oracle.w1a16(xb, packed, alpha, K)
    gp, ga = bl.bin_pack(W.cuda(), bl.BL_PACK_FBI)
    y = bl.bin_linear_w1a16(x.cuda(), gp, ga)
    torch.cuda.synchronize()
    ms, js = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    check_w1a16(bf16_to_f64(y).ravel(), y_ref.ravel(), alpha, xb, ms.ravel(), js.ravel())


def test_w1a16_negation_and_zero_tokens(bl):
    M, N, K = 33, 256, 256
    import synthetic
    W = synthetic.weights(N, K, 2).cuda()
    x = synthetic.activations(M, K, 2).cuda()
    packed, alpha = bl.bin_pack(W, bl.BL_PACK_FBI)
    y = bl.bin_linear_w1a16(x, packed, alpha)
    yn = bl.bin_linear_w1a16(-x, packed, alpha)
    assert torch.equal(yn, -y)
    y0 = bl.bin_linear_w1a16(x[:0], packed, alpha)
    assert y0.shape == (0, N)
    torch.cuda.synchronize()


def test_w1a16_overlap_flag_chain(bl, oracle):
    """BL_FLAG_OVERLAP_PREVIOUS on a chain of dependent single-token calls
    (each output is the next input): results must equal the oracle's."""
    import synthetic
    N = K = 2048
    layers = 6
    Ws = [synthetic.weights(N, K, 100 + i) for i in range(layers)]
    refs = [oracle.pack_fbi(W.numpy()) for W in Ws]
    x = synthetic.activations(1, K, 7)
    dev = [(torch.from_numpy(p.view(np.int32)).cuda(), torch.from_numpy(a).cuda()) for p, a in refs]
    h = x.cuda()
    outs = []
    for (dp, da) in dev:
        h = bl.bin_linear_w1a16(h, dp, da, flags=bl.BL_FLAG_OVERLAP_PREVIOUS)
        outs.append(h)
    torch.cuda.synchronize()
    from synthetic import bf16_bits
    xin = bf16_bits(x)
    for i, ((p, a), y) in enumerate(zip(refs, outs)):
        y_ref = oracle.w1a16(xin, p, a, K)
        js = np.arange(N)
        check_w1a16(bf16_to_f64(y).ravel(), y_ref.ravel(), a, xin, np.zeros(N, dtype=np.int64), js,
                    what=f"layer {i}")
        xin = bf16_bits(y.cpu())


@pytest.mark.parametrize("M", [16, 48, 300])
def test_w1a16_overlap_flag_chain_gemm(bl, M):
    """BL_FLAG_OVERLAP_PREVIOUS on calls that take the tensor-core path
    (M > 4, where the flag must not change anything): a chain of dependent
    calls that ping-pongs between two buffers, so every layer also overwrites
    the buffer the layer before it read. The results must equal, bit for bit,
    the same chain run without the flag."""
    import synthetic
    N = K = 1024
    layers = 6
    dev = []
    for i in range(layers):
        W = synthetic.weights(N, K, 300 + i, device="cuda")
        dev.append(bl.bin_pack(W, bl.BL_PACK_FBI))
    x = synthetic.activations(M, K, 11, device="cuda")

    def run(flags):
        bufs = [x.clone(), torch.empty_like(x)]
        for i, (p, a) in enumerate(dev):
            bl.bin_linear_w1a16(bufs[i % 2], p, a, out=bufs[(i + 1) % 2], flags=flags)
        torch.cuda.synchronize()
        return bufs[layers % 2].clone()

    ref = run(0)
    for _ in range(3):
        got = run(bl.BL_FLAG_OVERLAP_PREVIOUS)
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    assert bl.device_error() == (0, 0)
