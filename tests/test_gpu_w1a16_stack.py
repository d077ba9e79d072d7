"""bin_linear_w1a16_stack (single-token decode through a stack of FBI-linear
layers in one persistent launch) on the GPU.

* every output of every level against the oracle's W1A16 forward of the
  input that level actually read (the tolerance of tests/parity.py), for
  slices of one, two and three table pages, ragged N, several linears per
  level, and inputs produced by earlier levels;
* bit-identical to bin_linear_w1a16 called layer by layer where that call
  also splits K eight ways (K = 4096 and 11008, the 7B shapes);
* decode batches of 2..16 tokens (bin_linear_w1a16_stack_batch): every token
  of every level against the oracle, at small and 7B shapes;
* stacks longer than one launch (more than 96 levels or 144 linears), at
  one token and in batches, including the full 7B-shaped chain the benchmark
  times (sampled outputs across the launch boundary);
* the argument checks."""
import ctypes

import numpy as np
import pytest
import torch

from parity import bf16_to_f64, check_w1a16, sample_positions

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bl():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_linear_layers_b200 as m
    return m


def _linear(oracle, N, K, seed):
    import synthetic
    W = synthetic.weights(N, K, seed)
    packed, alpha = oracle.pack_fbi(W.numpy())
    return (torch.from_numpy(packed.view(np.int32)).cuda(), torch.from_numpy(alpha).cuda(), packed, alpha)


def _check_level(oracle, x_dev, linears, what):
    """linears: (packed_np, alpha_np, y_dev) of one level; x_dev the level input ([K] or [M, K])."""
    import synthetic
    K = x_dev.shape[-1]
    xb = synthetic.bf16_bits(x_dev.reshape(-1, K))
    M = xb.shape[0]
    for i, (packed, alpha, y) in enumerate(linears):
        y_ref = oracle.w1a16(xb, packed, alpha, K)
        N = packed.shape[0]
        ms, js = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
        check_w1a16(bf16_to_f64(y.reshape(M, N))[ms, js].ravel(), y_ref[ms, js].ravel(), alpha, xb,
                    ms.ravel(), js.ravel(), what=f"{what} linear {i}")


def _run_and_check(bl, oracle, spec, seed0, M=1):
    """spec: list of levels, each (K, [N...], src) where src is None (a fresh
    input) or (level, linear) whose output feeds this level; M tokens."""
    import synthetic
    levels, host, outs = [], [], []
    for li, (K, Ns, src) in enumerate(spec):
        if src is None:
            x = synthetic.activations(M, K, seed0 + 1000 * li).cuda()
            x = x.reshape(K) if M == 1 else x
        else:
            x = outs[src[0]][src[1]]
            assert x.numel() == M * K
        lins, hl, ys = [], [], []
        for j, N in enumerate(Ns):
            dp, da, packed, alpha = _linear(oracle, N, K, seed0 + 1000 * li + 7 * j + 1)
            y = torch.full((N,) if M == 1 else (M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            lins.append((dp, da, y))
            hl.append((packed, alpha, y))
            ys.append(y)
        levels.append((x, lins))
        host.append((x, hl))
        outs.append(ys)
    st = bl.W1A16Stack(levels)
    st.run()
    torch.cuda.synchronize()
    assert bl.device_error() == (0, 0)
    for li, (x, hl) in enumerate(host):
        _check_level(oracle, x, hl, f"level {li} (K={spec[li][0]})")
    return levels, outs


def test_stack_one_level_each_page_count(bl, oracle):
    # slices of 1..48 words: K = 256 (1 word), 3072 (12), 4096 (16), 8192 (32), 11008 (43), 12288 (48)
    spec = [(256, [100], None), (3072, [256], None), (4096, [300, 1], None), (8192, [513], None),
            (11008, [1000], None), (12288, [257], None)]
    _run_and_check(bl, oracle, spec, seed0=3)


def test_stack_chained_levels(bl, oracle):
    # a miniature transformer block stack: x -> (q, k, v); v -> o; o -> (gate, up); up -> down; repeat
    spec = []
    for layer in range(3):
        base = len(spec)
        src = None if layer == 0 else (base - 1, 0)
        spec.append((1024, [1024, 1024, 1024], src))   # q, k, v
        spec.append((1024, [1024], (base, 2)))         # o from v
        spec.append((1024, [2816, 2816], (base + 1, 0)))  # gate, up from o
        spec.append((2816, [1024], (base + 2, 1)))     # down from up
    _run_and_check(bl, oracle, spec, seed0=11)


def test_stack_matches_layer_by_layer_at_7b_shapes(bl, oracle):
    """K = 4096 and 11008 split 8 ways in both calls: identical bits."""
    import synthetic
    shapes = [(4096, 4096), (4096, 4096), (4096, 11008), (11008, 4096)]  # (K, N)
    x0 = synthetic.activations(1, 4096, 5).reshape(4096).cuda()
    mats = [_linear(oracle, N, K, 20 + i)[:2] for i, (K, N) in enumerate(shapes)]
    ys = [torch.empty(N, dtype=torch.bfloat16, device="cuda") for _, N in shapes]
    levels = [(x0, [(mats[0][0], mats[0][1], ys[0])]), (ys[0], [(mats[1][0], mats[1][1], ys[1])]),
              (ys[1], [(mats[2][0], mats[2][1], ys[2])]), (ys[2], [(mats[3][0], mats[3][1], ys[3])])]
    bl.W1A16Stack(levels).run()
    ref = []
    cur = x0.reshape(1, -1)
    for (dp, da), (K, N) in zip(mats, shapes):
        cur = bl.bin_linear_w1a16(cur, dp, da)
        ref.append(cur.reshape(N))
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(zip(ys, ref)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"level {i} differs"


@pytest.mark.parametrize("M", [2, 5, 8, 9, 16])
def test_stack_batch_chained_levels(bl, oracle, M):
    # the miniature block stack of test_stack_chained_levels, M tokens at once
    spec = []
    for layer in range(2):
        base = len(spec)
        src = None if layer == 0 else (base - 1, 0)
        spec.append((1024, [1024, 1024, 1024], src))
        spec.append((1024, [1024], (base, 2)))
        spec.append((1024, [2816, 2816], (base + 1, 0)))
        spec.append((2816, [1024], (base + 2, 1)))
    _run_and_check(bl, oracle, spec, seed0=31 + M, M=M)


def test_stack_batch_each_page_count(bl, oracle):
    # slices of 1..48 words, ragged N, 16 tokens
    spec = [(256, [100], None), (4096, [300, 1], None), (11008, [700], None), (12288, [257], None)]
    _run_and_check(bl, oracle, spec, seed0=41, M=16)


@pytest.mark.parametrize("M", [8, 16])
def test_stack_batch_at_7b_shapes(bl, oracle, M):
    """A 7B block's four levels (K = 4096 and 11008, the slices of 16 and 43
    words) at 8 and 16 tokens, every output against the oracle."""
    spec = [(4096, [4096, 512], None), (4096, [4096], (0, 0)), (4096, [11008], (1, 0)), (11008, [4096], (2, 0))]
    _run_and_check(bl, oracle, spec, seed0=60 + M, M=M)


@pytest.mark.parametrize("M", [1, 16])
def test_stack_7b_full_chain_sampled(bl, oracle, M):
    """The stacked decode exactly as the benchmark times it: all 224 linears of
    a 7B-shaped model (32 layers; the same seeded weights) in one call, which
    runs as two launches (82 and 46 levels), every level's input the previous
    level's output. Sampled outputs (every 256-row slab edge, both ends, random
    rows) of levels at the start, on both sides of the launch boundary and at
    the end, against the oracle on the input each level read."""
    import synthetic
    dev = torch.device("cuda")
    layers = []
    for layer in range(synthetic.LLAMA7B_LAYERS):
        mats = []
        for idx, (K, N) in enumerate(synthetic.LLAMA7B_LAYER):
            W = synthetic.weights(N, K, seed=5000 + 16 * layer + idx, device=dev)
            mats.append(bl.bin_pack(W, bl.BL_PACK_FBI))
            del W
        layers.append(mats)
    cur = synthetic.activations(M, 4096, seed=77, device=dev)
    levels = []
    for mats in layers:
        q, k, v, o, h = (torch.empty((M, 4096), dtype=torch.bfloat16, device=dev) for _ in range(5))
        g, u = (torch.empty((M, 11008), dtype=torch.bfloat16, device=dev) for _ in range(2))
        levels.append((cur, [(mats[0][0], mats[0][1], q), (mats[1][0], mats[1][1], k), (mats[2][0], mats[2][1], v)]))
        levels.append((v, [(mats[3][0], mats[3][1], o)]))
        levels.append((o, [(mats[4][0], mats[4][1], g), (mats[5][0], mats[5][1], u)]))
        levels.append((u, [(mats[6][0], mats[6][1], h)]))
        cur = h
    bl.W1A16Stack(levels).run()
    torch.cuda.synchronize()
    assert bl.device_error() == (0, 0)
    for li in (0, 1, 2, 3, 80, 81, 82, 83, 126, 127):
        xin, lins = levels[li]
        K = xin.shape[-1]
        xb = synthetic.bf16_bits(xin.reshape(M, K))
        for i, (p, a, y) in enumerate(lins):
            N = p.shape[0]
            ms, js = sample_positions(M, N, 48, seed=1000 * M + 10 * li + i, tile_m=16, tile_n=256)
            pk, al = p.cpu().numpy().view(np.uint32), a.cpu().numpy()
            y_ref = oracle.w1a16_at(xb, pk, al, K, ms, js)
            y_gpu = bf16_to_f64(y.reshape(M, N))[ms, js]
            check_w1a16(y_gpu, y_ref, al, xb, ms, js, what=f"level {li} linear {i} (K={K}, N={N})")


def test_stack_longer_than_one_launch(bl, oracle):
    # 140 levels (two launches), alternating between two buffers
    import synthetic
    K = N = 512
    dp, da, packed, alpha = _linear(oracle, N, K, 77)
    x0 = synthetic.activations(1, K, 78).reshape(K).cuda()
    bufs = [torch.empty(K, dtype=torch.bfloat16, device="cuda") for _ in range(140)]
    levels = [(x0 if i == 0 else bufs[i - 1], [(dp, da, bufs[i])]) for i in range(140)]
    bl.W1A16Stack(levels).run()
    torch.cuda.synchronize()
    assert bl.device_error() == (0, 0)
    for i in (0, 1, 127, 128, 129, 139):
        x = x0 if i == 0 else bufs[i - 1]
        _check_level(oracle, x, [(packed, alpha, bufs[i])], f"level {i}")


def test_stack_many_linears_per_launch(bl, oracle):
    # 300 linears over 3 levels (more than 144 linears: split between launches)
    import synthetic
    K = 256
    dp, da, packed, alpha = _linear(oracle, 64, K, 90)
    xs = [synthetic.activations(1, K, 91 + i).reshape(K).cuda() for i in range(3)]
    ys = [[torch.empty(64, dtype=torch.bfloat16, device="cuda") for _ in range(100)] for _ in range(3)]
    levels = [(xs[i], [(dp, da, y) for y in ys[i]]) for i in range(3)]
    bl.W1A16Stack(levels).run()
    torch.cuda.synchronize()
    assert bl.device_error() == (0, 0)
    for i in range(3):
        _check_level(oracle, xs[i], [(packed, alpha, y) for y in ys[i][::33]], f"level {i}")


@pytest.mark.parametrize("M", [3, 16])
def test_stack_batch_many_small_linears(bl, oracle, M):
    """300 linears of 64 rows over 3 levels: every slab is one linear's 4
    chunks, paired into passes; more linears than one launch takes."""
    import synthetic
    K = 256
    dp, da, packed, alpha = _linear(oracle, 64, K, 92)
    xs = [synthetic.activations(M, K, 93 + i).cuda() for i in range(3)]
    ys = [[torch.empty((M, 64), dtype=torch.bfloat16, device="cuda") for _ in range(100)] for _ in range(3)]
    levels = [(xs[i], [(dp, da, y) for y in ys[i]]) for i in range(3)]
    bl.W1A16Stack(levels).run()
    torch.cuda.synchronize()
    assert bl.device_error() == (0, 0)
    for i in range(3):
        _check_level(oracle, xs[i], [(packed, alpha, y) for y in ys[i][::11]], f"level {i}")


def test_stack_batch_longer_than_one_launch(bl, oracle):
    """110 chained levels at 5 tokens (two launches), alternating K = 512 and 768."""
    import synthetic
    M = 5
    mats = {(K, N): _linear(oracle, N, K, 70 + K // 256) for K, N in [(512, 768), (768, 512)]}
    x0 = synthetic.activations(M, 512, 79).cuda()
    levels, cur, outs = [], x0, []
    for i in range(110):
        K, N = (512, 768) if i % 2 == 0 else (768, 512)
        dp, da, _, _ = mats[(K, N)]
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        levels.append((cur, [(dp, da, y)]))
        outs.append((cur, (K, N), y))
        cur = y
    bl.W1A16Stack(levels).run()
    torch.cuda.synchronize()
    assert bl.device_error() == (0, 0)
    for i in (0, 1, 94, 95, 96, 97, 109):
        x, KN, y = outs[i]
        _, _, packed, alpha = mats[KN]
        _check_level(oracle, x, [(packed, alpha, y)], f"level {i}")


def test_stack_argument_checks(bl):
    K, N = 4096, 256
    x = torch.zeros(K, dtype=torch.bfloat16, device="cuda")
    p = torch.zeros((N, K // 32), dtype=torch.int32, device="cuda")
    a = torch.zeros(N, dtype=torch.float32, device="cuda")
    y = torch.zeros(N, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(bl.workspace_bytes(bl.BL_OP_W1A16_STACK, 0, N, 0), dtype=torch.uint8, device="cuda")
    job = bl.StackJob(p.data_ptr(), a.data_ptr(), y.data_ptr(), N)

    def call(K_, first=0, num=1, ws_bytes=ws.numel(), xp=x.data_ptr()):
        lv = bl.StackLevel(xp, K_, first, num)
        return bl.lib.bin_linear_w1a16_stack(ctypes.byref(lv), 1, ctypes.byref(job), 1, ws.data_ptr(), ws_bytes,
                                             torch.cuda.current_stream().cuda_stream)

    assert call(4096) == 0
    assert call(4000) == bl.BL_ERR_UNSUPPORTED     # not a multiple of 256
    assert call(12544) == bl.BL_ERR_UNSUPPORTED    # more than 48 words per slice
    assert call(4096, first=1) == bl.BL_ERR_INVALID_ARG
    assert call(4096, num=0) == bl.BL_ERR_INVALID_ARG
    assert call(4096, ws_bytes=4) == bl.BL_ERR_INVALID_ARG
    assert call(4096, xp=x.data_ptr() + 2) == bl.BL_ERR_INVALID_ARG  # x not 16-byte aligned
    torch.cuda.synchronize()
    assert bl.device_error() == (0, 0)
