"""Pins for the CPU oracle: facts fixed by the pages and by mathematics,
independent of the oracle's own code.

Each pin returns normally when it holds and raises ``AssertionError`` when it
does not. ``run_pins(oracle)`` runs them all and returns the failures, so the
same pins can be run against the real oracle (no failure allowed) and against
copies of it with a planted mistake (at least one failure required).

What pins what:
* the hand-worked examples in ``tests/golden`` (exact rational values
  derived from the FBI-linear paragraph and BitNet Eq.(1)-(8));
* closed forms: all-ones input gives alpha_j*(#pos - #neg); an all-positive
  row gives alpha * (exact sum of x); alternating +-1 input quantises to
  +-127;
* the W1A1 identity dot = K - 2*popcount(a XOR b), brute-forced over every
  pair of sign vectors for small K, and the W1A16 forward fed +-1 inputs;
* independent library routines: ``numpy.packbits`` for the packed layout,
  ``math.fsum`` (exact sums) for the scales;
* invariants: negation, scaling by powers of two, integer shifts, constant
  tokens, exact .5 ties (round half to even);
* for the b1.58 ternary weights: a hand-worked example with exact ties and
  clips, equal-magnitude weights reducing to the binary signs (through the
  separate FBI packing), popcount closed forms, inert sub-threshold weights;
* for the straight-through backward: adjoint identities against the
  forward, exact unit-step differences of the forward, all-ones closed
  forms, and dw's independence of the signs (with numpy's matmul).
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _frac(s) -> Fraction:
    return Fraction(s)


def _bf16_bits_of(values) -> np.ndarray:
    """bf16 patterns of values that are exactly representable in bf16."""
    f = np.asarray([float(v) for v in values], dtype=np.float32)
    u = f.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exact in bf16"
    return (u >> 16).astype(np.uint16)


def _bf16_values(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _to_bf16_bits(f32: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest even) -- input generation only."""
    u = np.ascontiguousarray(f32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def _popcounts(words: np.ndarray) -> np.ndarray:
    """Set bits per row of a uint32 array (rows = leading axis)."""
    return np.array([sum(int(w).bit_count() for w in row) for row in words], dtype=np.int64)


def _packbits_rows(bits: np.ndarray, K: int) -> np.ndarray:
    """Independent statement of the packed layout through numpy.packbits:
    little bit order inside each byte, little-endian bytes inside each word."""
    N = bits.shape[0]
    words = (K + 31) // 32
    padded = np.zeros((N, words * 32), dtype=np.uint8)
    padded[:, :K] = bits
    by = np.packbits(padded, axis=1, bitorder="little")
    return by.view("<u4").reshape(N, words).astype(np.uint32)


# ---------------------------------------------------------------- examples


def pin_example_a_pack(o):
    ex = _load("fbi_example_a.json")
    W = np.array([[float(_frac(v)) for v in row] for row in ex["W"]], dtype=np.float32)
    packed, alpha = o.pack_fbi(W)
    assert packed[:, 0].tolist() == ex["packed"], packed[:, 0].tolist()
    assert [Fraction(float(a)) for a in alpha] == [_frac(a) for a in ex["alpha"]], alpha
    u = ex["unbalanced_row"]
    Wu = np.array([[float(_frac(v)) for v in u["W"]]], dtype=np.float32)
    pu, au = o.pack_fbi(Wu)
    assert int(pu[0, 0]) == u["packed"] and Fraction(float(au[0])) == _frac(u["alpha"])
    y = o.w1a16(_bf16_bits_of([1, 1, 1, 1])[None, :], pu, au, 4)
    assert Fraction(float(y[0, 0])) == _frac(u["y_all_ones"]), y


def pin_example_a_forward(o):
    ex = _load("fbi_example_a.json")
    packed = np.array(ex["packed"], dtype=np.uint32)[:, None]
    alpha = np.array([float(_frac(a)) for a in ex["alpha"]], dtype=np.float32)
    for case in ex["cases"]:
        x = _bf16_bits_of([_frac(v) for v in case["x"]])[None, :]
        y = o.w1a16(x, packed, alpha, ex["K"])
        assert [Fraction(float(v)) for v in y[0]] == [_frac(v) for v in case["y"]], y


def pin_example_b_pack(o):
    ex = _load("bitnet_example_b.json")
    W = np.array([[float(_frac(v)) for v in row] for row in ex["W"]], dtype=np.float32)
    packed, alpha, beta = o.pack_bitnet(W)
    assert packed[:, 0].tolist() == ex["packed"], packed[:, 0].tolist()
    assert Fraction(alpha) == _frac(ex["alpha"]), alpha
    assert Fraction(beta) == _frac(ex["beta"]), beta


def pin_example_b_forward(o):
    ex = _load("bitnet_example_b.json")
    packed = np.array(ex["packed"], dtype=np.uint32)[:, None]
    beta = float(_frac(ex["beta"]))
    for tok in ex["tokens"]:
        x = _bf16_bits_of([_frac(v) for v in tok["x"]])[None, :]
        xq, gamma, pre = o.ln_absmax_quant(x, ex["eps"], want_pre=True)
        assert xq[0].tolist() == tok["xq"], xq
        # pre-round values: exact up to fp64 rounding of the LN steps
        for got, want in zip(pre[0], tok["pre"]):
            assert abs(got - float(_frac(want))) <= 1e-12 * 128, (pre, tok["pre"])
        assert abs(gamma[0] - float(tok["gamma"])) <= 4e-16 * float(tok["gamma"]), gamma
        acc = o.w1a8_acc(xq, packed, ex["K"])
        assert acc[0].tolist() == tok["acc"], acc
        y = o.w1a8_rescale(acc, gamma, beta)
        for got, want in zip(y[0], tok["y"]):
            assert abs(got - float(want)) <= 1e-15 * abs(float(want)), (y, tok["y"])


def pin_round_half_even_ties(o):
    ex = _load("rne_tie.json")
    c = ex["magnitudes"]
    x = _bf16_bits_of(list(c) + [-v for v in c])[None, :]
    xq, gamma = o.ln_absmax_quant(x, ex["eps"])
    want = list(ex["xq_magnitudes"]) + [-v for v in ex["xq_magnitudes"]]
    assert xq[0].tolist() == want, xq[0].tolist()
    assert Fraction(float(gamma[0])) == _frac(ex["gamma"]), gamma


# ------------------------------------------------------------ closed forms


def _random_case(seed, N, K, M=3, mean=0.0):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02 + mean).astype(np.float32)
    x = _to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    return W, x


def pin_packed_layout_numpy(o):
    for K in (32, 96, 100, 7):
        W, _ = _random_case(11 + K, 9, K)
        W[0, : min(K, 5)] = 0.0  # zeros must pack as -1 (bit clear)
        packed, _ = o.pack_fbi(W)
        assert np.array_equal(packed, _packbits_rows((W > 0).astype(np.uint8), K)), K


def pin_fbi_alpha_exact_sum(o):
    W, _ = _random_case(5, 17, 300)
    _, alpha = o.pack_fbi(W)
    for j in range(W.shape[0]):
        want = np.float32(math.fsum(abs(float(v)) for v in W[j]) / W.shape[1])
        assert abs(int(alpha[j].view(np.int32)) - int(want.view(np.int32))) <= 1, (j, alpha[j], want)


def pin_bitnet_global_scalars(o):
    W, _ = _random_case(6, 23, 128, mean=0.001)
    packed, alpha, beta = o.pack_bitnet(W)
    n = W.size
    a_exact = math.fsum(float(v) for v in W.ravel()) / n
    b_exact = math.fsum(abs(float(v)) for v in W.ravel()) / n
    assert abs(alpha - a_exact) <= 1e-12 * abs(a_exact), (alpha, a_exact)
    assert abs(beta - b_exact) <= 1e-14 * b_exact, (beta, b_exact)
    # signs of W - alpha, with the boundary decided on the exact mean
    bits = (W.astype(np.float64) > a_exact).astype(np.uint8)
    assert np.array_equal(packed, _packbits_rows(bits, W.shape[1]))


def pin_bitnet_sign_at_mean(o):
    # every weight equal to the global mean maps to -1 ([BitNet] Eq.(2): <= 0 -> -1)
    W = np.array([[1.0, 2.0, 3.0, 2.0], [2.0, 0.0, 4.0, 2.0]], dtype=np.float32)  # mean 2
    packed, alpha, _ = o.pack_bitnet(W)
    assert alpha == 2.0
    assert packed[:, 0].tolist() == [0b0100, 0b0100], packed[:, 0].tolist()


def pin_all_ones_closed_form(o):
    for K in (64, 130):
        W, _ = _random_case(21 + K, 13, K)
        packed, alpha = o.pack_fbi(W)
        y = o.w1a16(_bf16_bits_of([1] * K)[None, :], packed, alpha, K)
        pos = _popcounts(packed)
        want = alpha.astype(np.float64) * (2 * pos - K)
        assert np.array_equal(y[0], want), (y[0], want)


def pin_all_positive_row_is_plain_sum(o):
    K = 32
    rng = np.random.default_rng(3)
    x = _to_bf16_bits(rng.standard_normal((2, K)).astype(np.float32))
    W = np.abs(rng.standard_normal((1, K))).astype(np.float32) + 0.5
    packed, alpha = o.pack_fbi(W)
    assert int(packed[0, 0]) == 0xFFFFFFFF
    y = o.w1a16(x, packed, alpha, K)
    for m in range(2):
        s = math.fsum(_bf16_values(x[m]).tolist())
        assert y[m, 0] == float(alpha[0]) * s, (y[m, 0], s)


def pin_negation(o):
    W, x = _random_case(31, 19, 160, M=4)
    packed, alpha = o.pack_fbi(W)
    y = o.w1a16(x, packed, alpha, 160)
    yn = o.w1a16(x ^ np.uint16(0x8000), packed, alpha, 160)
    assert np.array_equal(yn, -y)


def pin_w1a1_identity_bruteforce(o):
    for K in (1, 2, 3, 5, 6, 10):
        vals = np.arange(1 << K, dtype=np.uint32)[:, None]
        dot = o.w1a1(vals, vals, K)
        xor = vals[:, 0][:, None] ^ vals[:, 0][None, :]
        pc = np.vectorize(lambda v: int(v).bit_count())(xor)
        assert np.array_equal(dot, K - 2 * pc), K


def pin_w1a1_multiword(o):
    K = 77
    rng = np.random.default_rng(8)
    wpr = (K + 31) // 32
    a = rng.integers(0, 2**32, size=(5, wpr), dtype=np.uint64).astype(np.uint32)
    b = rng.integers(0, 2**32, size=(6, wpr), dtype=np.uint64).astype(np.uint32)
    a[:, -1] &= (1 << (K % 32)) - 1
    b[:, -1] &= (1 << (K % 32)) - 1
    dot = o.w1a1(a, b, K)
    for i in range(5):
        for j in range(6):
            pc = sum(int(u ^ v).bit_count() for u, v in zip(a[i], b[j]))
            assert dot[i, j] == K - 2 * pc


def pin_w1a16_on_pm1_inputs_is_w1a1(o):
    # feeding the W1A16 forward +-1 activations (alpha = 1) must give the W1A1 dot
    K = 10
    vals = np.arange(1 << K, dtype=np.uint32)[:, None]
    bits = ((vals >> np.arange(K, dtype=np.uint32)) & 1).astype(np.int64)
    x = _bf16_bits_of((2 * bits - 1).ravel()).reshape(1 << K, K)
    sel = vals[::37]
    y = o.w1a16(x, sel, np.ones(sel.shape[0], dtype=np.float32), K)
    dot = o.w1a1(vals, sel, K)
    assert np.array_equal(y, dot.astype(np.float64))


def pin_quant_invariants(o):
    rng = np.random.default_rng(12)
    M, K = 6, 96
    xi = rng.integers(-100, 101, size=(M, K)).astype(np.float32)
    x = _bf16_bits_of(xi.ravel()).reshape(M, K)
    xq, gamma = o.ln_absmax_quant(x)
    # every token's largest |x - mu| sits on the clamp; all codes in range
    assert np.all(np.abs(xq).max(axis=1) == 127)
    assert np.all(np.abs(xq.astype(np.int32)) <= 127)
    # scaling by a power of two leaves the codes unchanged (LN cancels it)
    xs = _bf16_bits_of((xi * 4).ravel()).reshape(M, K)
    assert np.array_equal(o.ln_absmax_quant(xs)[0], xq)
    # shifting every token by an integer leaves the codes unchanged
    xh = _bf16_bits_of((xi + 64).ravel()).reshape(M, K)
    assert np.array_equal(o.ln_absmax_quant(xh)[0], xq)
    # negation negates the codes
    assert np.array_equal(o.ln_absmax_quant(x ^ np.uint16(0x8000))[0], -xq)


def pin_alternating_and_constant_tokens(o):
    K = 64
    alt = np.array([1.0 if k % 2 == 0 else -1.0 for k in range(K)], dtype=np.float32)
    const = np.full(K, 3.0, dtype=np.float32)
    x = np.stack([_bf16_bits_of(alt), _bf16_bits_of(const)])
    xq, gamma = o.ln_absmax_quant(x)
    assert xq[0].tolist() == [127 if k % 2 == 0 else -127 for k in range(K)]
    assert xq[1].tolist() == [0] * K and gamma[1] == 0.0
    W, _ = _random_case(41, 11, K)
    packed, _ = o.pack_fbi(W)
    acc = o.w1a8_acc(xq, packed, K)
    signs = 2 * ((packed[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(11, -1)[:, :K].astype(np.int64) - 1
    alt_sign = np.array([1 if k % 2 == 0 else -1 for k in range(K)], dtype=np.int64)
    assert np.array_equal(acc[0], 127 * (signs @ alt_sign))
    assert np.array_equal(acc[1], np.zeros(11, dtype=np.int64))
    y = o.w1a8_rescale(acc, gamma, 0.25)
    assert np.all(y[1] == 0.0)


def pin_acc_with_unit_codes(o):
    K = 160
    W, _ = _random_case(51, 14, K)
    packed, _ = o.pack_fbi(W)
    acc = o.w1a8_acc(np.ones((1, K), dtype=np.int8), packed, K)
    assert np.array_equal(acc[0], 2 * _popcounts(packed) - K)


def pin_sampled_equals_full(o):
    W, x = _random_case(61, 9, 64, M=5)
    packed, alpha = o.pack_fbi(W)
    y = o.w1a16(x, packed, alpha, 64)
    ms = np.array([0, 4, 2, 3], dtype=np.int64)
    js = np.array([8, 0, 5, 5], dtype=np.int64)
    assert np.array_equal(o.w1a16_at(x, packed, alpha, 64, ms, js), y[ms, js])
    xq, _ = o.ln_absmax_quant(x)
    acc = o.w1a8_acc(xq, packed, 64)
    assert np.array_equal(o.w1a8_acc_at(xq, packed, 64, ms, js), acc[ms, js])
    # the ternary sampler against its full product (M != N, and no sample
    # lies on the diagonal, so swapped token and output indices show)
    Wt, xt = _random_case(62, 9, 128, M=5)
    packed_t, _ = o.pack_ternary(Wt)
    xq_t, _ = o.ln_absmax_quant(xt)
    acc_t = o.w158a8_acc(xq_t, packed_t, 128)
    assert np.array_equal(o.w158a8_acc_at(xq_t, packed_t, 128, ms, js), acc_t[ms, js])


# ---- b1.58 ternary weights (BitNet b1.58 page, section 2, Eq.(9)-(11)) ----

def pin_ternary_example_c_pack(o):
    ex = _load("ternary_example_c.json")
    W = np.array([[float(_frac(v)) for v in row] for row in ex["W"]], dtype=np.float32)
    packed, gamma = o.pack_ternary(W, eps=ex["weight_eps"])
    assert Fraction(gamma) == _frac(ex["gamma"]), gamma
    assert packed[:, 0].tolist() == ex["plus_words"], packed
    assert packed[:, 4].tolist() == ex["minus_words"], packed
    assert not packed[:, [1, 2, 3, 5, 6, 7]].any(), packed


def pin_ternary_example_c_forward(o):
    ex = _load("ternary_example_c.json")
    W = np.array([[float(_frac(v)) for v in row] for row in ex["W"]], dtype=np.float32)
    packed, gamma_w = o.pack_ternary(W, eps=ex["weight_eps"])
    for tok in ex["tokens"]:
        x = _bf16_bits_of([_frac(v) for v in tok["x"]])[None, :]
        xq, gamma = o.ln_absmax_quant(x, ex["ln_eps"])
        assert xq[0].tolist() == tok["xq"], xq
        acc = o.w158a8_acc(xq, packed, ex["K"])
        assert acc[0].tolist() == tok["acc"], acc
        y = o.w1a8_rescale(acc, gamma, gamma_w)
        for got, want in zip(y[0], tok["y"]):
            assert abs(got - float(want)) <= 1e-15 * abs(float(want)), (y, tok["y"])


def pin_ternary_equal_magnitudes_are_signs(o):
    # |W_jk| = c everywhere: gamma = c, W/gamma = +-1, so the ternary weights
    # are Sign(W) and the b1.58 product equals the binary one (FBI packing)
    rng = np.random.default_rng(11)
    N, K = 5, 300
    W = np.where(rng.random((N, K)) < 0.5, -0.375, 0.375).astype(np.float32)
    packed_t, gamma = o.pack_ternary(W, eps=0.0)
    assert gamma == 0.375
    packed_s, _ = o.pack_fbi(W)
    xq = rng.integers(-127, 128, size=(3, K), dtype=np.int64).astype(np.int8)
    assert np.array_equal(o.w158a8_acc(xq, packed_t, K), o.w1a8_acc(xq, packed_s, K))


def pin_ternary_all_ones_codes(o):
    # codes all 1: acc_j = (number of +1 weights) - (number of -1 weights)
    rng = np.random.default_rng(12)
    N, K = 7, 260
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    packed, _ = o.pack_ternary(W)
    xq = np.ones((1, K), dtype=np.int8)
    acc = o.w158a8_acc(xq, packed, K)[0]
    w = packed.reshape(N, -1, 8)
    plus = _popcounts(w[:, :, :4].reshape(N, -1))
    minus = _popcounts(w[:, :, 4:].reshape(N, -1))
    assert not (w[:, :, :4] & w[:, :, 4:]).any(), "a weight is both +1 and -1"
    assert np.array_equal(acc, plus - minus), (acc, plus - minus)


def pin_ternary_small_weights_are_inert(o):
    # weights below half of gamma quantise to 0: changing the codes at those
    # positions leaves every accumulator unchanged
    N, K = 3, 128
    W = np.zeros((N, K), dtype=np.float32)
    W[:, ::2] = 1.0     # large: ratio 1/gamma > 1/2
    W[:, 1::2] = 0.125  # small: ratio 0.125/gamma < 1/2
    packed, gamma = o.pack_ternary(W, eps=0.0)
    assert gamma == (1.0 + 0.125) / 2
    rng = np.random.default_rng(13)
    xq = rng.integers(-127, 128, size=(2, K), dtype=np.int64).astype(np.int8)
    xq2 = xq.copy()
    xq2[:, 1::2] = -xq2[:, 1::2] // 2
    assert np.array_equal(o.w158a8_acc(xq, packed, K), o.w158a8_acc(xq2, packed, K))
    assert np.array_equal(o.w158a8_acc(xq, packed, K)[:, 0], xq[:, ::2].astype(np.int64).sum(axis=1))


def pin_ternary_eps_moves_the_threshold(o):
    # gamma = 1. eps = 0: every ratio (3/4, 5/4, 1, 1) rounds to 1. eps = 1:
    # 3/8 rounds to 0, 5/8 to 1, and 1/2 ties to the even 0
    W = np.array([[0.75, 1.25, 1.0, 1.0]], dtype=np.float32)
    p0, g0 = o.pack_ternary(W, eps=0.0)
    p1, g1 = o.pack_ternary(W, eps=1.0)
    assert g0 == g1 == 1.0
    assert p0[0, 0] == 0b1111 and p1[0, 0] == 0b0010, (p0, p1)
    assert p0[0, 4] == 0 and p1[0, 4] == 0


# ---- per-tensor Eq.(5) and the non-negative Eq.(6) quantisers ---------------

def pin_quant_tensor_example_d(o):
    ex = _load("quant_tensor_example_d.json")
    x = np.stack([_bf16_bits_of([_frac(v) for v in row]) for row in ex["x"]])
    for mode, key in ((0, "per_tensor"), (1, "nonneg")):
        want = ex[key]
        xq, gamma, eta, pre = o.ln_quant_tensor(x, mode, eps=ex["ln_eps"], want_pre=True)
        assert xq.tolist() == want["xq"], (key, xq)
        g = float(want["gamma"])
        assert np.all(np.abs(gamma - g) <= 4e-16 * g), (key, gamma)
        if mode == 1:
            assert abs(eta - float(want["eta"])) <= 4e-16 * abs(float(want["eta"])), eta
        for got_row, want_row in zip(pre, want["pre"]):
            for got, w in zip(got_row, want_row):
                assert abs(got - float(w)) <= 1e-12 * 128, (key, pre)


def pin_quant_tensor_one_token_is_per_token(o):
    # Eq.(5) over a one-token matrix is the per-token quantiser (a separate function)
    rng = np.random.default_rng(21)
    x = _to_bf16_bits((rng.standard_normal((1, 700)) * 3).astype(np.float32))
    xq_t, g_t, _ = o.ln_quant_tensor(x, 0)
    xq_p, g_p = o.ln_absmax_quant(x)
    assert np.array_equal(xq_t, xq_p) and np.array_equal(g_t, g_p)


def pin_quant_tensor_widest_token_keeps_its_codes(o):
    # the token with the largest max|LN| sets the tensor's gamma, so its codes
    # equal its per-token codes; every other token's |codes| can only shrink
    rng = np.random.default_rng(22)
    x = _to_bf16_bits((rng.standard_normal((6, 384)) * np.arange(1, 7)[:, None]).astype(np.float32))
    x[2, 5] = _to_bf16_bits(np.array([400.0], np.float32))[0]  # an outlier: token 2 is the widest
    xq_t, g_t, _ = o.ln_quant_tensor(x, 0)
    xq_p, g_p = o.ln_absmax_quant(x)
    w = int(np.argmax(g_p))
    assert w == 2 and np.all(g_t == g_p[w])
    assert np.array_equal(xq_t[w], xq_p[w])
    assert np.all(np.abs(xq_t.astype(int)) <= np.abs(xq_p.astype(int)))


def pin_quant_nonneg_range(o):
    # Eq.(6): codes in [0, 127]; the tensor's smallest LN value maps to 0 and the
    # largest to 127 (128 clamped); gamma = max LN - min LN
    rng = np.random.default_rng(23)
    x = _to_bf16_bits(rng.standard_normal((5, 256)).astype(np.float32))
    xq, gamma, eta, pre = o.ln_quant_tensor(x, 1, want_pre=True)
    assert xq.min() == 0 and xq.max() == 127
    i_min, i_max = np.unravel_index(np.argmin(pre), pre.shape), np.unravel_index(np.argmax(pre), pre.shape)
    assert xq[i_min] == 0 and xq[i_max] == 127 and pre[i_min] == 0.0 and pre[i_max] == 128.0
    assert eta < 0 < gamma[0] and np.all(gamma == gamma[0])


# ---------------------------------------------------------------- backward (STE)
#
# The forward is linear in x and in alpha, so its gradients are fixed by the
# forward alone: <dy, y> = <dx, x> = <dalpha, alpha> (adjoint identities), a
# unit step in x_mk or alpha_j changes <dy, y> by exactly dx_mk or dalpha_j,
# and the straight-through weight gradient satisfies <dw, S> = <dy, y> too
# (dw_jk = alpha_j sum_m dy_mj x_mk, summed against s_jk gives alpha_j z_mj).


def _backward_case(seed, M, N, K, small_ints=False):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    if small_ints:  # values whose unit steps stay exact in bf16
        x = _bf16_bits_of(rng.integers(-8, 9, M * K).tolist()).reshape(M, K)
        dy = _bf16_bits_of(rng.integers(-4, 5, M * N).tolist()).reshape(M, N)
    else:
        x = _to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
        dy = _to_bf16_bits(rng.standard_normal((M, N)).astype(np.float32))
    return W, x, dy


def _inner(a, b) -> float:
    return math.fsum((np.asarray(a, dtype=np.float64) * np.asarray(b, dtype=np.float64)).ravel().tolist())


def pin_backward_adjoint_identities(o):
    M, N, K = 3, 5, 70  # N != K and M != N: a transposed index changes shapes or values
    W, x, dy = _backward_case(41, M, N, K)
    packed, alpha = o.pack_fbi(W)
    y = o.w1a16(x, packed, alpha, K)
    dx, dw, da = o.w1a16_backward(x, packed, alpha, dy, K)
    assert dx.shape == (M, K) and dw.shape == (N, K) and da.shape == (N,)
    ref = _inner(_bf16_values(dy), y)
    S = np.where(W > 0, 1.0, -1.0)
    for name, val in (("<dx,x>", _inner(dx, _bf16_values(x))), ("<dalpha,alpha>", _inner(da, alpha)),
                      ("<dw,S>", _inner(dw, S))):
        assert abs(val - ref) <= 1e-12 * max(1.0, abs(ref)), (name, val, ref)


def pin_backward_unit_steps(o):
    # small integers: every sum below is exact in fp64, so the differences are exact
    M, N, K = 2, 3, 40
    W, x, dy = _backward_case(43, M, N, K, small_ints=True)
    packed, alpha = o.pack_fbi(W)
    alpha = np.array([0.5, 2.0, -1.25], dtype=np.float32)  # any scales (exact binary fractions)
    dyv = _bf16_values(dy)
    base = _inner(dyv, o.w1a16(x, packed, alpha, K))
    dx, dw, da = o.w1a16_backward(x, packed, alpha, dy, K)
    for (m, k) in ((0, 0), (1, 17), (0, 39)):
        xs = x.copy()
        xs[m, k] = _bf16_bits_of([_bf16_values(x[m:m + 1, k:k + 1])[0, 0] + 1.0])[0]
        step = _inner(dyv, o.w1a16(xs, packed, alpha, K)) - base
        assert step == dx[m, k], ((m, k), step, dx[m, k])
    for j in range(N):
        a2 = alpha.copy()
        a2[j] += np.float32(1.0)
        step = _inner(dyv, o.w1a16(x, packed, a2, K)) - base
        assert step == da[j], (j, step, da[j])


def pin_backward_all_ones_closed_form(o):
    M, N, K = 4, 6, 96
    W, _, _ = _backward_case(47, M, N, K)
    packed, alpha = o.pack_fbi(W)
    ones_x = _bf16_bits_of([1] * (M * K)).reshape(M, K)
    ones_dy = _bf16_bits_of([1] * (M * N)).reshape(M, N)
    dx, dw, da = o.w1a16_backward(ones_x, packed, alpha, ones_dy, K)
    S = np.where(W > 0, 1.0, -1.0)
    # dw_jk = alpha_j * M; dx_mk = sum_j alpha_j s_jk; dalpha_j = M (#pos_j - #neg_j)
    assert np.array_equal(dw, np.repeat(alpha.astype(np.float64)[:, None] * M, K, axis=1))
    for k in range(K):
        want = math.fsum((alpha.astype(np.float64) * S[:, k]).tolist())
        assert abs(dx[0, k] - want) <= 1e-15 * N and np.all(dx[:, k] == dx[0, k]), k
    assert np.array_equal(da, M * (2.0 * _popcounts(packed) - K))


def pin_backward_dw_ignores_signs(o):
    # straight-through: dw does not depend on which way the weights' signs went
    M, N, K = 3, 4, 64
    W, x, dy = _backward_case(53, M, N, K)
    packed, alpha = o.pack_fbi(W)
    _, dw1, _ = o.w1a16_backward(x, packed, alpha, dy, K)
    _, dw2, _ = o.w1a16_backward(x, packed ^ np.uint32(0xFFFFFFFF), alpha, dy, K)
    assert np.array_equal(dw1, dw2)
    # and it is alpha_j times a product that numpy computes independently
    P = _bf16_values(dy).T @ _bf16_values(x)
    assert np.allclose(dw1, alpha.astype(np.float64)[:, None] * P, rtol=1e-13, atol=1e-13)


def pin_backward_example_e(o):
    # hand-worked 2 x 3 x 4 example (tests/golden/ste_example_e.json), every value exact
    ex = _load("ste_example_e.json")
    W = np.array([[float(_frac(v)) for v in row] for row in ex["W"]], dtype=np.float32)
    packed, _ = o.pack_fbi(W)
    assert packed[:, 0].tolist() == ex["packed"], packed[:, 0].tolist()
    alpha = np.array([float(_frac(a)) for a in ex["alpha"]], dtype=np.float32)
    x = np.stack([_bf16_bits_of([_frac(v) for v in row]) for row in ex["x"]])
    dy = np.stack([_bf16_bits_of([_frac(v) for v in row]) for row in ex["dy"]])
    dx, dw, da = o.w1a16_backward(x, packed, alpha, dy, 4)
    assert [[Fraction(float(v)) for v in r] for r in dx] == [[_frac(v) for v in r] for r in ex["dx"]], dx
    assert [[Fraction(float(v)) for v in r] for r in dw] == [[_frac(v) for v in r] for r in ex["dW"]], dw
    assert [Fraction(float(v)) for v in da] == [_frac(v) for v in ex["dalpha"]], da
    # and the forward of the same layer gives alpha * z
    y = o.w1a16(x, packed, alpha, 4)
    want = [[_frac(a) * _frac(z) for a, z in zip(ex["alpha"], row)] for row in ex["z"]]
    assert [[Fraction(float(v)) for v in r] for r in y] == want, y


def pin_backward_sampled_equals_full(o):
    M, N, K = 3, 7, 96
    W, x, dy = _backward_case(59, M, N, K)
    packed, alpha = o.pack_fbi(W)
    dx, dw, da = o.w1a16_backward(x, packed, alpha, dy, K)
    ms, ks = np.meshgrid(np.arange(M), np.arange(K), indexing="ij")
    assert np.array_equal(o.w1a16_backward_at(x, packed, alpha, dy, K, "dx", ms.ravel(), ks.ravel()), dx.ravel())
    js, ks = np.meshgrid(np.arange(N), np.arange(K), indexing="ij")
    assert np.array_equal(o.w1a16_backward_at(x, packed, alpha, dy, K, "dw", js.ravel(), ks.ravel()), dw.ravel())
    assert np.array_equal(o.w1a16_backward_at(x, packed, alpha, dy, K, "dalpha", np.arange(N)), da)


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_") and callable(v)]


def run_pins(oracle) -> list[tuple[str, str]]:
    """Run every pin; return [(name, message)] for those that failed."""
    failures = []
    for pin in PINS:
        try:
            pin(oracle)
        except AssertionError as e:  # a pin that does not hold
            failures.append((pin.__name__, str(e)[:200]))
        except Exception as e:  # a broken oracle may also crash a pin
            failures.append((pin.__name__, f"{type(e).__name__}: {str(e)[:200]}"))
    return failures
