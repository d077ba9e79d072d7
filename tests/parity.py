"""Helpers shared by the GPU parity tests: tolerances, samples, conversions.

Tolerances (stated once, used by every parity test):
* packed signs, int8 codes, int32 accumulators: bit-exact;
* FBI alpha and BitNet alpha/beta (fp32 roundings of fp64 sums whose
  summation order differs): within 1 ulp of fp32;
* W1A16: |y - y_ref| <= 1e-4 * alpha_j * sum_k |x_mk|  +  half a bf16 ulp of
  (|y_ref| + that bound), the second term being the mandated bf16 output
  rounding;
* W1A8 y: within 2 ulp of fp32 of the oracle's fp64 value;
* gamma (fp64): relative difference <= (K/2 + 8) * 2^-53. The two sides sum
  the K squared deviations in different orders; a recursive fp64 sum of K
  non-negative terms is within (K-1) * 2^-53 relative of exact, the GPU's
  tree sum well inside that, and gamma = max|x-mu| / sqrt(var + eps) halves
  the variance's relative error (a few more roundings give the + 8);
* int8 codes may differ (by 1) only where the oracle's unrounded value is
  within 1e-9 of a half-integer: both readings are then correct.
"""
from __future__ import annotations

import numpy as np
import torch

W1A16_REL = 1e-4
W1A8_ULPS = 2
TIE_BAND = 1e-9


def u32(t: torch.Tensor) -> np.ndarray:
    """int32 device tensor of packed signs -> uint32 numpy (bit patterns)."""
    return t.detach().cpu().numpy().view(np.uint32)


def gamma_rel_bound(K: int) -> float:
    return (K / 2 + 8) * 2.0 ** -53


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().float().numpy().astype(np.float64)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 7)


def f32_ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in fp32 ulps between two fp32 arrays (same sign assumed or 0)."""
    ia = np.asarray(a, dtype=np.float32).view(np.int32).astype(np.int64)
    ib = np.asarray(b, dtype=np.float32).view(np.int32).astype(np.int64)
    # map sign-magnitude to a monotonic integer line
    ia = np.where(ia < 0, -(ia & 0x7FFFFFFF), ia)
    ib = np.where(ib < 0, -(ib & 0x7FFFFFFF), ib)
    return np.abs(ia - ib)


def w1a16_bound(alpha: np.ndarray, x_bits: np.ndarray, y_ref: np.ndarray, ms, js) -> np.ndarray:
    """Per-element W1A16 tolerance at positions (ms, js)."""
    xa = np.abs((x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)).sum(axis=1)
    tol = W1A16_REL * np.abs(alpha.astype(np.float64)[js]) * xa[ms]
    return tol + 0.5 * bf16_ulp(np.abs(y_ref) + tol)


def check_w1a16(y_gpu: np.ndarray, y_ref: np.ndarray, alpha, x_bits, ms, js, what=""):
    bound = w1a16_bound(alpha, x_bits, y_ref, ms, js)
    err = np.abs(y_gpu - y_ref)
    bad = np.nonzero(err > bound)[0]
    assert bad.size == 0, (
        f"{what}: {bad.size} of {err.size} outside tolerance; first at (m={ms[bad[0]]}, j={js[bad[0]]}) "
        f"gpu={y_gpu[bad[0]]!r} ref={y_ref[bad[0]]!r} bound={bound[bad[0]]!r}")
    return float((err / np.maximum(bound, 1e-300)).max()) if err.size else 0.0


def sample_positions(M: int, N: int, count: int, seed: int, tile_m=128, tile_n=128):
    """Sampled (m, j) positions: random ones plus every corner and tile edge."""
    rng = np.random.default_rng(seed)
    ms = list(rng.integers(0, M, size=count))
    js = list(rng.integers(0, N, size=count))
    edge_m = sorted({0, M - 1, *[min(M - 1, v) for t in range(tile_m, M, tile_m) for v in (t - 1, t)]})
    edge_n = sorted({0, N - 1, *[min(N - 1, v) for t in range(tile_n, N, tile_n) for v in (t - 1, t)]})
    for m in edge_m[:64]:
        for j in (0, N - 1, int(rng.integers(0, N))):
            ms.append(m)
            js.append(j)
    for j in edge_n[:256]:
        for m in (0, M - 1, int(rng.integers(0, M))):
            ms.append(m)
            js.append(j)
    return np.asarray(ms, dtype=np.int64), np.asarray(js, dtype=np.int64)


def guarded_empty(shape, dtype, device, guard_elems=64, fill=None):
    """A tensor view with sentinel guard bands on both sides, 16-byte aligned.
    Returns (view, full_buffer, sentinel_value)."""
    n = int(np.prod(shape))
    buf = torch.empty(n + 2 * guard_elems, dtype=dtype, device=device)
    if dtype.is_floating_point:
        sentinel = -12345.0 if fill is None else fill
    else:
        sentinel = -77 if fill is None else fill
    buf.fill_(sentinel)
    view = buf[guard_elems:guard_elems + n].view(shape)
    assert view.data_ptr() % 16 == 0
    return view, buf, sentinel


def guards_intact(buf: torch.Tensor, n: int, guard_elems=64, sentinel=None) -> bool:
    head = buf[:guard_elems]
    tail = buf[guard_elems + n:]
    return bool((head == sentinel).all().item() and (tail == sentinel).all().item())


# ---- straight-through backward of the FBI-linear forward
# dx (bf16): the W1A16 form with g = dy * alpha as the input:
#   |dx - ref| <= 1e-4 * sum_j |dy_mj alpha_j|  +  half a bf16 ulp of (|ref| + that);
# dw (fp32): |dw - ref| <= 1e-4 * |alpha_j| * sum_m |dy_mj x_mk|  +  one fp32 ulp of |ref|;
# dalpha (fp32): |dalpha - ref| <= 1e-4 * sum_m |dy_mj| sum_k |x_mk|  +  one fp32 ulp of |ref|.
def _f32_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 23)


def ste_dx_bound(dy_abs: np.ndarray, alpha: np.ndarray, ref: np.ndarray, ms) -> np.ndarray:
    tol = W1A16_REL * (dy_abs @ np.abs(alpha.astype(np.float64)))[ms]
    return tol + 0.5 * bf16_ulp(np.abs(ref) + tol)


def ste_dw_bound(dy_abs: np.ndarray, x_abs: np.ndarray, alpha: np.ndarray, ref: np.ndarray, js, ks) -> np.ndarray:
    s = np.einsum("mi,mi->i", dy_abs[:, js], x_abs[:, ks])
    return W1A16_REL * np.abs(alpha.astype(np.float64))[js] * s + _f32_ulp(ref)


def ste_dalpha_bound(dy_abs: np.ndarray, x_abs: np.ndarray, ref: np.ndarray, js) -> np.ndarray:
    return W1A16_REL * (dy_abs[:, js].T @ x_abs.sum(axis=1)) + _f32_ulp(ref)
