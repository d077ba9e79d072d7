"""ctypes front end of the C oracle -- TEST INFRASTRUCTURE ONLY.

The oracle is the plain fp64/int64 CPU statement of the binarized linear
layers (see ``oracle.c`` for the formulas, their sources and the readings).
Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the CUDA library never does.

Arrays are numpy arrays: weights fp32, activations as raw bf16 bit patterns
(``uint16``), packed signs ``uint32`` in the layout described in ``oracle.c``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_i64 = ctypes.c_int64
_dbl = ctypes.c_double
_p = ctypes.c_void_p


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """Bindings to one compiled copy of the oracle (the real one by default;
    the mutation tests load deliberately broken copies through ``path``)."""

    def __init__(self, path: str | None = None):
        if path is None:
            path = _build.ensure_built()
        self.path = path
        lib = ctypes.CDLL(path)
        sig = {
            "oracle_pack_fbi": [_p, _i64, _i64, _p, _p],
            "oracle_pack_bitnet": [_p, _i64, _i64, _p, _p, _p],
            "oracle_w1a16": [_p, _p, _p, _i64, _i64, _i64, _p],
            "oracle_w1a16_at": [_p, _p, _p, _i64, _p, _p, _i64, _p],
            "oracle_ln_absmax_quant": [_p, _i64, _i64, _dbl, _p, _p, _p],
            "oracle_w1a8_acc": [_p, _p, _i64, _i64, _i64, _p],
            "oracle_w1a8_acc_at": [_p, _p, _i64, _p, _p, _i64, _p],
            "oracle_w1a8_rescale": [_p, _p, _dbl, _i64, _i64, _p],
            "oracle_w1a1": [_p, _p, _i64, _i64, _i64, _p],
            "oracle_pack_ternary": [_p, _i64, _i64, _dbl, _p, _p],
            "oracle_ln_quant_tensor": [_p, _i64, _i64, _dbl, ctypes.c_int, _p, _p, _p, _p],
            "oracle_w158a8_acc": [_p, _p, _i64, _i64, _i64, _p],
            "oracle_w158a8_acc_at": [_p, _p, _i64, _p, _p, _i64, _p],
            "oracle_w1a16_backward": [_p, _p, _p, _p, _i64, _i64, _i64, _p, _p, _p],
            "oracle_w1a16_backward_at": [_p, _p, _p, _p, _i64, _i64, _i64, ctypes.c_int, _p, _p, _i64, _p],
        }
        for name, args in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = None
        self._lib = lib

    # -- binarise and pack ---------------------------------------------------
    @staticmethod
    def row_words(K: int) -> int:
        return (K + 31) // 32

    def pack_fbi(self, W: np.ndarray):
        """FBI-linear: signs of W and per-output-channel alpha = mean |W_j.|."""
        W = np.ascontiguousarray(W, dtype=np.float32)
        N, K = W.shape
        packed = np.zeros((N, self.row_words(K)), dtype=np.uint32)
        alpha = np.zeros(N, dtype=np.float32)
        self._lib.oracle_pack_fbi(_ptr(W), N, K, _ptr(packed), _ptr(alpha))
        return packed, alpha

    def pack_bitnet(self, W: np.ndarray):
        """BitNet: signs of W - mean(W); returns (packed, alpha_g, beta) in fp64."""
        W = np.ascontiguousarray(W, dtype=np.float32)
        N, K = W.shape
        packed = np.zeros((N, self.row_words(K)), dtype=np.uint32)
        a = np.zeros(1, dtype=np.float64)
        b = np.zeros(1, dtype=np.float64)
        self._lib.oracle_pack_bitnet(_ptr(W), N, K, _ptr(packed), _ptr(a), _ptr(b))
        return packed, float(a[0]), float(b[0])

    # -- W1A16 ----------------------------------------------------------------
    def w1a16(self, x_bf16: np.ndarray, packed: np.ndarray, alpha: np.ndarray, K: int):
        x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        alpha = np.ascontiguousarray(alpha, dtype=np.float32)
        M, N = x.shape[0], packed.shape[0]
        assert x.shape[1] == K and packed.shape[1] == self.row_words(K) and alpha.shape == (N,)
        y = np.zeros((M, N), dtype=np.float64)
        self._lib.oracle_w1a16(_ptr(x), _ptr(packed), _ptr(alpha), M, N, K, _ptr(y))
        return y

    def w1a16_backward(self, x_bf16: np.ndarray, packed: np.ndarray, alpha: np.ndarray, dy_bf16: np.ndarray,
                       K: int):
        """FBI-linear backward with the straight-through estimator (reading
        R18): returns (dx [M, K], dw [N, K], dalpha [N]) in fp64."""
        x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        dy = np.ascontiguousarray(dy_bf16, dtype=np.uint16)
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        alpha = np.ascontiguousarray(alpha, dtype=np.float32)
        M, N = dy.shape
        assert x.shape == (M, K) and packed.shape == (N, self.row_words(K)) and alpha.shape == (N,)
        dx = np.zeros((M, K), dtype=np.float64)
        dw = np.zeros((N, K), dtype=np.float64)
        da = np.zeros(N, dtype=np.float64)
        self._lib.oracle_w1a16_backward(_ptr(x), _ptr(packed), _ptr(alpha), _ptr(dy), M, N, K, _ptr(dx), _ptr(dw),
                                        _ptr(da))
        return dx, dw, da

    def w1a16_backward_at(self, x_bf16, packed, alpha, dy_bf16, K: int, which: str, i0, i1=None):
        """One of the backward outputs at positions: which = "dx" at (m, k) = (i0, i1),
        "dw" at (j, k) = (i0, i1), "dalpha" at j = i0."""
        x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        dy = np.ascontiguousarray(dy_bf16, dtype=np.uint16)
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        alpha = np.ascontiguousarray(alpha, dtype=np.float32)
        M, N = dy.shape
        assert x.shape == (M, K) and packed.shape == (N, self.row_words(K))
        i0 = np.ascontiguousarray(i0, dtype=np.int64)
        i1 = np.ascontiguousarray(np.zeros_like(i0) if i1 is None else i1, dtype=np.int64)
        code = {"dx": 0, "dw": 1, "dalpha": 2}[which]
        lim0 = M if code == 0 else N
        assert i0.size == 0 or (i0.min() >= 0 and i0.max() < lim0)
        assert code == 2 or i1.size == 0 or (i1.min() >= 0 and i1.max() < K)
        out = np.zeros(i0.shape, dtype=np.float64)
        self._lib.oracle_w1a16_backward_at(_ptr(x), _ptr(packed), _ptr(alpha), _ptr(dy), M, N, K, code, _ptr(i0),
                                           _ptr(i1), i0.size, _ptr(out))
        return out

    def w1a16_at(self, x_bf16, packed, alpha, K: int, ms, js):
        x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        alpha = np.ascontiguousarray(alpha, dtype=np.float32)
        ms = np.ascontiguousarray(ms, dtype=np.int64)
        js = np.ascontiguousarray(js, dtype=np.int64)
        assert ms.shape == js.shape
        assert ms.size == 0 or (ms.min() >= 0 and ms.max() < x.shape[0])
        assert js.size == 0 or (js.min() >= 0 and js.max() < packed.shape[0])
        y = np.zeros(ms.shape, dtype=np.float64)
        self._lib.oracle_w1a16_at(_ptr(x), _ptr(packed), _ptr(alpha), K, _ptr(ms), _ptr(js),
                                  ms.size, _ptr(y))
        return y

    # -- W1A8 -----------------------------------------------------------------
    def ln_absmax_quant(self, x_bf16: np.ndarray, eps: float = 1e-5, want_pre: bool = False):
        """Returns (xq int8 M x K, gamma fp64 M[, pre fp64 M x K])."""
        x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        M, K = x.shape
        xq = np.zeros((M, K), dtype=np.int8)
        gamma = np.zeros(M, dtype=np.float64)
        pre = np.zeros((M, K), dtype=np.float64) if want_pre else None
        self._lib.oracle_ln_absmax_quant(_ptr(x), M, K, float(eps), _ptr(xq), _ptr(gamma),
                                         _ptr(pre) if want_pre else None)
        return (xq, gamma, pre) if want_pre else (xq, gamma)

    def ln_quant_tensor(self, x_bf16: np.ndarray, mode: int, eps: float = 1e-5, want_pre: bool = False):
        """Per-tensor quantisation of the LN output: mode 0 = Eq.(5) over the
        whole matrix (codes in [-127, 127]), mode 1 = Eq.(6) (shift by the
        minimum, codes in [0, 127]). Returns (xq, gamma [M] (all equal), eta[, pre])."""
        x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        M, K = x.shape
        xq = np.zeros((M, K), dtype=np.int8)
        gamma = np.zeros(M, dtype=np.float64)
        eta = np.zeros(1, dtype=np.float64)
        pre = np.zeros((M, K), dtype=np.float64) if want_pre else None
        self._lib.oracle_ln_quant_tensor(_ptr(x), M, K, float(eps), int(mode), _ptr(xq), _ptr(gamma),
                                         _ptr(eta), _ptr(pre) if want_pre else None)
        return (xq, gamma, float(eta[0]), pre) if want_pre else (xq, gamma, float(eta[0]))

    def w1a8_acc(self, xq: np.ndarray, packed: np.ndarray, K: int):
        xq = np.ascontiguousarray(xq, dtype=np.int8)
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        M, N = xq.shape[0], packed.shape[0]
        acc = np.zeros((M, N), dtype=np.int64)
        self._lib.oracle_w1a8_acc(_ptr(xq), _ptr(packed), M, N, K, _ptr(acc))
        return acc

    def w1a8_acc_at(self, xq, packed, K: int, ms, js):
        xq = np.ascontiguousarray(xq, dtype=np.int8)
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        ms = np.ascontiguousarray(ms, dtype=np.int64)
        js = np.ascontiguousarray(js, dtype=np.int64)
        assert ms.shape == js.shape
        acc = np.zeros(ms.shape, dtype=np.int64)
        self._lib.oracle_w1a8_acc_at(_ptr(xq), _ptr(packed), K, _ptr(ms), _ptr(js), ms.size,
                                     _ptr(acc))
        return acc

    def w1a8_rescale(self, acc: np.ndarray, gamma: np.ndarray, beta: float):
        acc = np.ascontiguousarray(acc, dtype=np.int64)
        gamma = np.ascontiguousarray(gamma, dtype=np.float64)
        M, N = acc.shape
        y = np.zeros((M, N), dtype=np.float64)
        self._lib.oracle_w1a8_rescale(_ptr(acc), _ptr(gamma), float(beta), M, N, _ptr(y))
        return y

    def w1a8(self, x_bf16, packed, beta: float, K: int, eps: float = 1e-5):
        """Whole BitLinear forward: returns (y fp64, xq, gamma, acc)."""
        xq, gamma = self.ln_absmax_quant(x_bf16, eps)
        acc = self.w1a8_acc(xq, packed, K)
        return self.w1a8_rescale(acc, gamma, beta), xq, gamma, acc

    # -- b1.58 ternary weights -------------------------------------------------
    @staticmethod
    def ternary_row_words(K: int) -> int:
        return ((K + 127) // 128) * 8

    def pack_ternary(self, W: np.ndarray, eps: float = 1e-5):
        """b1.58: RoundClip(W / (gamma + eps), -1, 1) as two bit planes per
        128-k block; returns (packed, gamma = mean |W| in fp64)."""
        W = np.ascontiguousarray(W, dtype=np.float32)
        N, K = W.shape
        packed = np.zeros((N, self.ternary_row_words(K)), dtype=np.uint32)
        g = np.zeros(1, dtype=np.float64)
        self._lib.oracle_pack_ternary(_ptr(W), N, K, float(eps), _ptr(packed), _ptr(g))
        return packed, float(g[0])

    def w158a8_acc(self, xq: np.ndarray, packed: np.ndarray, K: int):
        xq = np.ascontiguousarray(xq, dtype=np.int8)
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        M, N = xq.shape[0], packed.shape[0]
        assert packed.shape[1] == self.ternary_row_words(K)
        acc = np.zeros((M, N), dtype=np.int64)
        self._lib.oracle_w158a8_acc(_ptr(xq), _ptr(packed), M, N, K, _ptr(acc))
        return acc

    def w158a8_acc_at(self, xq, packed, K: int, ms, js):
        xq = np.ascontiguousarray(xq, dtype=np.int8)
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        ms = np.ascontiguousarray(ms, dtype=np.int64)
        js = np.ascontiguousarray(js, dtype=np.int64)
        assert ms.shape == js.shape
        acc = np.zeros(ms.shape, dtype=np.int64)
        self._lib.oracle_w158a8_acc_at(_ptr(xq), _ptr(packed), K, _ptr(ms), _ptr(js), ms.size,
                                       _ptr(acc))
        return acc

    def w158a8(self, x_bf16, packed, beta: float, K: int, eps: float = 1e-5):
        """Whole b1.58 BitLinear forward: returns (y fp64, xq, gamma, acc)."""
        xq, gamma = self.ln_absmax_quant(x_bf16, eps)
        acc = self.w158a8_acc(xq, packed, K)
        return self.w1a8_rescale(acc, gamma, beta), xq, gamma, acc

    # -- W1A1 -----------------------------------------------------------------
    def w1a1(self, a: np.ndarray, b: np.ndarray, K: int):
        a = np.ascontiguousarray(a, dtype=np.uint32)
        b = np.ascontiguousarray(b, dtype=np.uint32)
        M, N = a.shape[0], b.shape[0]
        dot = np.zeros((M, N), dtype=np.int64)
        self._lib.oracle_w1a1(_ptr(a), _ptr(b), M, N, K, _ptr(dot))
        return dot


_default = None


def get() -> Oracle:
    """The real oracle (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def lib_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "liboracle.so")
