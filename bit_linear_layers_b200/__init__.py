"""Binarized linear layers on NVIDIA B200 (sm_100a).

Thin ctypes binding over ``libbitlinear.so`` (C ABI in ``include/bitlinear.h``).
Each function marshals torch tensors into device pointers and the current
CUDA stream and calls the entry point of the same name; every step of the
computation runs in the library's CUDA kernels. There is no CPU fallback:
if the library is missing, importing the binding raises.

    bin_pack(W, mode)                      -> packed, alpha[, beta]
    bin_linear_w1a16(x, packed, alpha)     -> y (bf16)
    bitlinear_w1a8(x, packed, beta)        -> y (fp32)
    bitlinear_w158a8(x, packed, beta)      -> y (fp32), b1.58 ternary weights
    bitlinear_w1a8_ex(x, packed, beta, f)  -> y (fp32), per-tensor / Eq.(6) quantisers
    bin_xnor_gemm(a, b, K)                 -> dot (int32), W1A1
    bin_linear_w1a16_backward(x, packed, alpha, dy) -> dx, dW, dalpha (straight-through)
    W1A16Stack(levels).run()               decode through a stack of layers in one launch
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbitlinear.so")

BL_OK = 0
BL_ERR_INVALID_ARG = -1
BL_ERR_UNSUPPORTED = -2
BL_ERR_CUDA = -3
BL_ERR_TIMEOUT = -4
BL_ERR_NO_DEVICE = -5
BL_ERR_SCRATCH_LIMIT = -6
W1A8_NOALLOC_SCRATCH_BYTES = 4 << 20

BL_FLAG_OVERLAP_PREVIOUS = 1

BL_PACK_FBI = 0
BL_PACK_BITNET = 1
BL_PACK_TERNARY = 2

BL_OP_PACK_FBI = 0
BL_OP_PACK_BITNET = 1
BL_OP_W1A16 = 2
BL_OP_W1A8 = 3
BL_OP_PACK_TERNARY = 4
BL_OP_W158A8 = 5
BL_OP_W1A8_EX = 6
BL_OP_W1A16_STACK = 7
BL_OP_W1A16_BACKWARD = 8

BL_W1A8_TERNARY = 1
BL_W1A8_PER_TENSOR = 2
BL_W1A8_NONNEG = 4


class StackJob(ctypes.Structure):
    """bl_stack_job: one linear of a stack level."""
    _fields_ = [("packed", ctypes.c_void_p), ("alpha", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("N", ctypes.c_int64)]


class StackLevel(ctypes.Structure):
    """bl_stack_level: one input vector and the linears that read it."""
    _fields_ = [("x", ctypes.c_void_p), ("K", ctypes.c_int64), ("first_job", ctypes.c_int32),
                ("num_jobs", ctypes.c_int32)]


# every symbol include/bitlinear.h declares, with its ctypes signature
_i64 = ctypes.c_int64
_p = ctypes.c_void_p
_int = ctypes.c_int
_sz = ctypes.c_size_t
SIGNATURES = {
    "bl_abi_version": ([], _int),
    "bl_status_string": ([_int], ctypes.c_char_p),
    "bl_workspace_bytes": ([_int, _i64, _i64, _i64], _sz),
    "bin_pack": ([_p, _i64, _i64, _int, _p, _p, _p, _p, _sz, _p], _int),
    "bin_linear_w1a16": ([_p, _p, _p, _p, _i64, _i64, _i64, _p], _int),
    "bin_linear_w1a16_ex": ([_p, _p, _p, _p, _i64, _i64, _i64, ctypes.c_uint, _p], _int),
    "bitlinear_w1a8": ([_p, _p, _p, _p, _i64, _i64, _i64, _p, _sz, _p], _int),
    "bitlinear_w1a8_debug": ([_p, _p, _p, _p, _i64, _i64, _i64, _p, _sz, _p, _p, _p, _p, _p, _p], _int),
    "bl_device_error": ([_p, _int, ctypes.POINTER(_int)], _int),
    "bitlinear_w1a8_noalloc": ([_p, _p, _p, _p, _i64, _i64, _i64, _p], _int),
    "bin_xnor_gemm": ([_p, _p, _p, _i64, _i64, _i64, _p], _int),
    "bin_linear_w1a16_stack": ([_p, _int, _p, _int, _p, _sz, _p], _int),
    "bin_linear_w1a16_stack_batch": ([_p, _int, _p, _int, _i64, _p, _sz, _p], _int),
    "bin_linear_w1a16_backward": ([_p, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _p, _sz, _p], _int),
    "bitlinear_w1a8_ex": ([_p, _p, _p, _p, _i64, _i64, _i64, ctypes.c_uint, _p, _sz, _p, _p, _p, _p], _int),
    "bitlinear_w158a8": ([_p, _p, _p, _p, _i64, _i64, _i64, _p, _sz, _p], _int),
    "bitlinear_w158a8_debug": ([_p, _p, _p, _p, _i64, _i64, _i64, _p, _sz, _p, _p, _p, _p, _p, _p], _int),
}


class BitLinearError(RuntimeError):
    def __init__(self, name: str, status: int):
        self.status = status
        super().__init__(f"{name} failed: {status} ({status_string(status)})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python bit_linear_layers_b200/build.py` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (args, res) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.bl_status_string(int(status)).decode()


def workspace_bytes(op: int, M: int, N: int, K: int) -> int:
    return int(lib.bl_workspace_bytes(int(op), int(M), int(N), int(K)))


def _check(name: str, rc: int) -> None:
    if rc != BL_OK:
        raise BitLinearError(name, rc)


def _dev_ptr(t: torch.Tensor | None, dtype: torch.dtype, name: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _workspace(op, M, N, K, device, ws):
    need = workspace_bytes(op, M, N, K)
    if ws is None and need:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
    return ws, need


# ---------------------------------------------------------------- entry points


def bin_pack(W: torch.Tensor, mode: int = BL_PACK_FBI, *, packed=None, alpha=None, beta=None,
             ws=None):
    """Binarise W [N, K] fp32 into packed signs [N, K/32] int32 (bit patterns)
    and scales. FBI: returns (packed, alpha[N]). BitNet: returns
    (packed, alpha[1] = mean W, beta[1] = mean |W|). Ternary (b1.58): returns
    (packed [N, K/16] with a +1 and a -1 plane per 128-k block, beta[1] = mean |W|)."""
    N, K = W.shape
    dev = W.device
    ternary = mode == BL_PACK_TERNARY
    if packed is None:
        packed = torch.empty((N, K // 16 if ternary else K // 32), dtype=torch.int32, device=dev)
    if alpha is None and not ternary:
        alpha = torch.empty(N if mode == BL_PACK_FBI else 1, dtype=torch.float32, device=dev)
    if mode != BL_PACK_FBI and beta is None:
        beta = torch.empty(1, dtype=torch.float32, device=dev)
    op = {BL_PACK_FBI: BL_OP_PACK_FBI, BL_PACK_BITNET: BL_OP_PACK_BITNET}.get(mode, BL_OP_PACK_TERNARY)
    ws, need = _workspace(op, 0, N, K, dev, ws)
    rc = lib.bin_pack(_dev_ptr(W, torch.float32, "W"), N, K, int(mode),
                      _dev_ptr(packed, torch.int32, "packed"), _dev_ptr(alpha, torch.float32, "alpha"),
                      _dev_ptr(beta, torch.float32, "beta"), _dev_ptr(ws, torch.uint8, "ws"),
                      ws.numel() if ws is not None else 0, _stream(dev))
    _check("bin_pack", rc)
    if ternary:
        return packed, beta
    return (packed, alpha) if mode == BL_PACK_FBI else (packed, alpha, beta)


def bin_linear_w1a16(x: torch.Tensor, packed: torch.Tensor, alpha: torch.Tensor, *, out=None,
                     flags: int = 0):
    """FBI-linear forward: y[m, j] = bf16(alpha[j] * sum_k sign_jk x[m, k]).
    ``flags`` (bin_linear_w1a16_ex): BL_FLAG_OVERLAP_PREVIOUS lets the
    single-token kernel stream its weights while the previous kernel on the
    stream finishes; only valid when that kernel does not write them."""
    M, K = x.shape
    N = packed.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    args = (_dev_ptr(x, torch.bfloat16, "x"), _dev_ptr(packed, torch.int32, "packed"),
            _dev_ptr(alpha, torch.float32, "alpha"), _dev_ptr(out, torch.bfloat16, "out"), M, N, K)
    if flags:
        rc = lib.bin_linear_w1a16_ex(*args, int(flags), _stream(x.device))
        _check("bin_linear_w1a16_ex", rc)
    else:
        rc = lib.bin_linear_w1a16(*args, _stream(x.device))
        _check("bin_linear_w1a16", rc)
    return out


def bin_linear_w1a16_backward(x: torch.Tensor, packed: torch.Tensor, alpha: torch.Tensor, dy: torch.Tensor, *,
                              want_dx: bool = True, want_dw: bool = True, dx=None, dw=None, dalpha=None, ws=None):
    """Straight-through backward of the FBI-linear forward: returns (dx [M, K]
    bf16 or None, dw [N, K] fp32 or None, dalpha [N] fp32 or None)."""
    M, K = x.shape
    N = packed.shape[0]
    dev = x.device
    if want_dx and dx is None:
        dx = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    if want_dw and dw is None:
        dw = torch.empty((N, K), dtype=torch.float32, device=dev)
    if want_dw and dalpha is None:
        dalpha = torch.empty(N, dtype=torch.float32, device=dev)
    if not want_dx:
        dx = None
    if not want_dw:
        dw = dalpha = None
    ws, _ = _workspace(BL_OP_W1A16_BACKWARD, M, N, K, dev, ws)
    rc = lib.bin_linear_w1a16_backward(
        _dev_ptr(x, torch.bfloat16, "x"), _dev_ptr(packed, torch.int32, "packed"),
        _dev_ptr(alpha, torch.float32, "alpha"), _dev_ptr(dy, torch.bfloat16, "dy"),
        _dev_ptr(dx, torch.bfloat16, "dx"), _dev_ptr(dw, torch.float32, "dw"),
        _dev_ptr(dalpha, torch.float32, "dalpha"), M, N, K, _dev_ptr(ws, torch.uint8, "ws"),
        ws.numel() if ws is not None else 0, _stream(dev))
    _check("bin_linear_w1a16_backward", rc)
    return dx, dw, dalpha


class W1A16Stack:
    """A stack of FBI-linear layers decoded by bin_linear_w1a16_stack(_batch).

    `levels` is a list of (x, linears), x a bf16 [K] or [M, K] device tensor
    (M tokens, 1 <= M <= 16, the same for every level) and linears a list of
    (packed, alpha, y) with y a bf16 [N] or [M, N] tensor the call writes.
    Every y is its own buffer; a level's x is either exactly the y of a
    linear of an earlier level or a buffer no linear writes. The descriptor
    arrays are built once; run() enqueues the whole stack on the current
    stream."""

    def __init__(self, levels, *, ws=None):
        jobs, lvls = [], []
        self._keep = []
        dev = None
        M = None
        for x, linears in levels:
            K = x.shape[-1]
            m = x.numel() // K
            if x.numel() != m * K or (M is not None and m != M):
                raise ValueError("stack inputs are [M, K] with the same M for every level")
            M = m
            dev = x.device
            lvls.append(StackLevel(_dev_ptr(x, torch.bfloat16, "x"), K, len(jobs), len(linears)))
            for packed, alpha, y in linears:
                N = packed.shape[0]
                if y.numel() != M * N or packed.shape[1] * 32 != K:
                    raise ValueError("linear shapes do not match the level input")
                jobs.append(StackJob(_dev_ptr(packed, torch.int32, "packed"), _dev_ptr(alpha, torch.float32, "alpha"),
                                     _dev_ptr(y, torch.bfloat16, "y"), N))
                self._keep += [packed, alpha, y]
            self._keep.append(x)
        self._levels = (StackLevel * max(len(lvls), 1))(*lvls)
        self._jobs = (StackJob * max(len(jobs), 1))(*jobs)
        self.num_levels, self.num_jobs = len(lvls), len(jobs)
        self.M = M or 1
        self.device = dev
        total_n = sum(j.N for j in jobs)
        self.ws, self.ws_bytes = _workspace(BL_OP_W1A16_STACK, self.M, total_n, 0, dev, ws)

    def run(self):
        rc = lib.bin_linear_w1a16_stack_batch(ctypes.byref(self._levels), self.num_levels, ctypes.byref(self._jobs),
                                              self.num_jobs, self.M, _dev_ptr(self.ws, torch.uint8, "ws"),
                                              self.ws.numel(), _stream(self.device))
        _check("bin_linear_w1a16_stack_batch", rc)


def bitlinear_w1a8(x: torch.Tensor, packed: torch.Tensor, beta: torch.Tensor, *, out=None, ws=None):
    """BitNet BitLinear forward: LN, per-token absmax int8, +-1 GEMM, beta*gamma/128."""
    M, K = x.shape
    N = packed.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=x.device)
    ws, _ = _workspace(BL_OP_W1A8, M, N, K, x.device, ws)
    rc = lib.bitlinear_w1a8(_dev_ptr(x, torch.bfloat16, "x"), _dev_ptr(packed, torch.int32, "packed"),
                            _dev_ptr(beta, torch.float32, "beta"), _dev_ptr(out, torch.float32, "out"),
                            M, N, K, _dev_ptr(ws, torch.uint8, "ws"), ws.numel() if ws is not None else 0,
                            _stream(x.device))
    _check("bitlinear_w1a8", rc)
    return out


def bitlinear_w1a8_debug(x, packed, beta, *, xq_in=None, gamma_in=None, ws=None):
    """As bitlinear_w1a8, also returning (xq int8 [M,K], gamma fp64 [M],
    acc int32 [M,N]). With xq_in/gamma_in the LN/quant step is skipped."""
    M, K = (xq_in.shape if xq_in is not None else x.shape)
    N = packed.shape[0]
    dev = packed.device
    y = torch.empty((M, N), dtype=torch.float32, device=dev)
    xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    gamma = torch.empty(M, dtype=torch.float64, device=dev)
    acc = torch.empty((M, N), dtype=torch.int32, device=dev)
    ws, _ = _workspace(BL_OP_W1A8, M, N, K, dev, ws)
    rc = lib.bitlinear_w1a8_debug(
        _dev_ptr(x, torch.bfloat16, "x") if x is not None else None,
        _dev_ptr(packed, torch.int32, "packed"), _dev_ptr(beta, torch.float32, "beta"),
        _dev_ptr(y, torch.float32, "y"), M, N, K, _dev_ptr(ws, torch.uint8, "ws"),
        ws.numel() if ws is not None else 0, _dev_ptr(xq, torch.int8, "xq"),
        _dev_ptr(gamma, torch.float64, "gamma"), _dev_ptr(acc, torch.int32, "acc"),
        _dev_ptr(xq_in, torch.int8, "xq_in"), _dev_ptr(gamma_in, torch.float64, "gamma_in"),
        _stream(dev))
    _check("bitlinear_w1a8_debug", rc)
    return y, xq, gamma, acc


def bitlinear_w158a8(x: torch.Tensor, packed: torch.Tensor, beta: torch.Tensor, *, out=None, ws=None):
    """BitNet b1.58 BitLinear forward: bitlinear_w1a8 with ternary weights
    (packed from bin_pack(..., BL_PACK_TERNARY), [N, K/16])."""
    M, K = x.shape
    N = packed.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=x.device)
    ws, _ = _workspace(BL_OP_W158A8, M, N, K, x.device, ws)
    rc = lib.bitlinear_w158a8(_dev_ptr(x, torch.bfloat16, "x"), _dev_ptr(packed, torch.int32, "packed"),
                              _dev_ptr(beta, torch.float32, "beta"), _dev_ptr(out, torch.float32, "out"),
                              M, N, K, _dev_ptr(ws, torch.uint8, "ws"), ws.numel() if ws is not None else 0,
                              _stream(x.device))
    _check("bitlinear_w158a8", rc)
    return out


def bitlinear_w158a8_debug(x, packed, beta, *, xq_in=None, gamma_in=None, ws=None):
    """As bitlinear_w158a8, also returning (xq int8 [M,K], gamma fp64 [M],
    acc int32 [M,N]). With xq_in/gamma_in the LN/quant step is skipped."""
    M, K = (xq_in.shape if xq_in is not None else x.shape)
    N = packed.shape[0]
    dev = packed.device
    y = torch.empty((M, N), dtype=torch.float32, device=dev)
    xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    gamma = torch.empty(M, dtype=torch.float64, device=dev)
    acc = torch.empty((M, N), dtype=torch.int32, device=dev)
    ws, _ = _workspace(BL_OP_W158A8, M, N, K, dev, ws)
    rc = lib.bitlinear_w158a8_debug(
        _dev_ptr(x, torch.bfloat16, "x") if x is not None else None,
        _dev_ptr(packed, torch.int32, "packed"), _dev_ptr(beta, torch.float32, "beta"),
        _dev_ptr(y, torch.float32, "y"), M, N, K, _dev_ptr(ws, torch.uint8, "ws"),
        ws.numel() if ws is not None else 0, _dev_ptr(xq, torch.int8, "xq"),
        _dev_ptr(gamma, torch.float64, "gamma"), _dev_ptr(acc, torch.int32, "acc"),
        _dev_ptr(xq_in, torch.int8, "xq_in"), _dev_ptr(gamma_in, torch.float64, "gamma_in"),
        _stream(dev))
    _check("bitlinear_w158a8_debug", rc)
    return y, xq, gamma, acc


def bitlinear_w1a8_ex(x: torch.Tensor, packed: torch.Tensor, beta: torch.Tensor, flags: int, *, out=None,
                      ws=None, debug: bool = False):
    """bitlinear_w1a8 with the page's other activation quantisers
    (BL_W1A8_PER_TENSOR: Eq.(5) over the matrix; BL_W1A8_NONNEG: Eq.(6)) and/or
    ternary weights (BL_W1A8_TERNARY). Returns y, or (y, xq, gamma, acc) with
    debug=True."""
    M, K = x.shape
    N = packed.shape[0]
    dev = x.device
    y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=dev)
    extra = [None, None, None]
    if debug:
        extra = [torch.empty((M, K), dtype=torch.int8, device=dev), torch.empty(M, dtype=torch.float64, device=dev),
                 torch.empty((M, N), dtype=torch.int32, device=dev)]
    op = BL_OP_W1A8_EX if flags & (BL_W1A8_PER_TENSOR | BL_W1A8_NONNEG) else BL_OP_W1A8
    ws, _ = _workspace(op, M, N, K, dev, ws)
    rc = lib.bitlinear_w1a8_ex(
        _dev_ptr(x, torch.bfloat16, "x"), _dev_ptr(packed, torch.int32, "packed"),
        _dev_ptr(beta, torch.float32, "beta"), _dev_ptr(y, torch.float32, "y"), M, N, K, int(flags),
        _dev_ptr(ws, torch.uint8, "ws"), ws.numel() if ws is not None else 0,
        _dev_ptr(extra[0], torch.int8, "xq"), _dev_ptr(extra[1], torch.float64, "gamma"),
        _dev_ptr(extra[2], torch.int32, "acc"), _stream(dev))
    _check("bitlinear_w1a8_ex", rc)
    return (y, *extra) if debug else y


def bitlinear_w1a8_noalloc(x: torch.Tensor, packed: torch.Tensor, beta: torch.Tensor, *, out=None):
    """bitlinear_w1a8 without a workspace, for callers that cannot allocate
    device memory while they run: the codes and gamma live in a fixed 4 MiB
    scratch array inside the library (bl_workspace_bytes(BL_OP_W1A8, M, N, K)
    must fit in it). Calls that overlap on the GPU share that array and race."""
    M, K = x.shape
    N = packed.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=x.device)
    rc = lib.bitlinear_w1a8_noalloc(_dev_ptr(x, torch.bfloat16, "x"), _dev_ptr(packed, torch.int32, "packed"),
                                    _dev_ptr(beta, torch.float32, "beta"), _dev_ptr(out, torch.float32, "out"),
                                    M, N, K, _stream(x.device))
    _check("bitlinear_w1a8_noalloc", rc)
    return out


def bin_xnor_gemm(a: torch.Tensor, b: torch.Tensor, K: int, *, out=None):
    """W1A1: dot[m, n] = K - 2 * popcount(a[m] XOR b[n]) for packed +-1 rows
    a [M, K/32] and b [N, K/32] (int32 bit patterns); returns int32 [M, N]."""
    M, N = a.shape[0], b.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.int32, device=a.device)
    rc = lib.bin_xnor_gemm(_dev_ptr(a, torch.int32, "a"), _dev_ptr(b, torch.int32, "b"),
                           _dev_ptr(out, torch.int32, "out"), M, N, K, _stream(a.device))
    _check("bin_xnor_gemm", rc)
    return out


def device_error(clear: bool = True, device=None) -> tuple[int, int]:
    """(status, where) of the first in-kernel fault on the current device."""
    where = ctypes.c_int(0)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    rc = lib.bl_device_error(_stream(dev), int(bool(clear)), ctypes.byref(where))
    return int(rc), int(where.value)
