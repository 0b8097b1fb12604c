"""Python binding of libttt.so (argument marshalling only).

Each function has the name of its C entry point in include/ttt.h and takes
torch tensors that already live on the GPU; it passes their device pointers,
sizes and the current CUDA stream to the library and raises TTTError on a
nonzero status.  No arithmetic of the layer happens here, and there is no
fallback: if the library cannot be loaded every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libttt.so")

TTT_OK, TTT_ERR_INVALID, TTT_ERR_UNSUPPORTED, TTT_ERR_WORKSPACE = 0, -1, -2, -3
TTT_ERR_CUDA, TTT_ERR_TIMEOUT, TTT_ERR_ALIGN, TTT_ERR_SCRATCH = -4, -5, -6, -7
TTT_ERR_RANGE = -8
TTT_FP32, TTT_BF16 = 0, 1


class TTTError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {code} ({msg})")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int), ("d", ctypes.c_int), ("m", ctypes.c_int)]


class Weights(ctypes.Structure):
    _fields_ = [("W1", ctypes.c_void_p), ("W3", ctypes.c_void_p), ("W2", ctypes.c_void_p)]


class NSCfg(ctypes.Structure):
    _fields_ = [("iters", ctypes.c_int), ("a", ctypes.c_float), ("b", ctypes.c_float), ("c", ctypes.c_float),
                ("eps", ctypes.c_float), ("lr", ctypes.c_float), ("renorm", ctypes.c_int)]


class IOCfg(ctypes.Structure):
    _fields_ = [("qk_l2norm", ctypes.c_int), ("ld_q", ctypes.c_int64), ("ld_k", ctypes.c_int64),
                ("ld_v", ctypes.c_int64), ("ld_o", ctypes.c_int64)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libttt.so; raises if it is missing (build it with test_weight_layers_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m test_weight_layers_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I, SZ, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        sigs = {
            "ttt_workspace_bytes": (SZ, [Dims, I64, I]),
            "ttt_reset_status": (I, [P, SZ, P]),
            "ttt_poll_status": (I, [P, P]),
            "ttt_l2norm": (I, [P, I64, Dims, I64, I, P]),
            "ttt_shortconv2d": (I, [P, I64, P, I64, P, I, I, I, I, I, I, P]),
            "ttt_grad": (I, [Weights, P, P, P, I64, Dims, ctypes.POINTER(IOCfg), I, P, P, SZ, P]),
            "ttt_grad_prepared": (I, [Weights, P, P, P, I64, Dims, ctypes.POINTER(IOCfg), I, P, P, SZ, P]),
            "ttt_step": (I, [Weights, P, ctypes.POINTER(NSCfg), Dims, I, P, SZ, P]),
            "ttt_update": (I, [Weights, P, P, P, I64, I, ctypes.POINTER(NSCfg), Dims, ctypes.POINTER(IOCfg), I, P, SZ,
                               P]),
            "ttt_update_conv": (I, [Weights, P, P, P, I64, I, ctypes.POINTER(NSCfg), P, I, I, I, Dims,
                                    ctypes.POINTER(IOCfg), I, P, SZ, P]),
            "ttt_apply": (I, [Weights, P, P, I64, Dims, ctypes.POINTER(IOCfg), I, P, SZ, P]),
            "ttt_apply_noalloc": (I, [Weights, P, P, I64, Dims, ctypes.POINTER(IOCfg), I, P]),
            "ttt_chunked": (I, [Weights, P, P, P, P, P, I64, I64, I, I, ctypes.POINTER(NSCfg), Dims,
                                ctypes.POINTER(IOCfg), I, P, SZ, P]),
            "ttt_host_buffer_bytes": (SZ, [Dims, I64, I, I]),
            "ttt_layer_host": (I, [Weights, P, P, P, P, P, I64, I64, I, I, ctypes.POINTER(NSCfg), P, I, I, Dims,
                                   ctypes.POINTER(IOCfg), I, P, SZ, P, SZ, P]),
            "ttt_gate_workspace_bytes": (SZ, [I64, I]),
            "ttt_output_gate": (I, [P, I64, P, P, I64, I64, I, I, P, SZ, P]),
            "ttt_status_string": (ctypes.c_char_p, [I]),
            "ttt_compiled_arch": (I, []),
            "ttt_kernel_binary_version": (I, [ctypes.POINTER(I)]),
            "ttt_selftest_wait_timeout": (I, [P, SZ, ctypes.c_uint, P]),
            "ttt_launch_count": (ctypes.c_uint64, []),
            "ttt_profile_enable": (I, [I]),
            "ttt_profile_reset": (I, []),
            "ttt_profile_query": (I, [I, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_uint64)]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(fn: str, rc: int):
    if rc != TTT_OK:
        raise TTTError(fn, rc, lib().ttt_status_string(rc).decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return TTT_BF16
    if t == torch.float32:
        return TTT_FP32
    raise ValueError(f"unsupported dtype {t}")


def dims(heads: int, d: int, m: int) -> Dims:
    return Dims(heads, d, m)


def weights(W1: torch.Tensor, W3: torch.Tensor, W2: torch.Tensor) -> Weights:
    for w in (W1, W3, W2):
        if w.dtype != torch.float32 or not w.is_cuda or not w.is_contiguous():
            raise ValueError("fast weights must be contiguous fp32 CUDA tensors")
    return Weights(W1.data_ptr(), W3.data_ptr(), W2.data_ptr())


def ns_cfg(iters=5, a=3.4445, b=-4.7750, c=2.0315, eps=1e-7, lr=1.0, renorm=1) -> NSCfg:
    return NSCfg(iters, a, b, c, eps, lr, renorm)


def io_cfg(qk_l2norm=1, ld_q=0, ld_k=0, ld_v=0, ld_o=0) -> IOCfg:
    return IOCfg(qk_l2norm, ld_q, ld_k, ld_v, ld_o)


def ttt_workspace_bytes(dm: Dims, T: int, dtype: int) -> int:
    return int(lib().ttt_workspace_bytes(dm, T, dtype))


def workspace(dm: Dims, T: int, dtype: int, device="cuda") -> torch.Tensor:
    """A zeroed workspace tensor of the size the library asks for (torch allocates, 256-byte aligned)."""
    n = ttt_workspace_bytes(dm, T, dtype)
    if n == 0:
        raise ValueError("invalid dims")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def ttt_reset_status(ws: torch.Tensor, stream=None):
    _check("ttt_reset_status", lib().ttt_reset_status(_ptr(ws), ws.numel(), _stream(stream)))


def ttt_poll_status(ws: torch.Tensor, stream=None) -> int:
    return int(lib().ttt_poll_status(_ptr(ws), _stream(stream)))


def ttt_l2norm(X: torch.Tensor, T: int, dm: Dims, ld: int = 0, stream=None):
    _check("ttt_l2norm", lib().ttt_l2norm(_ptr(X), T, dm, ld, dtype_code(X.dtype), _stream(stream)))


def ttt_shortconv2d(V, Vout, taps, N, h, w, C, act=0, ld_v=0, ld_out=0, stream=None):
    _check("ttt_shortconv2d", lib().ttt_shortconv2d(_ptr(V), ld_v, _ptr(Vout), ld_out, _ptr(taps), N, h, w, C, act,
                                                    dtype_code(V.dtype), _stream(stream)))


def ttt_grad(W: Weights, K, V, eta, T, dm: Dims, io: IOCfg, G, ws, stream=None):
    _check("ttt_grad", lib().ttt_grad(W, _ptr(K), _ptr(V), _ptr(eta), T, dm, ctypes.byref(io), dtype_code(K.dtype),
                                      _ptr(G), _ptr(ws), ws.numel(), _stream(stream)))


def ttt_grad_prepared(W: Weights, K, V, eta, T, dm: Dims, io: IOCfg, G, ws, stream=None):
    """ttt_grad reusing the operands the last ttt_grad on `ws` prepared (same K, V, eta, T)."""
    _check("ttt_grad_prepared", lib().ttt_grad_prepared(W, _ptr(K), _ptr(V), _ptr(eta), T, dm, ctypes.byref(io),
                                                        dtype_code(K.dtype), _ptr(G), _ptr(ws), ws.numel(),
                                                        _stream(stream)))


def ttt_step(W: Weights, G, ns: NSCfg, dm: Dims, dtype: int, ws, stream=None):
    _check("ttt_step", lib().ttt_step(W, _ptr(G), ctypes.byref(ns), dm, dtype, _ptr(ws), ws.numel(), _stream(stream)))


def ttt_update(W: Weights, K, V, eta, T, steps, ns: NSCfg, dm: Dims, io: IOCfg, ws, stream=None):
    _check("ttt_update", lib().ttt_update(W, _ptr(K), _ptr(V), _ptr(eta), T, steps, ctypes.byref(ns), dm,
                                          ctypes.byref(io), dtype_code(K.dtype), _ptr(ws), ws.numel(),
                                          _stream(stream)))


def ttt_update_conv(W: Weights, K, V, eta, T, steps, ns: NSCfg, taps, grid_h, grid_w, dm: Dims, io: IOCfg, ws,
                    act=0, stream=None):
    """ttt_update on ShortConv2D(V), the conv folded into the update's operand preparation."""
    _check("ttt_update_conv", lib().ttt_update_conv(W, _ptr(K), _ptr(V), _ptr(eta), T, steps, ctypes.byref(ns),
                                                    _ptr(taps), grid_h, grid_w, act, dm, ctypes.byref(io),
                                                    dtype_code(K.dtype), _ptr(ws), ws.numel(), _stream(stream)))


def ttt_apply(W: Weights, Q, O, T, dm: Dims, io: IOCfg, ws, stream=None):
    _check("ttt_apply", lib().ttt_apply(W, _ptr(Q), _ptr(O), T, dm, ctypes.byref(io), dtype_code(Q.dtype), _ptr(ws),
                                        ws.numel(), _stream(stream)))


def ttt_apply_noalloc(W: Weights, Q, O, T, dm: Dims, io: IOCfg, stream=None):
    """ttt_apply without a workspace: the library uses its own fixed 8 MiB device array as scratch."""
    _check("ttt_apply_noalloc", lib().ttt_apply_noalloc(W, _ptr(Q), _ptr(O), T, dm, ctypes.byref(io),
                                                        dtype_code(Q.dtype), _stream(stream)))


def gate_workspace(T: int, D: int, device="cuda") -> torch.Tensor:
    n = int(lib().ttt_gate_workspace_bytes(T, D))
    if n == 0:
        raise TTTError("ttt_gate_workspace_bytes", TTT_ERR_UNSUPPORTED, "D must be a positive multiple of 256")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def ttt_output_gate(Oprime, Wg, O, T, D, ws, ld_in=0, ld_out=0, stream=None):
    """O = RMSNorm(O') * SiLU(O' W_g^T) per token (bf16 O', O; fp32 W_g [D][D])."""
    _check("ttt_output_gate", lib().ttt_output_gate(_ptr(Oprime), ld_in, _ptr(Wg), _ptr(O), ld_out, T, D,
                                                    dtype_code(Oprime.dtype), _ptr(ws), ws.numel(), _stream(stream)))


def ttt_chunked(W: Weights, Q, K, V, eta, O, T, chunk, order, steps, ns: NSCfg, dm: Dims, io: IOCfg, ws, stream=None):
    _check("ttt_chunked", lib().ttt_chunked(W, _ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(O), T, chunk, order, steps,
                                            ctypes.byref(ns), dm, ctypes.byref(io), dtype_code(Q.dtype), _ptr(ws),
                                            ws.numel(), _stream(stream)))


def ttt_host_buffer_bytes(dm: Dims, T: int, dtype: int, conv: bool = False) -> int:
    return int(lib().ttt_host_buffer_bytes(dm, T, dtype, 1 if conv else 0))


def host_buffer(dm: Dims, T: int, dtype: int, conv: bool = False, device="cuda") -> torch.Tensor:
    """Device staging area for ttt_layer_host (256-byte aligned, as torch allocations are)."""
    n = ttt_host_buffer_bytes(dm, T, dtype, conv)
    if n == 0:
        raise TTTError("ttt_host_buffer_bytes", TTT_ERR_INVALID, "invalid dims")
    return torch.empty(n, dtype=torch.uint8, device=device)


def ttt_layer_host(W: Weights, hQ, hK, hV, hEta, hO, T, chunk, order, steps, ns: NSCfg, dm: Dims, io: IOCfg, dbuf,
                   ws, taps=None, grid_h=0, grid_w=0, stream=None):
    """hQ, hK, hV, hEta, hO are host (pinned CPU) tensors; dbuf, ws, taps and W are on the device.
    chunk > 0 runs the causal carry in the given order (0 apply then update, 1 update then apply)."""
    _check("ttt_layer_host", lib().ttt_layer_host(
        W, _ptr(hQ), _ptr(hK), _ptr(hV), _ptr(hEta), _ptr(hO), T, chunk, order, steps, ctypes.byref(ns), _ptr(taps),
        grid_h, grid_w, dm, ctypes.byref(io), dtype_code(hQ.dtype), _ptr(dbuf), dbuf.numel(), _ptr(ws), ws.numel(),
        _stream(stream)))


def ttt_selftest_wait_timeout(ws, timeout_us: int, stream=None):
    _check("ttt_selftest_wait_timeout", lib().ttt_selftest_wait_timeout(_ptr(ws), ws.numel(), timeout_us,
                                                                        _stream(stream)))


def ttt_launch_count() -> int:
    return int(lib().ttt_launch_count())


TTT_PROF_GRAD, TTT_PROF_APPLY, TTT_PROF_NS, TTT_PROF_NORM, TTT_PROF_CONV, TTT_PROF_REDUCE, TTT_PROF_SHADOW = range(7)
PROF_NAMES = ["grad", "apply", "newton_schulz_step", "row_norms", "shortconv2d", "split_reduce", "weight_shadow"]


def ttt_profile_enable(on: bool = True):
    _check("ttt_profile_enable", lib().ttt_profile_enable(1 if on else 0))


def ttt_profile_reset():
    _check("ttt_profile_reset", lib().ttt_profile_reset())


def ttt_profile_query(kind: int):
    """(total milliseconds, number of recorded launches) of one kernel kind."""
    ms, n = ctypes.c_double(0), ctypes.c_uint64(0)
    _check("ttt_profile_query", lib().ttt_profile_query(kind, ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, int(n.value)
