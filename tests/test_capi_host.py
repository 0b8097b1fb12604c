"""The C-ABI library loads, exports every entry point the header declares, and
its host-side argument checks return the documented codes before touching a GPU."""
import ctypes
import os
import re

import pytest

from test_weight_layers_b200 import build as B
from test_weight_layers_b200 import ttt as T

HEADER = os.path.join(B.INCLUDE, "ttt.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return T.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w[\w\s\*]*?\b(ttt_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_entry_points():
    names = declared_functions()
    for required in ("ttt_update", "ttt_apply", "ttt_shortconv2d", "ttt_chunked", "ttt_grad", "ttt_step",
                     "ttt_l2norm", "ttt_workspace_bytes", "ttt_poll_status"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_library_is_built_for_sm100a(lib):
    assert lib.ttt_compiled_arch() == 1000


def test_status_strings(lib):
    for code in (T.TTT_OK, T.TTT_ERR_INVALID, T.TTT_ERR_UNSUPPORTED, T.TTT_ERR_WORKSPACE, T.TTT_ERR_CUDA,
                 T.TTT_ERR_TIMEOUT, T.TTT_ERR_ALIGN):
        s = lib.ttt_status_string(code).decode()
        assert s and s != "unknown status"


def test_workspace_bytes(lib):
    d = T.dims(4, 192, 768)
    small = T.ttt_workspace_bytes(d, 1000, T.TTT_BF16)
    big = T.ttt_workspace_bytes(d, 1_000_000, T.TTT_BF16)
    n = 4 * 192 * 768
    assert small >= 3 * n * 4 + 4 * n * 2
    assert big - small >= 2 * (1_000_000 - 1000) * 4 * 4 - 4096
    assert T.ttt_workspace_bytes(T.dims(0, 192, 768), 10, T.TTT_BF16) == 0
    assert T.ttt_workspace_bytes(d, -1, T.TTT_BF16) == 0


FAKE = ctypes.c_void_p(1 << 20)  # 256-aligned, never dereferenced: checks fail before any device work


def _call_update(lib, dims, dtype, ws_bytes, K=FAKE, ld=0, T_=256, eta=FAKE):
    W = T.Weights(1 << 20, 1 << 21, 1 << 22)
    ns = T.ns_cfg()
    io = T.io_cfg(ld_k=ld, ld_v=ld)
    return lib.ttt_update(W, K, FAKE, eta, T_, 1, ctypes.byref(ns), dims, ctypes.byref(io), dtype, FAKE, ws_bytes,
                          None)


def test_host_validation_codes(lib):
    d = T.dims(4, 192, 768)
    need = T.ttt_workspace_bytes(d, 256, T.TTT_BF16)
    assert _call_update(lib, d, T.TTT_BF16, need - 1) == T.TTT_ERR_WORKSPACE
    assert _call_update(lib, T.dims(4, 96, 768), T.TTT_BF16, 1 << 40) == T.TTT_ERR_UNSUPPORTED
    assert _call_update(lib, T.dims(4, 192, 700), T.TTT_BF16, 1 << 40) == T.TTT_ERR_UNSUPPORTED
    assert _call_update(lib, d, 7, need) == T.TTT_ERR_INVALID
    assert _call_update(lib, d, T.TTT_BF16, need, ld=100) == T.TTT_ERR_INVALID           # ld < H*d
    assert _call_update(lib, d, T.TTT_BF16, need, ld=772) == T.TTT_ERR_ALIGN             # 1544-byte rows
    assert _call_update(lib, d, T.TTT_BF16, need, K=ctypes.c_void_p((1 << 20) + 2)) == T.TTT_ERR_ALIGN
    assert _call_update(lib, d, T.TTT_BF16, need, K=None) == T.TTT_ERR_INVALID
    assert _call_update(lib, d, T.TTT_BF16, need, eta=None) == T.TTT_ERR_INVALID
    assert _call_update(lib, T.dims(1, 64, 100), T.TTT_FP32, 1 << 40) == T.TTT_ERR_UNSUPPORTED


def test_chunked_and_conv_validation(lib):
    d = T.dims(4, 192, 768)
    W = T.Weights(1 << 20, 1 << 21, 1 << 22)
    ns, io = T.ns_cfg(), T.io_cfg()
    need = T.ttt_workspace_bytes(d, 4096, T.TTT_BF16)
    rc = lib.ttt_chunked(W, FAKE, FAKE, FAKE, FAKE, FAKE, 100000, 0, 0, 1, ctypes.byref(ns), d, ctypes.byref(io),
                         T.TTT_BF16, FAKE, need, None)
    assert rc == T.TTT_ERR_INVALID  # chunk = 0
    rc = lib.ttt_chunked(W, FAKE, FAKE, FAKE, FAKE, FAKE, 100000, 4096, 2, 1, ctypes.byref(ns), d, ctypes.byref(io),
                         T.TTT_BF16, FAKE, need, None)
    assert rc == T.TTT_ERR_INVALID  # order = 2
    rc = lib.ttt_chunked(W, FAKE, FAKE, FAKE, FAKE, FAKE, 100000, 8192, 0, 1, ctypes.byref(ns), d, ctypes.byref(io),
                         T.TTT_BF16, FAKE, need, None)
    assert rc == T.TTT_ERR_WORKSPACE  # workspace sized for 4096-token chunks
    assert lib.ttt_shortconv2d(FAKE, 0, FAKE, 0, FAKE, 2, 4, 4, 12, 0, T.TTT_BF16, None) == T.TTT_ERR_UNSUPPORTED
    assert lib.ttt_shortconv2d(FAKE, 0, FAKE, 0, FAKE, 2, 4, 4, 16, 3, T.TTT_BF16, None) == T.TTT_ERR_INVALID
    assert lib.ttt_shortconv2d(FAKE, 0, FAKE, 0, FAKE, 2, 4, 4, 16, 0, T.TTT_BF16, None) == T.TTT_ERR_INVALID  # alias


def _call_layer_host(lib, dims, dtype, T_, chunk, dbuf_bytes, ws_bytes, taps=None, gh=0, gw=0, hQ=FAKE, order=0):
    W = T.Weights(1 << 20, 1 << 21, 1 << 22)
    ns, io = T.ns_cfg(), T.io_cfg()
    return lib.ttt_layer_host(W, hQ, FAKE, FAKE, FAKE, FAKE, T_, chunk, order, 1, ctypes.byref(ns), taps, gh, gw, dims,
                              ctypes.byref(io), dtype, FAKE, dbuf_bytes, FAKE, ws_bytes, None)


def test_layer_host_validation(lib):
    d = T.dims(4, 192, 768)
    T_ = 1024
    need_ws = T.ttt_workspace_bytes(d, T_, T.TTT_BF16)
    need_db = T.ttt_host_buffer_bytes(d, T_, T.TTT_BF16)
    # staging area: Q, K, V, O token matrices and eta (and the convolved V with conv)
    assert need_db >= 4 * T_ * 4 * 192 * 2 + T_ * 4 * 4
    assert T.ttt_host_buffer_bytes(d, T_, T.TTT_BF16, conv=True) >= need_db + T_ * 4 * 192 * 2
    assert T.ttt_host_buffer_bytes(T.dims(0, 192, 768), T_, T.TTT_BF16) == 0
    assert _call_layer_host(lib, d, T.TTT_BF16, T_, 256, need_db, need_ws, order=2) == T.TTT_ERR_INVALID
    assert _call_layer_host(lib, d, T.TTT_BF16, T_, 256, need_db, need_ws, order=-1) == T.TTT_ERR_INVALID
    assert _call_layer_host(lib, d, T.TTT_BF16, T_, 0, need_db - 1, need_ws) == T.TTT_ERR_WORKSPACE
    assert _call_layer_host(lib, d, T.TTT_BF16, T_, 0, need_db, need_ws - 1) == T.TTT_ERR_WORKSPACE
    assert _call_layer_host(lib, d, T.TTT_BF16, T_, -1, need_db, need_ws) == T.TTT_ERR_INVALID
    assert _call_layer_host(lib, d, T.TTT_BF16, T_, 0, need_db, need_ws, hQ=None) == T.TTT_ERR_INVALID
    # chunk mode needs a workspace for one chunk only
    assert _call_layer_host(lib, d, T.TTT_BF16, T_, 256, need_db, T.ttt_workspace_bytes(d, 256, T.TTT_BF16) - 1) \
        == T.TTT_ERR_WORKSPACE
    # ShortConv2D: T and the chunk must be whole frames
    need_dbc = T.ttt_host_buffer_bytes(d, T_, T.TTT_BF16, conv=True)
    assert _call_layer_host(lib, d, T.TTT_BF16, T_, 0, need_dbc, need_ws, taps=FAKE, gh=7, gw=7) == T.TTT_ERR_INVALID
    assert _call_layer_host(lib, d, T.TTT_BF16, T_, 100, need_dbc, need_ws, taps=FAKE, gh=4, gw=4) \
        == T.TTT_ERR_INVALID


def test_output_gate_validation(lib):
    D, T_ = 1024, 300
    need = lib.ttt_gate_workspace_bytes(T_, D)
    assert need >= D * D * 2 + T_ * 4
    assert lib.ttt_gate_workspace_bytes(T_, 1000) == 0   # D must be a multiple of 256
    call = lambda Op, Wg, O_, D_, dt, ws_bytes: lib.ttt_output_gate(Op, 0, Wg, O_, 0, T_, D_, dt, FAKE, ws_bytes, None)
    A, B, C = ctypes.c_void_p(1 << 21), ctypes.c_void_p(1 << 22), ctypes.c_void_p(1 << 23)
    assert call(A, B, C, D, T.TTT_FP32, need) == T.TTT_ERR_UNSUPPORTED
    assert call(A, B, C, 768 + 8, T.TTT_BF16, need) == T.TTT_ERR_UNSUPPORTED
    assert call(A, B, C, D, T.TTT_BF16, need - 1) == T.TTT_ERR_WORKSPACE
    assert call(A, B, A, D, T.TTT_BF16, need) == T.TTT_ERR_INVALID          # O aliases O'
    assert call(None, B, C, D, T.TTT_BF16, need) == T.TTT_ERR_INVALID
    assert call(ctypes.c_void_p((1 << 21) + 2), B, C, D, T.TTT_BF16, need) == T.TTT_ERR_ALIGN


def test_wide_head_shapes_are_accepted(lib):
    # d and m multiples of 256 run the wide-head path in bf16; the workspace holds its
    # fp16 intermediates (K^, V', Z, dH1, dH3, u: 2 (2 d + 4 m) bytes per token and head)
    d = T.dims(1, 1024, 2048)
    small = T.ttt_workspace_bytes(d, 1000, T.TTT_BF16)
    big = T.ttt_workspace_bytes(d, 2000, T.TTT_BF16)
    assert big - small >= 1000 * 2 * (2 * 1024 + 4 * 2048)
    assert _call_update(lib, d, T.TTT_BF16, small - 1, T_=1000) == T.TTT_ERR_WORKSPACE
    assert _call_update(lib, T.dims(1, 1024, 2000), T.TTT_BF16, 1 << 40) == T.TTT_ERR_UNSUPPORTED
    assert _call_update(lib, T.dims(1, 1024, 2048), T.TTT_FP32, 1 << 40) == T.TTT_ERR_UNSUPPORTED
    # the no-allocation apply has no room for the wide path's per-token intermediate
    W = T.Weights(1 << 20, 1 << 21, 1 << 22)
    rc = lib.ttt_apply_noalloc(W, FAKE, ctypes.c_void_p(1 << 23), 10, T.dims(1, 256, 256),
                               ctypes.byref(T.io_cfg()), T.TTT_BF16, None)
    assert rc == T.TTT_ERR_UNSUPPORTED


def test_update_conv_validation(lib):
    d = T.dims(4, 192, 768)
    W = T.Weights(1 << 20, 1 << 21, 1 << 22)
    ns, io = T.ns_cfg(), T.io_cfg()
    need = T.ttt_workspace_bytes(d, 2 * 37 * 37 + 1, T.TTT_BF16)
    call = lambda T_, gh, gw, dt, act=0: lib.ttt_update_conv(W, FAKE, FAKE, FAKE, T_, 1, ctypes.byref(ns), FAKE, gh, gw,
                                                            act, d, ctypes.byref(io), dt, FAKE, need, None)
    assert call(2 * 37 * 37 + 1, 37, 37, T.TTT_BF16) == T.TTT_ERR_INVALID       # not whole frames
    assert call(2 * 37 * 37, 37, 37, T.TTT_BF16, act=2) == T.TTT_ERR_INVALID    # act is 0 or 1
    assert call(2 * 37 * 37, 0, 37, T.TTT_BF16) == T.TTT_ERR_INVALID
    need32 = T.ttt_workspace_bytes(d, 2 * 37 * 37, T.TTT_FP32)
    assert lib.ttt_update_conv(W, FAKE, FAKE, FAKE, 2 * 37 * 37, 1, ctypes.byref(ns), FAKE, 37, 37, 0, d,
                               ctypes.byref(io), T.TTT_FP32, FAKE, need32, None) == T.TTT_ERR_UNSUPPORTED
