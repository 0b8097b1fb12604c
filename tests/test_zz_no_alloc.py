"""ttt_apply_noalloc against ttt_apply, through the C ABI.

ttt_apply_noalloc is for callers that cannot hand the library device memory
for scratch: a host whose GPU memory is fully reserved in its own pool, a
plugin environment that forbids cudaMalloc/cudaFree, or a query loop that must
never enter the allocator.  Instead of a workspace it uses one fixed 8 MiB
array that the library keeps in device memory.  It has to give the same
outputs as the workspace-based ttt_apply, including on consecutive calls that
reuse (and must not be disturbed by) what the previous call left in that array.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

from test_weight_layers_b200 import ttt as T

from _gpu import DevWeights, need_gpu, rand_tokens, rand_weights, rel_fro, f64

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-5}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _reference(W, Q, T_, dm):
    ws = T.workspace(dm, T_, T.dtype_code(Q.dtype))
    O = torch.zeros_like(Q)
    T.ttt_apply(W.abi, Q, O, T_, dm, T.io_cfg(), ws)
    assert T.ttt_poll_status(ws) == T.TTT_OK
    return O


@pytest.mark.parametrize("dtype,H,d,m,T_", [
    (torch.bfloat16, 4, 192, 768, 250_000),   # spans two internal token chunks of the fixed scratch
    (torch.bfloat16, 2, 128, 256, 1_000),
    (torch.float32, 2, 64, 128, 300),
])
def test_noalloc_matches_apply_on_two_consecutive_calls(dtype, H, d, m, T_):
    dm = T.dims(H, d, m)
    for call in range(2):
        W = DevWeights(*rand_weights(H, d, m, 100 + call))
        Q = rand_tokens(T_, H, d, dtype, 200 + call).cuda()
        ref = _reference(W, Q, T_, dm)
        O = torch.full_like(Q, float("nan"))
        T.ttt_apply_noalloc(W.abi, Q, O, T_, dm, T.io_cfg())
        torch.cuda.synchronize()
        err = rel_fro(f64(O), f64(ref))
        assert err <= TOL[dtype], (call, err)
        # same kernels on the same rows (the apply is independent per token), so the
        # outputs agree bit for bit, whatever token chunk a row falls in
        assert torch.equal(O, ref), call


def test_noalloc_rejects_dims_beyond_its_scratch():
    dm = T.dims(8, 192, 768)  # 8*H*m*d bytes of bf16 weight copies exceed the 8 MiB array
    W = DevWeights(*rand_weights(8, 192, 768, 1))
    Q = rand_tokens(256, 8, 192, torch.bfloat16, 2).cuda()
    O = torch.zeros_like(Q)
    rc = T.lib().ttt_apply_noalloc(W.abi, ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(O.data_ptr()), 256, dm,
                                   ctypes.byref(T.io_cfg()), T.TTT_BF16, ctypes.c_void_p(0))
    assert rc == T.TTT_ERR_SCRATCH
    assert "8 MiB" in T.lib().ttt_status_string(rc).decode()
