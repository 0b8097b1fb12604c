"""GPU parity of each entry point against the fp64 oracle at small sizes
(several 128-token tiles plus a ragged tail), through the C ABI."""
import ctypes
import numpy as np
import pytest
import torch

import oracle as O
from test_weight_layers_b200 import ttt as T

from _gpu import (TOL_BF16, TOL_FP32, DevWeights, check_status, f64, need_gpu, rand_eta, rand_tokens, rand_weights,
                  rel_fro, weight_errors)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_l2norm_in_place(dtype):
    H, d, T_ = 4, 192, 333
    X = rand_tokens(T_, H, d, dtype, 1, ld=H * d + 8, scale=3.0)
    X[5, :d] = 0  # zero row stays zero (eps clamp)
    ref = O.l2norm_heads(f64(X), H, d)
    Xd = X.cuda()
    T.ttt_l2norm(Xd, T_, T.dims(H, d, 64), ld=H * d + 8)
    torch.cuda.synchronize()
    got = f64(Xd)
    tol = 4e-3 if dtype == torch.bfloat16 else 1e-6
    assert rel_fro(got[:, :H * d], ref) < tol
    assert np.all(got[5, :d] == 0)
    assert np.array_equal(got[:, H * d:], f64(X)[:, H * d:])  # padding untouched


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("act", [0, 1])
def test_shortconv2d(dtype, act):
    N, h, w, C = 3, 5, 7, 64
    V = rand_tokens(N * h * w, 1, C, dtype, 2, ld=C + 8)
    taps = torch.randn((C, 3, 3), generator=torch.Generator().manual_seed(3)) / 3
    ref = O.shortconv2d(f64(V)[:, :C], taps.double().numpy(), N, h, w, act)
    out = torch.zeros((N * h * w, C), dtype=dtype, device="cuda")
    T.ttt_shortconv2d(V.cuda(), out, taps.cuda(), N, h, w, C, act, ld_v=C + 8, ld_out=C)
    torch.cuda.synchronize()
    tol = 5e-3 if dtype == torch.bfloat16 else 1e-6
    assert rel_fro(f64(out), ref) < tol


@pytest.mark.parametrize("H,d,m,T_", [(1, 192, 64, 1), (2, 192, 768, 300), (3, 128, 192, 1000), (4, 192, 256, 129)])
def test_apply_bf16(H, d, m, T_):
    W = DevWeights(*rand_weights(H, d, m, 10 + m))
    Q = rand_tokens(T_, H, d, torch.bfloat16, 11)
    dm = T.dims(H, d, m)
    ws = T.workspace(dm, T_, T.TTT_BF16)
    O_ = torch.full((T_, H * d), float("nan"), dtype=torch.bfloat16, device="cuda")
    T.ttt_apply(W.abi, Q.cuda(), O_, T_, dm, T.io_cfg(), ws)
    check_status(ws)
    ref = O.apply(W.oracle(), f64(Q))
    err = rel_fro(f64(O_), ref)
    assert err < 1e-2, err


def test_apply_bf16_strided_rows():
    H, d, m, T_ = 2, 192, 128, 260
    W = DevWeights(*rand_weights(H, d, m, 12))
    Q = rand_tokens(T_, H, d, torch.bfloat16, 13, ld=H * d + 64)
    dm = T.dims(H, d, m)
    ws = T.workspace(dm, T_, T.TTT_BF16)
    O_ = torch.zeros((T_, H * d + 16), dtype=torch.bfloat16, device="cuda")
    T.ttt_apply(W.abi, Q.cuda(), O_, T_, dm, T.io_cfg(ld_q=H * d + 64, ld_o=H * d + 16), ws)
    check_status(ws)
    ref = O.apply(W.oracle(), f64(Q)[:, :H * d])
    assert rel_fro(f64(O_)[:, :H * d], ref) < 1e-2
    assert torch.all(O_[:, H * d:] == 0)


@pytest.mark.parametrize("qk", [1, 0])
def test_apply_fp32(qk):
    H, d, m, T_ = 2, 64, 128, 77
    W = DevWeights(*rand_weights(H, d, m, 14))
    Q = rand_tokens(T_, H, d, torch.float32, 15)
    dm = T.dims(H, d, m)
    ws = T.workspace(dm, T_, T.TTT_FP32)
    O_ = torch.zeros((T_, H * d), dtype=torch.float32, device="cuda")
    T.ttt_apply(W.abi, Q.cuda(), O_, T_, dm, T.io_cfg(qk_l2norm=qk), ws)
    check_status(ws)
    ref = O.apply(W.oracle(), f64(Q), qk_l2norm=bool(qk))
    assert rel_fro(f64(O_), ref) < 1e-5


def _grad_case(H, d, m, T_, dtype, seed=20):
    W = DevWeights(*rand_weights(H, d, m, seed))
    K = rand_tokens(T_, H, d, dtype, seed + 1)
    V = rand_tokens(T_, H, d, dtype, seed + 2)
    eta = rand_eta(T_, H, seed + 3, scale=1.0)
    return W, K, V, eta


def _run_grad(W, K, V, eta, dm, dtype_code):
    T_ = K.shape[0]
    ws = T.workspace(dm, T_, dtype_code)
    n = dm.heads * dm.m * dm.d
    G = torch.full((3 * n,), float("nan"), dtype=torch.float32, device="cuda")
    T.ttt_grad(W.abi, K.cuda(), V.cuda(), eta.cuda(), T_, dm, T.io_cfg(), G, ws)
    check_status(ws)
    H, d, m = dm.heads, dm.d, dm.m
    g = f64(G)
    return O.FastWeights(g[:n].reshape(H, m, d), g[n:2 * n].reshape(H, m, d), g[2 * n:].reshape(H, d, m)), G


@pytest.mark.parametrize("H,d,m,T_", [(1, 192, 64, 1), (2, 192, 128, 1000), (2, 128, 256, 129), (4, 192, 768, 384)])
def test_grad_bf16(H, d, m, T_):
    W, K, V, eta = _grad_case(H, d, m, T_, torch.bfloat16)
    got, _ = _run_grad(W, K, V, eta, T.dims(H, d, m), T.TTT_BF16)
    ref = O.grad(W.oracle(), O.l2norm_heads(f64(K), H, d), f64(V), f64(eta))
    errs = weight_errors(got, ref)
    assert max(errs) < 2e-2, errs


@pytest.mark.parametrize("H,d,m,T_", [(1, 64, 128, 128), (2, 64, 64, 200), (1, 96, 32, 33)])
def test_grad_fp32(H, d, m, T_):
    W, K, V, eta = _grad_case(H, d, m, T_, torch.float32)
    got, _ = _run_grad(W, K, V, eta, T.dims(H, d, m), T.TTT_FP32)
    ref = O.grad(W.oracle(), O.l2norm_heads(f64(K), H, d), f64(V), f64(eta))
    errs = weight_errors(got, ref)
    assert max(errs) < 1e-5, errs


@pytest.mark.parametrize("dt", [T.TTT_BF16, T.TTT_FP32])
def test_grad_is_deterministic(dt):
    dtype = torch.bfloat16 if dt == T.TTT_BF16 else torch.float32
    d = 192 if dt == T.TTT_BF16 else 64
    W, K, V, eta = _grad_case(2, d, 128, 1500, dtype, seed=30)
    _, G1 = _run_grad(W, K, V, eta, T.dims(2, d, 128), dt)
    _, G2 = _run_grad(W, K, V, eta, T.dims(2, d, 128), dt)
    assert torch.equal(G1, G2)


@pytest.mark.parametrize("dt,d,m", [(T.TTT_BF16, 192, 256), (T.TTT_FP32, 64, 128), (T.TTT_BF16, 256, 512)])
def test_grad_prepared_equals_grad_after_a_step(dt, d, m):
    # the second inner step of the multi-device update: gradient, step, then the gradient
    # at the new weights from the operands the first call prepared -- the same result
    # as a fresh ttt_grad, bit for bit
    dtype = torch.bfloat16 if dt == T.TTT_BF16 else torch.float32
    H, T_ = 2, 700
    W, K, V, eta = _grad_case(H, d, m, T_, dtype, seed=35)
    dm = T.dims(H, d, m)
    Kd, Vd, ed = K.cuda(), V.cuda(), eta.cuda()
    ws = T.workspace(dm, T_, dt)
    n = H * m * d
    G = torch.empty((3 * n,), dtype=torch.float32, device="cuda")
    T.ttt_grad(W.abi, Kd, Vd, ed, T_, dm, T.io_cfg(), G, ws)
    T.ttt_step(W.abi, G, T.ns_cfg(), dm, dt, ws)
    G2 = torch.full_like(G, float("nan"))
    T.ttt_grad_prepared(W.abi, Kd, Vd, ed, T_, dm, T.io_cfg(), G2, ws)
    G3 = torch.full_like(G, float("nan"))
    T.ttt_grad(W.abi, Kd, Vd, ed, T_, dm, T.io_cfg(), G3, ws)
    check_status(ws)
    assert torch.equal(G2, G3)


# bf16 shapes cover every Newton-Schulz path: one cluster launch with 192 rows and
# 6, 3 or 2 column blocks, with 128 rows and 2 or 1 blocks; per-product launches
# for 192 x 320 (columns not a multiple of 128) and 64 x 128 (64 rows)
@pytest.mark.parametrize("dt,d,m", [(T.TTT_BF16, 192, 768), (T.TTT_BF16, 192, 384), (T.TTT_BF16, 128, 256),
                                    (T.TTT_BF16, 128, 128), (T.TTT_BF16, 192, 256), (T.TTT_BF16, 192, 320),
                                    (T.TTT_BF16, 128, 64),
                                    (T.TTT_FP32, 64, 128), (T.TTT_FP32, 96, 32)])
@pytest.mark.parametrize("iters,renorm,lr", [(5, 1, 1.0), (0, 0, 0.01), (3, 0, 0.5), (1, 1, 1.0)])
def test_step_matches_oracle(dt, d, m, iters, renorm, lr):
    H = 2
    W = DevWeights(*rand_weights(H, d, m, 40))
    Wo = W.oracle()
    dtype = torch.bfloat16 if dt == T.TTT_BF16 else torch.float32
    K = rand_tokens(64, H, d, torch.float32, 41)
    V = rand_tokens(64, H, d, torch.float32, 42)
    G = O.grad(Wo, O.l2norm_heads(f64(K), H, d), f64(V), f64(rand_eta(64, H, 43, 1.0)))
    Gflat = torch.from_numpy(np.concatenate([G.W1.ravel(), G.W3.ravel(), G.W2.ravel()])).float()
    dm = T.dims(H, d, m)
    ws = T.workspace(dm, 0, dt)
    cfg = O.NSConfig(iters=iters, renorm=renorm, lr=lr)
    T.ttt_step(W.abi, Gflat.cuda(), T.ns_cfg(iters=iters, renorm=renorm, lr=lr), dm, dt, ws)
    check_status(ws)
    ref = O.muon_step(Wo, O.FastWeights(*(f64(x) for x in (Gflat[:H * m * d].reshape(H, m, d),
                                                            Gflat[H * m * d:2 * H * m * d].reshape(H, m, d),
                                                            Gflat[2 * H * m * d:].reshape(H, d, m)))), cfg)
    errs = weight_errors(W.oracle(), ref)
    # fp32 mode: fp32 CUDA-core products.  bf16 mode: Newton-Schulz products on
    # the tensor cores from split bf16 operands (hi + lo), ~2^-16 relative each,
    # chained through 5 iterations of 3 products
    assert max(errs) < (1e-5 if dt == T.TTT_FP32 else 1e-4), errs
    del dtype


# the wide-head path's Newton-Schulz: products on 2-SM tensor-core pairs from split
# bf16 operands (three K segments), for r x c = 256 x 512 (tall and wide gradients)
# and ZipMap's 1,024 x 2,048
@pytest.mark.parametrize("H,d,m,iters,renorm,lr", [(2, 256, 512, 5, 1, 1.0), (1, 512, 256, 3, 0, 0.5),
                                                   (1, 1024, 2048, 5, 1, 1.0)])
def test_step_matches_oracle_wide(H, d, m, iters, renorm, lr):
    W = DevWeights(*rand_weights(H, d, m, 44))
    Wo = W.oracle()
    K = rand_tokens(300, H, d, torch.float32, 45)
    V = rand_tokens(300, H, d, torch.float32, 46)
    G = O.grad(Wo, O.l2norm_heads(f64(K), H, d), f64(V), f64(rand_eta(300, H, 47, 1.0)))
    Gflat = torch.from_numpy(np.concatenate([G.W1.ravel(), G.W3.ravel(), G.W2.ravel()])).float()
    dm = T.dims(H, d, m)
    ws = T.workspace(dm, 0, T.TTT_BF16)
    cfg = O.NSConfig(iters=iters, renorm=renorm, lr=lr)
    T.ttt_step(W.abi, Gflat.cuda(), T.ns_cfg(iters=iters, renorm=renorm, lr=lr), dm, T.TTT_BF16, ws)
    check_status(ws)
    n = H * m * d
    ref = O.muon_step(Wo, O.FastWeights(f64(Gflat[:n].reshape(H, m, d)), f64(Gflat[n:2 * n].reshape(H, m, d)),
                                        f64(Gflat[2 * n:].reshape(H, d, m))), cfg)
    errs = weight_errors(W.oracle(), ref)
    assert max(errs) < 1e-4, errs


@pytest.mark.parametrize("H,d,m,N,gh,gw,act", [(2, 192, 256, 3, 5, 7, 0), (2, 128, 128, 2, 9, 4, 1),
                                                (1, 256, 256, 2, 6, 6, 0), (4, 192, 768, 4, 37, 37, 0)])
def test_update_conv_matches_conv_then_update(H, d, m, N, gh, gw, act):
    # ShortConv2D folded into the update's preparation: the same update as ttt_shortconv2d
    # followed by ttt_update (only the rounding of V' differs: once to fp16 instead of
    # bf16 then fp16), and within the layer tolerance of the oracle
    T_ = N * gh * gw
    g = torch.Generator().manual_seed(60 + d)
    K = rand_tokens(T_, H, d, torch.bfloat16, 61)
    V = rand_tokens(T_, H, d, torch.bfloat16, 62)
    eta = rand_eta(T_, H, 63, scale=0.01)
    taps = torch.randn((H * d, 3, 3), generator=g) / 3
    dm = T.dims(H, d, m)
    ns = T.ns_cfg()
    W1 = DevWeights(*rand_weights(H, d, m, 64))
    W2 = DevWeights(*rand_weights(H, d, m, 64))
    W0 = W1.oracle()
    ws = T.workspace(dm, T_, T.TTT_BF16)
    Kd, Vd, ed, td = K.cuda(), V.cuda(), eta.cuda(), taps.cuda()
    T.ttt_update_conv(W1.abi, Kd, Vd, ed, T_, 2, ns, td, gh, gw, dm, T.io_cfg(), ws, act=act)
    check_status(ws)
    Vc = torch.empty_like(Vd)
    T.ttt_shortconv2d(Vd, Vc, td, N, gh, gw, H * d, act)
    T.ttt_update(W2.abi, Kd, Vc, ed, T_, 2, ns, dm, T.io_cfg(), ws)
    check_status(ws)
    assert max(weight_errors(W1.oracle(), W2.oracle())) < 1e-2
    ref = O.update(W0, f64(K), f64(V), f64(eta), 2, O.NSConfig(), conv=(taps.double().numpy(), N, gh, gw, act))
    errs = weight_errors(W1.oracle(), ref)
    assert max(errs) < TOL_BF16, errs


def test_update_eta_zero_keeps_weights_bf16():
    H, d, m, T_ = 2, 192, 128, 500
    W = DevWeights(*rand_weights(H, d, m, 50))
    before = W.oracle()
    K = rand_tokens(T_, H, d, torch.bfloat16, 51).cuda()
    V = rand_tokens(T_, H, d, torch.bfloat16, 52).cuda()
    eta = torch.zeros((T_, H), dtype=torch.float32, device="cuda")
    dm = T.dims(H, d, m)
    ws = T.workspace(dm, T_, T.TTT_BF16)
    T.ttt_update(W.abi, K, V, eta, T_, 1, T.ns_cfg(), dm, T.io_cfg(), ws)
    check_status(ws)
    assert max(weight_errors(W.oracle(), before)) < 1e-6


def test_device_wait_timeout_is_reported_and_context_survives():
    # a wait on a barrier nothing signals gives up after its limit, records the
    # timeout in the status word and returns; the context keeps working afterwards
    dm = T.dims(1, 128, 64)
    ws = T.workspace(dm, 256, T.TTT_BF16)
    T.ttt_reset_status(ws)
    assert T.ttt_poll_status(ws) == T.TTT_OK
    T.ttt_selftest_wait_timeout(ws, 50_000)
    assert T.ttt_poll_status(ws) == T.TTT_ERR_TIMEOUT
    T.ttt_reset_status(ws)
    assert T.ttt_poll_status(ws) == T.TTT_OK
    W = DevWeights(*rand_weights(1, 128, 64, 60))
    Q = rand_tokens(256, 1, 128, torch.bfloat16, 61).cuda()
    O_ = torch.zeros_like(Q)
    T.ttt_apply(W.abi, Q, O_, 256, dm, T.io_cfg(), ws)
    check_status(ws)
    assert rel_fro(f64(O_), O.apply(W.oracle(), f64(Q))) < 1e-2


def test_kernels_run_as_sm100a_binaries():
    v = ctypes.c_int(0)
    assert T.lib().ttt_kernel_binary_version(ctypes.byref(v)) == T.TTT_OK
    assert v.value == 100
