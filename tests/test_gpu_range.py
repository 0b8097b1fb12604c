"""The fp16 operands of the tensor-core update: wide ranges of eta and of the
token values, raw (not normalised) keys and queries, and inputs beyond fp16's
range, which must be reported rather than written into the fast weights.

The preparation pass writes the fp16 operands k^ (normalised per row when the
L2 norm is on) and V' = -s eta v for a power of two s chosen per call from
max|eta| (so the scale of eta does not matter).  A value that still overflows
fp16 makes the gradient non-finite: ttt_poll_status then returns
TTT_ERR_RANGE and the weight step is skipped."""
import numpy as np
import pytest
import torch

import oracle as O
from test_weight_layers_b200 import ttt as T

from _gpu import TOL_BF16, DevWeights, f64, need_gpu, rand_eta, rand_tokens, rand_weights, weight_errors, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _update(W, K, V, eta, dm, qk=1, steps=1):
    T_ = K.shape[0]
    ws = T.workspace(dm, T_, T.TTT_BF16)
    T.ttt_update(W.abi, K.cuda(), V.cuda(), eta.cuda(), T_, steps, T.ns_cfg(), dm, T.io_cfg(qk_l2norm=qk), ws)
    return T.ttt_poll_status(ws)


def _oracle_update(W0, K, V, eta, H, d, qk=1, steps=1):
    return O.update(W0, f64(K), f64(V), f64(eta), steps, O.NSConfig(), qk_l2norm=bool(qk))


@pytest.mark.parametrize("eta_scale,k_scale,v_scale", [
    (1e3, 1.0, 1.0),        # eta = 10^3 softplus(N(0,1)): V' would overflow with a fixed scale
    (1e-7, 1.0, 1.0),       # tiny eta: without the per-call scale V' falls into fp16 subnormals
    (0.01, 1e-5, 1e-4),     # small keys and values (raw keys partly in fp16's subnormal range)
    (0.01, 30.0, 20.0),     # large keys and values
    (0.01, 3e5, 1.0),       # keys beyond fp16's range: normalised before the conversion
])
def test_update_over_wide_input_ranges(eta_scale, k_scale, v_scale):
    H, d, m, T_ = 2, 192, 256, 700
    W = DevWeights(*rand_weights(H, d, m, 400))
    W0 = W.oracle()
    K = rand_tokens(T_, H, d, torch.bfloat16, 401, scale=k_scale)
    V = rand_tokens(T_, H, d, torch.bfloat16, 402, scale=v_scale)
    eta = rand_eta(T_, H, 403, scale=eta_scale)
    assert _update(W, K, V, eta, T.dims(H, d, m)) == T.TTT_OK
    ref = _oracle_update(W0, K, V, eta, H, d)
    errs = weight_errors(W.oracle(), ref)
    assert max(errs) < TOL_BF16, errs


def test_grad_without_key_norm_bf16():
    # qk_l2norm = 0 on the tensor cores: raw keys with |k| up to ~10^2
    H, d, m, T_ = 2, 192, 128, 517
    W = DevWeights(*rand_weights(H, d, m, 410))
    K = rand_tokens(T_, H, d, torch.bfloat16, 411, scale=25.0)
    V = rand_tokens(T_, H, d, torch.bfloat16, 412)
    eta = rand_eta(T_, H, 413, scale=1.0)
    dm = T.dims(H, d, m)
    ws = T.workspace(dm, T_, T.TTT_BF16)
    n = H * m * d
    G = torch.full((3 * n,), float("nan"), dtype=torch.float32, device="cuda")
    T.ttt_grad(W.abi, K.cuda(), V.cuda(), eta.cuda(), T_, dm, T.io_cfg(qk_l2norm=0), G, ws)
    assert T.ttt_poll_status(ws) == T.TTT_OK
    g = f64(G)
    got = O.FastWeights(g[:n].reshape(H, m, d), g[n:2 * n].reshape(H, m, d), g[2 * n:].reshape(H, d, m))
    ref = O.grad(W.oracle(), f64(K), f64(V), f64(eta))
    errs = weight_errors(got, ref)
    assert max(errs) < 2e-2, errs


def test_update_without_key_norm_bf16():
    H, d, m, T_ = 2, 128, 192, 300
    W = DevWeights(*rand_weights(H, d, m, 420))
    W0 = W.oracle()
    K = rand_tokens(T_, H, d, torch.bfloat16, 421, scale=4.0)
    V = rand_tokens(T_, H, d, torch.bfloat16, 422)
    eta = rand_eta(T_, H, 423)
    assert _update(W, K, V, eta, T.dims(H, d, m), qk=0, steps=2) == T.TTT_OK
    ref = _oracle_update(W0, K, V, eta, H, d, qk=0, steps=2)
    assert max(weight_errors(W.oracle(), ref)) < TOL_BF16


def test_apply_without_query_norm_bf16():
    H, d, m, T_ = 2, 192, 256, 333
    W = DevWeights(*rand_weights(H, d, m, 430))
    Q = rand_tokens(T_, H, d, torch.bfloat16, 431, scale=25.0)
    dm = T.dims(H, d, m)
    ws = T.workspace(dm, T_, T.TTT_BF16)
    O_ = torch.full((T_, H * d), float("nan"), dtype=torch.bfloat16, device="cuda")
    T.ttt_apply(W.abi, Q.cuda(), O_, T_, dm, T.io_cfg(qk_l2norm=0), ws)
    assert T.ttt_poll_status(ws) == T.TTT_OK
    ref = O.apply(W.oracle(), f64(Q), qk_l2norm=False)
    assert rel_fro(f64(O_), ref) < 1e-2


@pytest.mark.parametrize("what", ["values", "keys"])
def test_out_of_range_operand_is_reported_and_weights_kept(what):
    # |v| ~ 10^5 overflows V' = -s eta v (s max|eta| >= 16); without the key norm a
    # key element of 10^5 overflows the fp16 key operand
    H, d, m, T_ = 2, 192, 128, 260
    W = DevWeights(*rand_weights(H, d, m, 440))
    before = [w.clone() for w in (W.W1, W.W3, W.W2)]
    K = rand_tokens(T_, H, d, torch.bfloat16, 441)
    V = rand_tokens(T_, H, d, torch.bfloat16, 442)
    if what == "values":
        V[:, :] = (V.float() * 1e5).to(torch.bfloat16)
    else:
        K[7, 3] = 1e5
    eta = rand_eta(T_, H, 443)
    qk = 1 if what == "values" else 0
    assert _update(W, K, V, eta, T.dims(H, d, m), qk=qk, steps=2) == T.TTT_ERR_RANGE
    for a, b in zip((W.W1, W.W3, W.W2), before):
        assert torch.equal(a, b)
