"""End-to-end GPU parity on the six workloads' recipes (update + apply through
the C ABI, compared with the fp64 oracle on the same seeded inputs).

The tiny (fp32) and object-scale workloads run at their full sizes; the three
large workloads run with the same heads/dims/recipe on fewer frames so the
oracle finishes in seconds (their full sizes are covered by test_gpu_fullsize)."""
import numpy as np
import pytest
import torch

import oracle as O
from test_weight_layers_b200 import synth as S
from test_weight_layers_b200 import ttt as T

from _gpu import TOL_BF16, TOL_FP32, DevWeights, check_status, f64, need_gpu, rel_fro, weight_errors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def ns_of(cfg):
    return O.NSConfig(cfg.ns_iters, cfg.ns_a, cfg.ns_b, cfg.ns_c, cfg.ns_eps, cfg.lr, cfg.renorm)


def abi_ns(cfg):
    return T.ns_cfg(cfg.ns_iters, cfg.ns_a, cfg.ns_b, cfg.ns_c, cfg.ns_eps, cfg.lr, cfg.renorm)


def run_layer(cfg):
    """GPU: [ShortConv2D] + update + apply (or chunked), returning (W_final, O, inputs)."""
    inp = S.Inputs(cfg)
    W = DevWeights(*inp.weights())
    K, V, Q, eta = inp.k(), inp.v(), inp.q(), inp.eta()
    Tn, Ta = cfg.tokens, cfg.apply_tokens
    dm = T.dims(cfg.heads, cfg.d, cfg.m)
    dt = T.dtype_code(cfg.torch_dtype)
    ws = T.workspace(dm, cfg.chunk or max(Tn, Ta), dt)
    Kd, Vd, Qd, ed = K.cuda(), V.cuda(), Q.cuda(), eta.cuda()
    Od = torch.zeros((Ta, cfg.model_dim), dtype=cfg.torch_dtype, device="cuda")
    if cfg.conv:
        Vc = torch.empty_like(Vd)
        T.ttt_shortconv2d(Vd, Vc, inp.taps().cuda(), cfg.frames, cfg.grid_h, cfg.grid_w, cfg.model_dim)
        Vd = Vc
    if cfg.chunk:
        T.ttt_chunked(W.abi, Qd, Kd, Vd, ed, Od, Tn, cfg.chunk, cfg.order, cfg.steps, abi_ns(cfg), dm, T.io_cfg(),
                      ws)
    else:
        T.ttt_update(W.abi, Kd, Vd, ed, Tn, cfg.steps, abi_ns(cfg), dm, T.io_cfg(), ws)
        T.ttt_apply(W.abi, Qd, Od, Ta, dm, T.io_cfg(), ws)
    check_status(ws)
    return W.oracle(), f64(Od), (inp, K, V, Q, eta)


def oracle_layer(cfg, inp, K, V, Q, eta):
    W0 = O.FastWeights.of(*(w.numpy() for w in inp.weights()))
    conv = (inp.taps().double().numpy(), cfg.frames, cfg.grid_h, cfg.grid_w, 0) if cfg.conv else None
    if cfg.chunk:
        return O.chunked(W0, f64(Q), f64(K), f64(V), f64(eta), cfg.chunk, cfg.steps, ns_of(cfg), order=cfg.order)
    Wf = O.update(W0, f64(K), f64(V), f64(eta), cfg.steps, ns_of(cfg), conv=conv)
    return Wf, O.apply(Wf, f64(Q))


CASES = {
    "tiny": S.WORKLOADS["tiny"],
    "object": S.WORKLOADS["object"],
    "zipmap-12f": S.WORKLOADS["zipmap"].with_frames(12),
    "vggt3-4f": S.WORKLOADS["vggt3"].with_frames(4),
    "loger-16f": S.WORKLOADS["loger"].with_frames(16, chunk=4096),
    "stream-6f": S.WORKLOADS["stream"].with_frames(6),
}


@pytest.mark.parametrize("name", list(CASES))
def test_workload_parity(name):
    cfg = CASES[name]
    Wg, Og, data = run_layer(cfg)
    Wr, Or = oracle_layer(cfg, *data)
    tol = TOL_FP32 if cfg.dtype == "fp32" else TOL_BF16
    errs = weight_errors(Wg, Wr)
    assert max(errs) < tol, (name, errs)
    eo = rel_fro(Og, Or)
    assert eo < tol, (name, eo)
    # the update must have moved W measurably (the comparison is not vacuous)
    W0 = data[0].weights()
    moved = rel_fro(Wr.W1, W0[0].double().numpy())
    assert moved > 10 * max(errs[: cfg.heads]), (moved, errs)


def test_chunk_equal_to_sequence_is_one_update():
    cfg = S.WORKLOADS["loger"].with_frames(4, chunk=4096)
    inp = S.Inputs(cfg)
    dm, dt = T.dims(cfg.heads, cfg.d, cfg.m), T.TTT_BF16
    K, V, Q, eta = (x.cuda() for x in (inp.k(), inp.v(), inp.q(), inp.eta()))
    Tn = cfg.tokens
    ws = T.workspace(dm, Tn, dt)
    Wa = DevWeights(*inp.weights())
    Oa = torch.zeros((Tn, cfg.model_dim), dtype=torch.bfloat16, device="cuda")
    T.ttt_chunked(Wa.abi, Q, K, V, eta, Oa, Tn, Tn, 0, 1, abi_ns(cfg), dm, T.io_cfg(), ws)
    Wb = DevWeights(*inp.weights())
    Ob = torch.zeros_like(Oa)
    T.ttt_apply(Wb.abi, Q, Ob, Tn, dm, T.io_cfg(), ws)
    T.ttt_update(Wb.abi, K, V, eta, Tn, 1, abi_ns(cfg), dm, T.io_cfg(), ws)
    check_status(ws)
    assert torch.equal(Wa.W1, Wb.W1) and torch.equal(Wa.W2, Wb.W2) and torch.equal(Oa, Ob)


def test_chunked_resume_is_bitwise():
    cfg = S.WORKLOADS["loger"].with_frames(12, chunk=4096)
    inp = S.Inputs(cfg)
    dm, dt = T.dims(cfg.heads, cfg.d, cfg.m), T.TTT_BF16
    K, V, Q, eta = (x.cuda() for x in (inp.k(), inp.v(), inp.q(), inp.eta()))
    Tn = cfg.tokens
    ws = T.workspace(dm, 4096, dt)
    Wa = DevWeights(*inp.weights())
    Oa = torch.zeros((Tn, cfg.model_dim), dtype=torch.bfloat16, device="cuda")
    T.ttt_chunked(Wa.abi, Q, K, V, eta, Oa, Tn, 4096, 0, 1, abi_ns(cfg), dm, T.io_cfg(), ws)
    Wb = DevWeights(*inp.weights())
    Ob = torch.zeros_like(Oa)
    half = 2 * 4096
    T.ttt_chunked(Wb.abi, Q[:half], K[:half], V[:half], eta[:half], Ob[:half], half, 4096, 0, 1, abi_ns(cfg), dm,
                  T.io_cfg(), ws)
    T.ttt_chunked(Wb.abi, Q[half:], K[half:], V[half:], eta[half:], Ob[half:], Tn - half, 4096, 0, 1, abi_ns(cfg), dm,
                  T.io_cfg(), ws)
    check_status(ws)
    assert torch.equal(Wa.W2, Wb.W2) and torch.equal(Oa, Ob)


def test_two_steps_equal_grad_step_twice():
    cfg = S.WORKLOADS["vggt3"].with_frames(2)
    inp = S.Inputs(cfg)
    dm, dt = T.dims(cfg.heads, cfg.d, cfg.m), T.TTT_BF16
    K, V, eta = (x.cuda() for x in (inp.k(), inp.v(), inp.eta()))
    Tn = cfg.tokens
    ws = T.workspace(dm, Tn, dt)
    Wa = DevWeights(*inp.weights())
    T.ttt_update(Wa.abi, K, V, eta, Tn, 2, abi_ns(cfg), dm, T.io_cfg(), ws)
    Wb = DevWeights(*inp.weights())
    G = torch.empty(3 * cfg.heads * cfg.m * cfg.d, dtype=torch.float32, device="cuda")
    for _ in range(2):
        T.ttt_grad(Wb.abi, K, V, eta, Tn, dm, T.io_cfg(), G, ws)
        T.ttt_step(Wb.abi, G, abi_ns(cfg), dm, dt, ws)
    check_status(ws)
    assert torch.equal(Wa.W1, Wb.W1) and torch.equal(Wa.W3, Wb.W3) and torch.equal(Wa.W2, Wb.W2)


def test_empty_inputs_are_no_ops():
    dm = T.dims(2, 192, 128)
    ws = T.workspace(dm, 1, T.TTT_BF16)
    W = DevWeights(*(torch.ones(s) for s in ((2, 128, 192), (2, 128, 192), (2, 192, 128))))
    x = torch.zeros((1, 384), dtype=torch.bfloat16, device="cuda")
    e = torch.zeros((1, 2), device="cuda")
    T.ttt_update(W.abi, x, x, e, 0, 1, T.ns_cfg(), dm, T.io_cfg(), ws)
    T.ttt_apply(W.abi, x, x.clone(), 0, dm, T.io_cfg(), ws)
    G = torch.full((3 * 2 * 128 * 192,), 7.0, device="cuda")
    T.ttt_grad(W.abi, x, x, e, 0, dm, T.io_cfg(), G, ws)
    check_status(ws)
    assert torch.all(W.W1 == 1) and torch.all(G == 0)
