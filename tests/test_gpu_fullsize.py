"""GPU parity at the three large workloads' full sizes, in the launch
configuration the bench times (ttt_update + ttt_apply, or ttt_chunked, through
the C ABI on the full token count).

The oracle computes the full update itself, streamed over token blocks (the
loss is a sum over tokens, so the gradient is the sum of block gradients), in
fp64; the fast weights are compared in full and the outputs on a seeded sample
of rows (apply is row-independent).  Minutes of host time per workload."""
import numpy as np
import pytest
import torch

import oracle as O
from test_weight_layers_b200 import synth as S
from test_weight_layers_b200 import ttt as T

from _gpu import TOL_BF16, DevWeights, check_status, f64, need_gpu, rel_fro, weight_errors

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

BLOCK = 1 << 15


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def ns_of(cfg):
    return O.NSConfig(cfg.ns_iters, cfg.ns_a, cfg.ns_b, cfg.ns_c, cfg.ns_eps, cfg.lr, cfg.renorm)


def abi_ns(cfg):
    return T.ns_cfg(cfg.ns_iters, cfg.ns_a, cfg.ns_b, cfg.ns_c, cfg.ns_eps, cfg.lr, cfg.renorm)


def oracle_grad_blocks(W, K, V, eta, t0, t1, cfg, taps=None):
    """Oracle gradient over tokens [t0, t1), in blocks of whole frames when a conv is used."""
    H, d = cfg.heads, cfg.d
    G = O.zeros_like(W)
    fr = cfg.grid_h * cfg.grid_w
    step = (BLOCK // fr) * fr if taps is not None else BLOCK
    for b0 in range(t0, t1, step):
        b1 = min(t1, b0 + step)
        Kb = O.l2norm_heads(f64(K[b0:b1]), H, d)
        if taps is not None:
            Vb = O.shortconv2d(f64(V[b0:b1]), taps, (b1 - b0) // fr, cfg.grid_h, cfg.grid_w)
        else:
            Vb = f64(V[b0:b1])
        G = O.add(G, O.grad(W, Kb, Vb, f64(eta[b0:b1])))
    return G


def sample_rows(n, k, seed):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(n, size=min(k, n), replace=False))


@pytest.mark.parametrize("name", ["zipmap", "vggt3"])
def test_full_bidirectional_layer(name):
    cfg = S.WORKLOADS[name]
    inp = S.Inputs(cfg)
    K, V, Q, eta = inp.k(), inp.v(), inp.q(), inp.eta()
    Tn = cfg.tokens
    dm = T.dims(cfg.heads, cfg.d, cfg.m)
    W = DevWeights(*inp.weights())
    ws = T.workspace(dm, Tn, T.TTT_BF16)
    Kd, Vd, Qd, ed = K.cuda(), V.cuda(), Q.cuda(), eta.cuda()
    taps = inp.taps() if cfg.conv else None
    if cfg.conv:
        Vc = torch.empty_like(Vd)
        T.ttt_shortconv2d(Vd, Vc, taps.cuda(), cfg.frames, cfg.grid_h, cfg.grid_w, cfg.model_dim)
        Vd = Vc
    Od = torch.zeros_like(Qd)
    T.ttt_update(W.abi, Kd, Vd, ed, Tn, cfg.steps, abi_ns(cfg), dm, T.io_cfg(), ws)
    T.ttt_apply(W.abi, Qd, Od, Tn, dm, T.io_cfg(), ws)
    check_status(ws)
    del Kd, Vd, Qd, ed
    # oracle: the full update, then apply on sampled rows
    Wr = O.FastWeights.of(*(w.numpy() for w in inp.weights()))
    tp = taps.double().numpy() if taps is not None else None
    for _ in range(cfg.steps):
        Wr = O.muon_step(Wr, oracle_grad_blocks(Wr, K, V, eta, 0, Tn, cfg, tp), ns_of(cfg))
    errs = weight_errors(W.oracle(), Wr)
    assert max(errs) < TOL_BF16, errs
    rows = sample_rows(Tn, 4096, 5)
    Og = f64(Od)[rows]
    Or = O.apply(Wr, f64(Q[rows]))
    assert rel_fro(Og, Or) < TOL_BF16


def test_full_causal_chunked_layer():
    cfg = S.WORKLOADS["loger"]
    inp = S.Inputs(cfg)
    K, V, Q, eta = inp.k(), inp.v(), inp.q(), inp.eta()
    Tn, ch = cfg.tokens, cfg.chunk
    dm = T.dims(cfg.heads, cfg.d, cfg.m)
    W = DevWeights(*inp.weights())
    ws = T.workspace(dm, ch, T.TTT_BF16)
    Kd, Vd, Qd, ed = K.cuda(), V.cuda(), Q.cuda(), eta.cuda()
    Od = torch.zeros_like(Qd)
    T.ttt_chunked(W.abi, Qd, Kd, Vd, ed, Od, Tn, ch, 0, cfg.steps, abi_ns(cfg), dm, T.io_cfg(), ws)
    check_status(ws)
    Og_all = f64(Od)
    del Kd, Vd, Qd, ed
    Wr = O.FastWeights.of(*(w.numpy() for w in inp.weights()))
    errs_o = []
    for c, c0 in enumerate(range(0, Tn, ch)):
        c1 = min(Tn, c0 + ch)
        rows = c0 + sample_rows(c1 - c0, 512, 100 + c)
        errs_o.append(rel_fro(Og_all[rows], O.apply(Wr, f64(Q[rows]))))
        Wr = O.muon_step(Wr, oracle_grad_blocks(Wr, K, V, eta, c0, c1, cfg), ns_of(cfg))
    errs = weight_errors(W.oracle(), Wr)
    assert max(errs) < TOL_BF16, errs
    assert max(errs_o) < TOL_BF16, errs_o
