"""GPU parity of the wide-head path (d and m multiples of 256; ZipMap's own
single head of d = 1024, m = 2048) and of the gated output
o = RMSNorm(o') SiLU(W_g o'), against the fp64 oracle, through the C ABI.

Small token counts span several 256-token tiles and a ragged tail; the
zipmap1024 recipe runs on a few frames here and at its full 1,030,500 tokens
in test_wide_full_size_sampled (gradient rows and output rows the oracle
computes one by one)."""
import numpy as np
import pytest
import torch

import oracle as O
from test_weight_layers_b200 import synth as S
from test_weight_layers_b200 import ttt as T

from _gpu import TOL_BF16, DevWeights, check_status, f64, need_gpu, rand_eta, rand_tokens, rand_weights, rel_fro, \
    weight_errors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _grad(W, K, V, eta, dm, qk=1):
    T_ = K.shape[0]
    ws = T.workspace(dm, T_, T.TTT_BF16)
    H, d, m = dm.heads, dm.d, dm.m
    n = H * m * d
    G = torch.full((3 * n,), float("nan"), dtype=torch.float32, device="cuda")
    T.ttt_grad(W.abi, K.cuda(), V.cuda(), eta.cuda(), T_, dm, T.io_cfg(qk_l2norm=qk), G, ws)
    check_status(ws)
    g = f64(G)
    return O.FastWeights(g[:n].reshape(H, m, d), g[n:2 * n].reshape(H, m, d), g[2 * n:].reshape(H, d, m))


@pytest.mark.parametrize("H,d,m,T_,qk", [(1, 256, 512, 700, 1), (2, 256, 256, 300, 1), (1, 512, 256, 129, 0),
                                         (1, 1024, 2048, 513, 1)])
def test_wide_grad(H, d, m, T_, qk):
    W = DevWeights(*rand_weights(H, d, m, 500 + d))
    K = rand_tokens(T_, H, d, torch.bfloat16, 501, scale=1.0 if qk else 0.3)
    V = rand_tokens(T_, H, d, torch.bfloat16, 502)
    eta = rand_eta(T_, H, 503, scale=1.0)
    got = _grad(W, K, V, eta, T.dims(H, d, m), qk)
    Kr = O.l2norm_heads(f64(K), H, d) if qk else f64(K)
    ref = O.grad(W.oracle(), Kr, f64(V), f64(eta))
    errs = weight_errors(got, ref)
    assert max(errs) < 2e-2, errs


@pytest.mark.parametrize("H,d,m,T_", [(1, 256, 512, 600), (2, 512, 256, 257), (1, 1024, 2048, 300)])
def test_wide_apply(H, d, m, T_):
    W = DevWeights(*rand_weights(H, d, m, 510 + d))
    Q = rand_tokens(T_, H, d, torch.bfloat16, 511, ld=H * d + 64)
    dm = T.dims(H, d, m)
    ws = T.workspace(dm, T_, T.TTT_BF16)
    O_ = torch.full((T_, H * d + 32), float("nan"), dtype=torch.bfloat16, device="cuda")
    T.ttt_apply(W.abi, Q.cuda(), O_, T_, dm, T.io_cfg(ld_q=H * d + 64, ld_o=H * d + 32), ws)
    check_status(ws)
    ref = O.apply(W.oracle(), f64(Q)[:, :H * d])
    assert rel_fro(f64(O_)[:, :H * d], ref) < 1e-2
    assert torch.isnan(O_[:, H * d:].float()).all()  # columns past H*d untouched


@pytest.mark.parametrize("D,T_", [(1024, 700), (768, 300), (256, 1)])
def test_output_gate(D, T_):
    g = torch.Generator().manual_seed(520 + D)
    Op = (torch.randn((T_, D), generator=g) * 0.7).to(torch.bfloat16)
    Wg = torch.randn((D, D), generator=g) / D ** 0.5
    ws = T.gate_workspace(T_, D)
    Out = torch.full((T_, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    T.ttt_output_gate(Op.cuda(), Wg.cuda(), Out, T_, D, ws)
    torch.cuda.synchronize()
    ref = O.output_gate(f64(Op), Wg.double().numpy())
    assert rel_fro(f64(Out), ref) < 1e-2


def _layer(cfg):
    inp = S.Inputs(cfg)
    W = DevWeights(*inp.weights())
    K, V, Q, eta = inp.k(), inp.v(), inp.q(), inp.eta()
    Wg = inp.gate_weight()
    Tn = cfg.tokens
    dm = T.dims(cfg.heads, cfg.d, cfg.m)
    ws = T.workspace(dm, Tn, T.TTT_BF16)
    gws = T.gate_workspace(Tn, cfg.model_dim)
    ns = T.ns_cfg(cfg.ns_iters, cfg.ns_a, cfg.ns_b, cfg.ns_c, cfg.ns_eps, cfg.lr, cfg.renorm)
    Op = torch.zeros((Tn, cfg.model_dim), dtype=torch.bfloat16, device="cuda")
    Od = torch.zeros_like(Op)
    T.ttt_update(W.abi, K.cuda(), V.cuda(), eta.cuda(), Tn, cfg.steps, ns, dm, T.io_cfg(), ws)
    T.ttt_apply(W.abi, Q.cuda(), Op, Tn, dm, T.io_cfg(), ws)
    T.ttt_output_gate(Op, Wg.cuda(), Od, Tn, cfg.model_dim, gws)
    check_status(ws)
    return W, Op, Od, (inp, K, V, Q, eta, Wg)


def test_zipmap1024_layer_small():
    cfg = S.WORKLOADS["zipmap1024"].with_frames(2)
    W, Op, Od, (inp, K, V, Q, eta, Wg) = _layer(cfg)
    W0 = O.FastWeights.of(*(w.numpy() for w in inp.weights()))
    nsc = O.NSConfig(cfg.ns_iters, cfg.ns_a, cfg.ns_b, cfg.ns_c, cfg.ns_eps, cfg.lr, cfg.renorm)
    Wr = O.update(W0, f64(K), f64(V), f64(eta), cfg.steps, nsc)
    errs = weight_errors(W.oracle(), Wr)
    assert max(errs) < TOL_BF16, errs
    Opr = O.apply(Wr, f64(Q))
    assert rel_fro(f64(Op), Opr) < TOL_BF16
    assert rel_fro(f64(Od), O.output_gate(Opr, Wg.double().numpy())) < TOL_BF16


@pytest.mark.slow
def test_wide_full_size_sampled():
    # zipmap1024 at its full 1,030,500 tokens: sampled rows of g1, g3 and columns of g2
    # (each needs one weight row, so the oracle computes them for any token count),
    # then the layer and sampled rows of its gated output against the GPU's own
    # updated weights (the apply and the gate are row-independent)
    cfg = S.WORKLOADS["zipmap1024"]
    inp = S.Inputs(cfg)
    K, V, Q, eta = inp.k(), inp.v(), inp.q(), inp.eta()
    Tn, H, d, m = cfg.tokens, cfg.heads, cfg.d, cfg.m
    dm = T.dims(H, d, m)
    W = DevWeights(*inp.weights())
    W0 = W.oracle()
    ws = T.workspace(dm, Tn, T.TTT_BF16)
    n = H * m * d
    G = torch.empty((3 * n,), dtype=torch.float32, device="cuda")
    Kd, Vd, ed = K.cuda(), V.cuda(), eta.cuda()
    T.ttt_grad(W.abi, Kd, Vd, ed, Tn, dm, T.io_cfg(), G, ws)
    check_status(ws)
    g = f64(G)
    rows = [(0, j) for j in np.random.default_rng(530).choice(m, size=6, replace=False)]

    def blocks():
        for b0 in range(0, Tn, 1 << 15):
            b1 = min(Tn, b0 + (1 << 15))
            yield O.l2norm_heads(f64(K[b0:b1]), H, d), f64(V[b0:b1]), f64(eta[b0:b1])
    ref = O.grad_rows(W0, blocks(), rows)
    for (h, j) in rows:
        got1 = g[:n].reshape(H, m, d)[h, j]
        got3 = g[n:2 * n].reshape(H, m, d)[h, j]
        got2 = g[2 * n:].reshape(H, d, m)[h, :, j]
        for got, want in ((got1, ref[(h, j)][0]), (got3, ref[(h, j)][1]), (got2, ref[(h, j)][2])):
            assert rel_fro(got, want) < 2e-2, (h, j)
    # the whole layer, in the configuration the bench times
    Wg = inp.gate_weight()
    gws = T.gate_workspace(Tn, cfg.model_dim)
    Op = torch.empty((Tn, cfg.model_dim), dtype=torch.bfloat16, device="cuda")
    Od = torch.empty_like(Op)
    ns = T.ns_cfg(cfg.ns_iters, cfg.ns_a, cfg.ns_b, cfg.ns_c, cfg.ns_eps, cfg.lr, cfg.renorm)
    Qd = Q.cuda()
    T.ttt_update(W.abi, Kd, Vd, ed, Tn, cfg.steps, ns, dm, T.io_cfg(), ws)
    T.ttt_apply(W.abi, Qd, Op, Tn, dm, T.io_cfg(), ws)
    T.ttt_output_gate(Op, Wg.cuda(), Od, Tn, cfg.model_dim, gws)
    check_status(ws)
    sample = np.sort(np.random.default_rng(531).choice(Tn, size=2048, replace=False))
    Wn = W.oracle()
    Opr = O.apply(Wn, f64(Q[sample]))
    assert rel_fro(f64(Op)[sample], Opr) < 1e-2
    assert rel_fro(f64(Od)[sample], O.output_gate(Opr, Wg.double().numpy())) < 1e-2
