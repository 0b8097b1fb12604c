"""ttt_layer_host: the whole layer over host-resident tokens with the copies
overlapped with the computation.  Parity with the fp64 oracle on the workloads'
recipes, and agreement with the device-memory entry points: bitwise in chunk
mode (same kernels in the same order), up to the order of the block-gradient
sum in bidirectional mode."""
import pytest
import torch

from test_weight_layers_b200 import synth as S
from test_weight_layers_b200 import ttt as T

from _gpu import TOL_BF16, TOL_FP32, DevWeights, check_status, f64, need_gpu, rel_fro, weight_errors
from test_gpu_workloads import CASES, abi_ns, oracle_layer, run_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def run_host(cfg, pinned=True):
    inp = S.Inputs(cfg)
    W = DevWeights(*inp.weights())
    K, V, Q, eta = inp.k(), inp.v(), inp.q(), inp.eta()
    Tn = cfg.tokens
    assert cfg.apply_tokens == Tn
    dm = T.dims(cfg.heads, cfg.d, cfg.m)
    dt = T.dtype_code(cfg.torch_dtype)

    def host(x):
        return x.contiguous().pin_memory() if pinned else x.contiguous().clone()

    hK, hV, hQ, he = host(K), host(V), host(Q), host(eta)
    hO = host(torch.full((Tn, cfg.model_dim), float("nan"), dtype=cfg.torch_dtype))
    ws = T.workspace(dm, cfg.chunk or Tn, dt)
    dbuf = T.host_buffer(dm, Tn, dt, conv=cfg.conv)
    taps = inp.taps().cuda() if cfg.conv else None
    T.ttt_layer_host(W.abi, hQ, hK, hV, he, hO, Tn, cfg.chunk, cfg.order, cfg.steps, abi_ns(cfg), dm, T.io_cfg(),
                     dbuf, ws,
                     taps=taps, grid_h=cfg.grid_h if cfg.conv else 0, grid_w=cfg.grid_w if cfg.conv else 0)
    check_status(ws)  # synchronises the stream: hO is complete
    return W, hO, (inp, K, V, Q, eta)


@pytest.mark.parametrize("name", list(CASES))
def test_host_layer_matches_oracle_and_device_path(name):
    cfg = CASES[name]
    Wh, Oh, data = run_host(cfg)
    Wr, Or = oracle_layer(cfg, *data)
    tol = TOL_FP32 if cfg.dtype == "fp32" else TOL_BF16
    errs = weight_errors(Wh.oracle(), Wr)
    assert max(errs) < tol, (name, errs)
    assert rel_fro(f64(Oh), Or) < tol
    Wd, Od, _ = run_layer(cfg)
    if cfg.chunk:
        # chunk mode queues the same kernels in the same order as ttt_chunked
        assert max(weight_errors(Wh.oracle(), Wd)) == 0.0
        assert rel_fro(f64(Oh), Od) == 0.0
    else:
        # block-wise gradient: same terms, summed block by block
        assert max(weight_errors(Wh.oracle(), Wd)) < 1e-3
        assert rel_fro(f64(Oh), Od) < 5e-3


def test_host_layer_pageable_memory_and_repeat():
    cfg = S.WORKLOADS["zipmap"].with_frames(3)
    W1, O1, _ = run_host(cfg, pinned=False)
    W2, O2, _ = run_host(cfg, pinned=True)
    # the same queue of kernels whatever the host memory: bitwise equal
    assert torch.equal(W1.W1, W2.W1) and torch.equal(W1.W2, W2.W2) and torch.equal(O1, O2)


def test_host_layer_without_update_is_apply():
    cfg = S.WORKLOADS["zipmap"].with_frames(2)
    inp = S.Inputs(cfg)
    Tn, dm = cfg.tokens, T.dims(cfg.heads, cfg.d, cfg.m)
    Wa = DevWeights(*inp.weights())
    hQ, hK, hV, he = (x.contiguous().pin_memory() for x in (inp.q(), inp.k(), inp.v(), inp.eta()))
    hO = torch.empty((Tn, cfg.model_dim), dtype=torch.bfloat16).pin_memory()
    ws = T.workspace(dm, Tn, T.TTT_BF16)
    dbuf = T.host_buffer(dm, Tn, T.TTT_BF16)
    T.ttt_layer_host(Wa.abi, hQ, hK, hV, he, hO, Tn, 0, 0, 0, abi_ns(cfg), dm, T.io_cfg(), dbuf, ws)
    Od = torch.empty((Tn, cfg.model_dim), dtype=torch.bfloat16, device="cuda")
    T.ttt_apply(Wa.abi, hQ.cuda(), Od, Tn, dm, T.io_cfg(), ws)
    check_status(ws)
    assert torch.equal(hO, Od.cpu())
