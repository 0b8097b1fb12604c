"""Multi-rank layer (gradient summed across ranks) on world-size-2 gloo CPU ranks.

Each rank runs the fp64 oracle on its token shard through the same sequencing
function the bench uses with NCCL; the result must equal one process running the
whole sequence: identical fast weights on every rank, equal to the unsharded
update, and each rank's outputs equal to the unsharded outputs of its rows."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from test_weight_layers_b200.gcs import sharded_layer


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _data(H=2, d=6, m=8, T=48, seed=7):
    rng = np.random.default_rng(seed)
    W = O.FastWeights(rng.normal(size=(H, m, d)) / np.sqrt(d), rng.normal(size=(H, m, d)) / np.sqrt(d),
                      rng.normal(size=(H, d, m)) / np.sqrt(m))
    K, V, Q = (rng.normal(size=(T, H * d)) for _ in range(3))
    eta = rng.uniform(0.05, 1.0, size=(T, H))
    return W, K, V, Q, eta


def _rank_main(rank, world, port, chunk, steps, order, again, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W, K, V, Q, eta = _data()
        T = K.shape[0]
        per = T // world
        sl = slice(rank * per, (rank + 1) * per)
        Kl, Vl, Ql, el = K[sl], V[sl], Q[sl], eta[sl]
        H, d, m = W.dims
        cfg = O.NSConfig()
        state = {"W": W}
        calls = {"grad": 0, "again": 0}
        outs = np.zeros((per, H * d))

        def grad_of(t0, t1):
            g = O.grad(state["W"], O.l2norm_heads(Kl[t0:t1], H, d), Vl[t0:t1], el[t0:t1])
            return torch.from_numpy(np.concatenate([g.W1.ravel(), g.W3.ravel(), g.W2.ravel()]))

        def grad(t0, t1):
            calls["grad"] += 1
            return grad_of(t0, t1)

        def grad_again(t0, t1):
            calls["again"] += 1
            return grad_of(t0, t1)

        def allreduce(G):
            dist.all_reduce(G)

        def step(G):
            g = G.numpy()
            n = H * m * d
            Gw = O.FastWeights(g[:n].reshape(H, m, d), g[n:2 * n].reshape(H, m, d), g[2 * n:].reshape(H, d, m))
            state["W"] = O.muon_step(state["W"], Gw, cfg)

        def apply(t0, t1):
            outs[t0:t1] = O.apply(state["W"], Ql[t0:t1])

        sharded_layer(per, steps, grad, allreduce, step, apply, chunk=chunk, order=order,
                      grad_again=grad_again if again else None)
        Wf = state["W"]
        out_q.put((rank, np.concatenate([Wf.W1.ravel(), Wf.W3.ravel(), Wf.W2.ravel()]), outs, calls))
    finally:
        dist.destroy_process_group()


# again: the later inner steps of a chunk go through grad_again (the library's
# ttt_grad_prepared, which reuses the operands the chunk's first ttt_grad prepared)
@pytest.mark.parametrize("chunk,steps,order,again", [(0, 1, 0, False), (0, 2, 0, False), (8, 1, 0, False),
                                                     (8, 1, 1, False), (0, 2, 0, True), (8, 2, 1, True)])
def test_two_rank_gcs_equals_single_process(chunk, steps, order, again):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, chunk, steps, order, again, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, w, o, calls = q.get(timeout=120)
        res[r] = (w, o)
        # one first-step gradient per chunk; the later steps through grad_again when given
        n_chunks = 1 if chunk == 0 else (len(_data()[1]) // 2) // chunk
        later = n_chunks * (steps - 1)
        assert calls == ({"grad": n_chunks, "again": later} if again else {"grad": n_chunks + later, "again": 0})
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # all ranks hold identical weights
    np.testing.assert_array_equal(res[0][0], res[1][0])
    # equal to one process over the whole sequence
    W, K, V, Q, eta = _data()
    T = K.shape[0]
    cfg = O.NSConfig()
    if chunk == 0:
        Wr = O.update(W, K, V, eta, steps, cfg)
        Or = O.apply(Wr, Q)
    else:
        # the whole sequence's chunk c is the union of both ranks' local chunk c
        per = T // 2
        Wr = W
        Or = np.zeros_like(Q)
        for c0 in range(0, per, chunk):
            idx = np.r_[c0:c0 + chunk, per + c0:per + c0 + chunk]
            if order == 0:
                Or[idx] = O.apply(Wr, Q[idx])
            Wr = O.update(Wr, K[idx], V[idx], eta[idx], steps, cfg)
            if order == 1:
                Or[idx] = O.apply(Wr, Q[idx])
    wr = np.concatenate([Wr.W1.ravel(), Wr.W3.ravel(), Wr.W2.ravel()])
    np.testing.assert_allclose(res[0][0], wr, rtol=0, atol=1e-10)
    np.testing.assert_allclose(np.vstack([res[0][1], res[1][1]]), Or, rtol=0, atol=1e-10)


def _failing_rank_main(rank, world, port, out_q):
    """Rank 1 fails inside its first gradient (an exception on the host, before the
    collective); rank 0 must see its all-reduce fail rather than wait for ever."""
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=20))
    W, K, V, Q, eta = _data()
    H, d, m = W.dims
    per = K.shape[0] // world
    Kl, Vl, el = K[rank * per:(rank + 1) * per], V[rank * per:(rank + 1) * per], eta[rank * per:(rank + 1) * per]
    state = {"W": W}

    def grad(t0, t1):
        if rank == 1:
            raise RuntimeError("injected host-side failure")
        g = O.grad(state["W"], O.l2norm_heads(Kl[t0:t1], H, d), Vl[t0:t1], el[t0:t1])
        return torch.from_numpy(np.concatenate([g.W1.ravel(), g.W3.ravel(), g.W2.ravel()]))

    def step(G):
        pass

    code = 0
    try:
        sharded_layer(per, 1, grad, lambda G: dist.all_reduce(G), step)
        out_q.put((rank, "completed"))
    except Exception as e:  # noqa: BLE001 - the test reports what each rank saw
        out_q.put((rank, type(e).__name__))
        code = 3 if rank == 1 else 0
    out_q.close()
    out_q.join_thread()  # the report is flushed before the process leaves
    os._exit(code)  # no destroy_process_group: rank 1 leaves as a crashed rank would


def test_a_failing_rank_surfaces_as_an_error_on_the_others():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    seen = {}
    for _ in range(2):
        r, what = q.get(timeout=120)
        seen[r] = what
    for p in procs:
        p.join(timeout=60)
    assert seen[1] == "RuntimeError"
    # the surviving rank's collective raised (peer gone or timed out) instead of hanging
    assert seen[0] != "completed", seen
    assert procs[1].exitcode == 3
