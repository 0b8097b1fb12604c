#!/usr/bin/env python
"""Throughput of the large-chunk TTT layer (update + apply) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload zipmap] [--impl ours|reference]

One step is one pass of the whole layer over the workload's tokens, starting
from the initial fast weights: [ShortConv2D on V] + L2-normalised update
(gradient over every token, Newton-Schulz, norm-preserving step; twice for the
two-step workload; per chunk for the streaming workload) + apply.  Inputs are
seeded synthetic tensors already resident in HBM; at the large workloads they
are larger than L2, so no flush is needed between steps; smaller workloads
overwrite a buffer larger than L2 before every step, outside its events.  With N > 1 (torchrun, one rank per GPU)
each rank holds its own token shard of one N-times-larger layer and the
per-step gradient is summed over ranks with an NCCL all-reduce before the
Muon step (the pages' global context synchronisation); per-GPU work is fixed,
so scaling is weak.

Prints one JSON line (rank 0).  --impl reference times the fp64 CPU oracle on
this machine's host cores on a bounded token sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TTT-layer tokens/sec (update+apply) and % of B200 bf16 tensor peak"
UNIT = "tokens/s"
L2_BYTES = 126 << 20
L2_FLUSH_BYTES = 512 << 20
UPDATE_OPERANDS = ("fp16 tensor-core operands: K^ (normalised), V' = -s eta v with a per-call power-of-two s "
                   "(s max|eta| in [16, 32); one rounding), fast-weight copy, dH and u (fp32 accumulation); "
                   "out-of-range operands are reported as TTT_ERR_RANGE and leave W unchanged")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="zipmap")
    ap.add_argument("--frames", type=int, default=0, help="override the workload's frame count (profiling runs)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ---------------------------------------------------------------------------- peaks, clocks


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d.get("hbm_gbs"), "bf16_tflops": d.get("bf16_tflops"),
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a timed region."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = (bus_id or "").upper()
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        with open(self.out.name) as f:
            rows = [ln.strip().split(",") for ln in f if ln.strip()]
        os.unlink(self.out.name)
        rows = [[c.strip() for c in r] for r in rows if len(r) >= 10]
        if self.bus_id:
            mine = [r for r in rows if self.bus_id.endswith(r[1].upper()[-12:]) or r[1].upper().endswith(self.bus_id[-12:])]
            rows = mine or rows
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        smax = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def bus_id_of(dev):
    import torch
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


# ---------------------------------------------------------------------------- oracle (CPU) timing


def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample_times(cfg, sample):
    """Seconds of the fp64 oracle on `sample` tokens of the workload: (per-token update, per-token apply, per-step NS)."""
    import numpy as np
    import oracle as O
    from test_weight_layers_b200 import synth as S
    inp = S.Inputs(cfg)
    K = inp.k(0, sample).double().numpy()
    V = inp.v(0, sample).double().numpy()
    Q = inp.q(0, sample).double().numpy()
    eta = inp.eta(0, sample).double().numpy()
    W = O.FastWeights.of(*(w.numpy() for w in inp.weights()))
    ns = O.NSConfig(cfg.ns_iters, cfg.ns_a, cfg.ns_b, cfg.ns_c, cfg.ns_eps, cfg.lr, cfg.renorm)
    H, d = cfg.heads, cfg.d
    t0 = time.perf_counter()
    Kh = O.l2norm_heads(K, H, d)
    if cfg.conv:
        fr = max(1, sample // (cfg.grid_h * cfg.grid_w))
        n = fr * cfg.grid_h * cfg.grid_w
        Vp = np.array(V)
        Vp[:n] = O.shortconv2d(V[:n], inp.taps().double().numpy(), fr, cfg.grid_h, cfg.grid_w)
    else:
        Vp = V
    G = O.grad(W, Kh, Vp, eta)
    t1 = time.perf_counter()
    Wn = O.muon_step(W, G, ns)
    t2 = time.perf_counter()
    Oq = O.apply(Wn, Q)
    if cfg.gate:
        O.output_gate(Oq, inp.gate_weight().double().numpy())
    t3 = time.perf_counter()
    return (t1 - t0) / sample, (t3 - t2) / sample, (t2 - t1)


def oracle_tokens_per_s(cfg, per_tok_update, per_tok_apply, ns_step):
    T, Ta = cfg.tokens, cfg.apply_tokens
    steps = cfg.steps
    t = steps * (per_tok_update * T) + per_tok_apply * Ta + steps * cfg.n_chunks * ns_step
    return T / t, t


def cpu_baseline(cfg, budget_s=15.0):
    sample = 2048
    u, a, n = oracle_sample_times(cfg, sample)
    est = (u + a) * 1.0
    if est > 0:
        sample = int(min(cfg.tokens, max(2048, budget_s / 2 / est)))
        sample = max(2048, (sample // 2048) * 2048)
        u, a, n = oracle_sample_times(cfg, sample)
    v, _ = oracle_tokens_per_s(cfg, u, a, n)
    return {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": (f"fp64 oracle (numpy/BLAS) on the first {sample} of {cfg.tokens} tokens: gradient, "
                       f"Newton-Schulz step and apply timed, extrapolated linearly in tokens to the full workload "
                       f"(Newton-Schulz counted once per step per chunk)")}


def run_reference(args, cfg):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    sample = min(4096, cfg.tokens)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        u, a, n = oracle_sample_times(cfg, sample)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append((u, a, n, dt))
    u = statistics.median(t[0] for t in times)
    a = statistics.median(t[1] for t in times)
    n = statistics.median(t[2] for t in times)
    v, t_full = oracle_tokens_per_s(cfg, u, a, n)
    line = {"metric": METRIC, "value": v, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_full * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(cfg, args.gpus, "host-side oracle; no GPU caches involved"),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": f"each step: fp64 oracle on {sample} of {cfg.tokens} tokens (gradient, "
                                       f"Newton-Schulz step, apply), extrapolated linearly in tokens"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------- GPU arm


def workload_config(cfg, n, l2_note):
    return {"workload": (f"{cfg.name}: {cfg.frames} frames x ({cfg.grid_h}x{cfg.grid_w}+{cfg.special}) = "
                         f"{cfg.tokens} tokens per GPU, {cfg.heads} heads d={cfg.d} m={cfg.m}, {cfg.steps} Muon "
                         f"step(s){', ShortConv2D on V' if cfg.conv else ''}"
                         f"{f', {cfg.n_chunks} causal chunks of {cfg.chunk} (' if cfg.chunk else ''}"
                         f"{('update then apply)' if cfg.order else 'apply then update)') if cfg.chunk else ''}, "
                         f"apply on {cfg.apply_tokens} tokens"
                         f"{', gated output RMSNorm(o) SiLU(W_g o)' if cfg.gate else ''}"),
            "tokens_per_gpu": cfg.tokens, "heads": cfg.heads, "d": cfg.d, "m": cfg.m, "inner_steps": cfg.steps,
            "chunk": cfg.chunk or None, "order": cfg.order if cfg.chunk else None, "qk_l2norm": True,
            "l2": l2_note,
            "parallelism": "single GPU" if n == 1 else f"token-sharded x{n}, NCCL all-reduce of the gradient"}


def source_sha():
    """Hash of the gradient kernel's source: kernels_tc.cuh up to the apply kernel's
    layout, and common.cuh (the stored traffic is void once either changes)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "test_weight_layers_b200", "csrc")
    with open(os.path.join(csrc, "kernels_tc.cuh"), "rb") as fh:
        tc = fh.read()
    h.update(tc[:tc.index(b"template <int D>\nstruct ApLayout")])
    with open(os.path.join(csrc, "common.cuh"), "rb") as fh:
        h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_per_launch(tokens_per_launch):
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_sha") != source_sha():
        return None
    return d["dram_bytes_per_token"] * tokens_per_launch


def run_ours(args, cfg):
    import torch
    import torch.distributed as dist
    from test_weight_layers_b200 import build as B
    from test_weight_layers_b200 import synth as S
    from test_weight_layers_b200 import ttt as T
    from test_weight_layers_b200.gcs import sharded_layer

    world, rank, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    B.build()
    T.lib()

    H, d, m = cfg.heads, cfg.d, cfg.m
    Tn, Ta = cfg.tokens, cfg.apply_tokens
    D = H * d
    dm = T.dims(H, d, m)
    ns = T.ns_cfg(cfg.ns_iters, cfg.ns_a, cfg.ns_b, cfg.ns_c, cfg.ns_eps, cfg.lr, cfg.renorm)
    io = T.io_cfg()

    g = torch.Generator(device=dev)
    g.manual_seed(cfg.seed * 1000 + rank)

    tdt = cfg.torch_dtype
    dcode = T.dtype_code(tdt)

    def randn_rows(rows, cols):
        out = torch.empty((rows, cols), dtype=tdt, device=dev)
        step = 1 << 17
        for r0 in range(0, rows, step):
            r1 = min(rows, r0 + step)
            out[r0:r1] = torch.randn((r1 - r0, cols), generator=g, device=dev).to(tdt)
        return out

    K = randn_rows(Tn, D)
    V = randn_rows(Tn, D)
    Q = randn_rows(Ta, D)
    if cfg.eta_kind == "linear":
        w_eta = torch.randn((cfg.model_dim, H), generator=g, device=dev) / math.sqrt(cfg.model_dim)
        eta = torch.empty((Tn, H), dtype=torch.float32, device=dev)
        for r0 in range(0, Tn, 1 << 17):
            r1 = min(Tn, r0 + (1 << 17))
            x = torch.randn((r1 - r0, cfg.model_dim), generator=g, device=dev)
            eta[r0:r1] = torch.nn.functional.softplus(x @ w_eta)
    else:
        eta = 0.01 * torch.nn.functional.softplus(torch.randn((Tn, H), generator=g, device=dev))
    W0 = [w.to(dev) for w in S.init_weights(cfg.seed, H, d, m)]
    W = [w.clone() for w in W0]
    Wabi = T.weights(*W)
    taps = S.conv_taps(cfg.seed, D).to(dev) if cfg.conv else None
    Vc = torch.empty_like(V) if cfg.conv else None
    O = torch.empty((Ta, D), dtype=tdt, device=dev)
    # gated output (ZipMap): the apply writes O' and the gate writes the layer output
    Wg = S.gate_weight(cfg.seed, D).to(dev) if cfg.gate else None
    Og = torch.empty_like(O) if cfg.gate else None
    gws = T.gate_workspace(Ta, D, device=dev) if cfg.gate else None
    G = torch.empty(3 * H * m * d, dtype=torch.float32, device=dev)
    ws = T.workspace(dm, cfg.chunk or max(Tn, Ta), dcode, device=dev)
    stream = torch.cuda.current_stream(dev)

    def layer(Kx, Vx, Qx, ex, Ox):
        for w, w0 in zip(W, W0):
            w.copy_(w0, non_blocking=True)
        Vuse = Vx
        if cfg.conv and world == 1 and not cfg.chunk and dcode == T.TTT_BF16:
            # ShortConv2D folded into the update's operand preparation
            T.ttt_update_conv(Wabi, Kx, Vx, ex, Tn, cfg.steps, ns, taps, cfg.grid_h, cfg.grid_w, dm, io, ws)
            T.ttt_apply(Wabi, Qx, Ox, Ta, dm, io, ws)
            return
        if cfg.conv:
            T.ttt_shortconv2d(Vx, Vc, taps, cfg.frames, cfg.grid_h, cfg.grid_w, D)
            Vuse = Vc
        if world == 1 and not cfg.chunk:
            T.ttt_update(Wabi, Kx, Vuse, ex, Tn, cfg.steps, ns, dm, io, ws)
            T.ttt_apply(Wabi, Qx, Ox, Ta, dm, io, ws)
            if cfg.gate:
                T.ttt_output_gate(Ox, Wg, Og, Ta, D, gws)
        elif world == 1:
            T.ttt_chunked(Wabi, Qx, Kx, Vuse, ex, Ox, Tn, cfg.chunk, cfg.order, cfg.steps, ns, dm, io, ws)
        else:
            sharded_layer(
                Tn, cfg.steps,
                grad=lambda t0, t1: (T.ttt_grad(Wabi, Kx[t0:t1], Vuse[t0:t1], ex[t0:t1], t1 - t0, dm, io, G, ws), G)[1],
                grad_again=lambda t0, t1: (T.ttt_grad_prepared(Wabi, Kx[t0:t1], Vuse[t0:t1], ex[t0:t1], t1 - t0, dm,
                                                               io, G, ws), G)[1],
                allreduce=lambda g_: dist.all_reduce(g_),
                step=lambda g_: T.ttt_step(Wabi, g_, ns, dm, dcode, ws),
                apply=(lambda t0, t1: T.ttt_apply(Wabi, Qx[t0:t1], Ox[t0:t1], t1 - t0, dm, io, ws))
                if cfg.chunk else None,
                chunk=cfg.chunk, order=cfg.order)
            if not cfg.chunk:
                T.ttt_apply(Wabi, Qx, Ox, Ta, dm, io, ws)
                if cfg.gate:
                    T.ttt_output_gate(Ox, Wg, Og, Ta, D, gws)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    resident = sum(x.numel() * x.element_size() for x in (K, V, Q, eta, O))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev) if resident < 2 * L2_BYTES else None
    for _ in range(args.warmup):
        layer(K, V, Q, eta, O)
    torch.cuda.synchronize(dev)
    assert T.ttt_poll_status(ws) == T.TTT_OK, "device-side wait timed out during warm-up"

    # ---- timed region (device time, CUDA events on the launching stream)
    T.ttt_profile_reset()
    T.ttt_profile_enable(True)
    barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(bus_id_of(dev))
    time.sleep(0.3)  # let the sampler start
    launches0 = T.ttt_launch_count()
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            layer(K, V, Q, eta, O)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / args.steps
    else:
        # inputs fit in L2: overwrite a buffer larger than L2 before every step and
        # time each step on its own events, so the flush is outside the timed steps
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for a, b in evs:
            flush.fill_(1)
            a.record(stream)
            layer(K, V, Q, eta, O)
            b.record(stream)
        torch.cuda.synchronize(dev)
        ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    launches = T.ttt_launch_count() - launches0
    clk = clocks.stop()
    barrier()
    T.ttt_profile_enable(False)
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    assert T.ttt_poll_status(ws) == T.TTT_OK, "device-side wait timed out during the timed region"
    prof = {T.PROF_NAMES[k]: T.ttt_profile_query(k) for k in range(7)}

    total_tokens = Tn * world
    value = total_tokens / (ms / 1e3)
    peaks = measured_peaks()
    flops_layer = cfg.update_flops() + cfg.apply_flops()
    tflops = flops_layer * world / (ms / 1e3) / 1e12

    # The denominator follows the clocks this run earned: a short timed region at
    # (near) maximum SM clock is a burst, so it is compared with the burst GEMM
    # peak; a long or power-capped one with the sustained peak.  Both fractions
    # are printed.
    region_s = ms * args.steps / 1e3
    at_max = bool(clk and clk.get("sm_mhz") and clk.get("sm_max_mhz")
                  and clk["sm_mhz"] >= 0.95 * clk["sm_max_mhz"])
    use_burst = region_s < 1.0 and at_max
    peak_tf = peaks["bf16_tflops"] if use_burst else peaks["bf16_tflops_sustained"]
    peak_kind = (f"{'burst' if use_burst else 'sustained'} ({peaks['source']}): timed region {region_s:.2f} s, "
                 f"median SM clock {clk.get('sm_mhz') if clk else None} of {clk.get('sm_max_mhz') if clk else None} MHz")

    # dominant kernel: the tensor-core gradient kernel
    g_ms, g_n = prof["grad"]
    tok_per_launch = Tn if not cfg.chunk else cfg.chunk
    grad_flops = 12.0 * H * d * m * tok_per_launch
    roof = None
    if g_n and dcode == T.TTT_BF16:
        ach = grad_flops / (g_ms / g_n / 1e3) / 1e12
        wide = d % 256 == 0 and m % 256 == 0 and d >= 256
        roof = {"bound": "tensor", "achieved": ach, "peak": peak_tf, "unit": "TFLOP/s", "frac": ach / peak_tf,
                "frac_of_burst": ach / peaks["bf16_tflops"], "frac_of_sustained": ach / peaks["bf16_tflops_sustained"],
                "traffic": None if wide else traffic_per_launch(tok_per_launch),
                "kernel": ("k_wgemm gradient products on 2-SM pairs: Z, [H1|H3] with the SwiGLU backward, weight gradients" if wide else "k_update_grad_tc"),
                "peak_kind": "fp16/bf16 dense (same tensor rate), " + peak_kind,
                "launch_ms": g_ms / g_n}
    elif g_n:
        # fp32 mode: CUDA-core FMA pipe, 148 SMs x 128 FMA/clk x 2 flop x 1.965 GHz
        ach = grad_flops / (g_ms / g_n / 1e3) / 1e12
        peak = 148 * 128 * 2 * 1.965e9 / 1e12
        roof = {"bound": "alu", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                "traffic": None, "kernel": "k_grad_f32", "peak_kind": "fp32 FMA, derived from unit counts and max clock",
                "launch_ms": g_ms / g_n}
    kernels = {k: {"ms_per_step": v[0] / args.steps, "launches_per_step": v[1] / args.steps} for k, v in prof.items()}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if dcode == T.TTT_BF16 else "f32", "data": "synthetic",
            "config": workload_config(cfg, world, "inputs larger than L2 (126 MB), no flush between steps"
                                      if flush is None else
                                      f"inputs fit in L2: {L2_FLUSH_BYTES >> 20} MB written before every step, "
                                      "outside its events"),
            "tflops": tflops,
            "layer_frac_of_bf16_peak": {"frac": tflops / world / peak_tf,
                                        "frac_of_burst": tflops / world / peaks["bf16_tflops"],
                                        "frac_of_sustained": tflops / world / peaks["bf16_tflops_sustained"],
                                        "peak_kind": peak_kind},
            "update_operands": UPDATE_OPERANDS if dcode == T.TTT_BF16 else "fp32",
            "roofline": roof, "kernels": kernels, "gpu_launches": launches, "clocks": clk}

    # ---- end to end through the public API with host buffers (pinned), copies inside the timed region
    if not args.no_e2e:
        hK, hV, hQ = (torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in (K, V, Q))
        he = torch.empty(eta.shape, dtype=eta.dtype, pin_memory=True)
        hO = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
        for h_, d_ in ((hK, K), (hV, V), (hQ, Q), (he, eta)):
            h_.copy_(d_)
        bytes_in = sum(x.numel() * x.element_size() for x in (hK, hV, hQ, he))
        bytes_out = hO.numel() * hO.element_size()

        if world == 1 and Ta == Tn and not cfg.gate:
            # the library's host-buffer entry point: copies overlapped with the computation
            dbuf = T.host_buffer(dm, Tn, dcode, conv=cfg.conv, device=dev)

            def e2e_step():
                for w, w0 in zip(W, W0):
                    w.copy_(w0, non_blocking=True)
                T.ttt_layer_host(Wabi, hQ, hK, hV, he, hO, Tn, cfg.chunk, cfg.order, cfg.steps, ns, dm, io, dbuf, ws,
                                 taps=taps, grid_h=cfg.grid_h if cfg.conv else 0,
                                 grid_w=cfg.grid_w if cfg.conv else 0)
            e2e_api = "ttt_layer_host (host buffers, copies overlapped with compute)"
        else:
            def e2e_step():
                K.copy_(hK, non_blocking=True)
                V.copy_(hV, non_blocking=True)
                Q.copy_(hQ, non_blocking=True)
                eta.copy_(he, non_blocking=True)
                layer(K, V, Q, eta, O)
                hO.copy_(Og if cfg.gate else O, non_blocking=True)
            e2e_api = "device entry points with torch copies before and after"

        e2e_step()
        torch.cuda.synchronize(dev)
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = a0.elapsed_time(a1) / args.e2e_steps
        if world > 1:
            t = torch.tensor([e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
        line["e2e"] = {"value": total_tokens / (e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": bytes_in,
                       "d2h_bytes_per_step": bytes_out, "ms_per_step": e_ms, "api": e2e_api}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    from test_weight_layers_b200 import synth as S
    cfg = S.WORKLOADS[args.workload]
    if args.frames:
        cfg = cfg.with_frames(args.frames)
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
