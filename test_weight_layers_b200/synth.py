"""Seeded synthetic inputs for the large-chunk TTT layer.

This module holds the workload recipes (shapes, value distributions) and the
seeded generators that produce every input the layer consumes: Q, K, V token
matrices, per-token learning rates eta, fast-weight initialisations and the
ShortConv2D taps.  It contains none of the layer's own arithmetic; it is
shared, unchanged, by the CPU oracle's tests and by the GPU tests and bench so
that both sides see bit-identical inputs.

Randomness is drawn from ``torch.Generator`` on the CPU, reseeded per block of
``BLOCK`` rows from a 64-bit mix of (config seed, tensor id, block index).  Any
row range can therefore be regenerated independently, which lets the oracle
stream over a million-token workload block by block.

Workloads (the pages give shapes, not data; these stand in for their datasets):

* ``tiny``      1 head, d=64, m=128, 2 frames x 8x8 patches = 128 tokens, fp32.
* ``object``    tttLRM object-scale layer: model dim 768 as 4 heads of d=192,
                m=768; 8 input views x 32x32 tokens (256^2 image, 8x8 patches)
                = 8192 context tokens, plus 8 virtual views x 1024 query tokens.
* ``zipmap``    ZipMap-scale bidirectional chunk: 750 frames x (37x37 + 5
                special tokens) = 1,030,500 tokens; eta = softplus(Linear(x)).
* ``vggt3``     VGG-T3 test-time scaling: 1000 frames x 37x37 = 1,369,000
                tokens, ShortConv2D on V, 2 inner steps.
* ``loger``     LoGeR-style causal stream: 2048 frames x 32x32 = 2,097,152
                tokens in 16 chunks of 131,072.
* ``stream``    ZipMap streaming reconstruction: the zipmap recipe updated
                frame by frame (chunk = one frame of 37x37 + 5 tokens, 750
                chunks), each frame's outputs from the weights after its own
                update (order 1).
* ``zipmap1024`` ZipMap's own head shape: one head with token dim d = 1024
                and hidden m = 2048 (state 6 d^2), the zipmap token recipe, and
                the gated output o = RMSNorm(o') SiLU(W_g o') with a random
                W_g ~ N(0, 1/D).
"""
from __future__ import annotations

import dataclasses
import math

import torch

BLOCK = 1 << 14

# tensor ids used to derive independent streams
TID_Q, TID_K, TID_V, TID_ETA, TID_ETA_X, TID_ETA_W, TID_W, TID_TAPS, TID_GATE = 1, 2, 3, 4, 5, 6, 7, 8, 9

_MASK64 = (1 << 64) - 1


def _mix64(x: int) -> int:
    """SplitMix64 finaliser (Steele, Lea, Flood 2014) on a Python int."""
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _MASK64
    return x ^ (x >> 31)


def stream_seed(seed: int, tensor_id: int, block: int) -> int:
    s = _mix64(_mix64(_mix64(seed) ^ tensor_id) ^ block)
    return s & ((1 << 63) - 1)


def _gen(seed: int, tensor_id: int, block: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(stream_seed(seed, tensor_id, block))
    return g


def normal_rows(seed: int, tensor_id: int, t0: int, t1: int, cols: int,
                dtype: torch.dtype = torch.bfloat16, std: float = 1.0) -> torch.Tensor:
    """Rows [t0, t1) of a [*, cols] matrix of N(0, std^2) values, rounded to ``dtype``.

    Row r is generated from block r // BLOCK, so any slice is reproducible alone.
    """
    if t1 <= t0:
        return torch.empty((0, cols), dtype=dtype)
    out = torch.empty((t1 - t0, cols), dtype=dtype)
    b0, b1 = t0 // BLOCK, (t1 - 1) // BLOCK
    for b in range(b0, b1 + 1):
        blk = torch.randn((BLOCK, cols), generator=_gen(seed, tensor_id, b), dtype=torch.float32)
        if std != 1.0:
            blk = blk * std
        r0 = max(t0, b * BLOCK)
        r1 = min(t1, (b + 1) * BLOCK)
        out[r0 - t0:r1 - t0] = blk[r0 - b * BLOCK:r1 - b * BLOCK].to(dtype)
    return out


def _softplus64(x: torch.Tensor) -> torch.Tensor:
    x = x.double()
    return torch.clamp(x, min=0) + torch.log1p(torch.exp(-x.abs()))


def eta_rows(cfg: "Workload", t0: int, t1: int) -> torch.Tensor:
    """Per-token, per-head learning rates, fp32 [t1-t0, H].

    ``scaled``: 0.01 * softplus(z), z ~ N(0,1) (the tiny workload's recipe).
    ``linear``: softplus(x . w_h), x ~ N(0, I_768) a synthetic model token and
    w_h ~ N(0, 1/768) a random Linear layer, computed in fp64 (ZipMap's
    per-token learning rate predicted by a linear layer from the token).
    """
    H = cfg.heads
    if cfg.eta_kind == "scaled":
        z = normal_rows(cfg.seed, TID_ETA, t0, t1, H, torch.float32)
        return (0.01 * _softplus64(z)).float()
    if cfg.eta_kind == "linear":
        D = cfg.model_dim
        x = normal_rows(cfg.seed, TID_ETA_X, t0, t1, D, torch.float32).double()
        w = normal_rows(cfg.seed, TID_ETA_W, 0, D, H, torch.float32, std=1.0 / math.sqrt(D)).double()
        return _softplus64(x @ w).float()
    raise ValueError(cfg.eta_kind)


def init_weights(seed: int, H: int, d: int, m: int):
    """Fast-weight initialisation W1, W3 ~ N(0, 1/d) [H, m, d]; W2 ~ N(0, 1/m) [H, d, m], fp32."""
    W1 = normal_rows(seed, TID_W, 0, H * m, d, torch.float32, std=1.0 / math.sqrt(d)).reshape(H, m, d)
    W3 = normal_rows(seed, TID_W + 100, 0, H * m, d, torch.float32, std=1.0 / math.sqrt(d)).reshape(H, m, d)
    W2 = normal_rows(seed, TID_W + 200, 0, H * d, m, torch.float32, std=1.0 / math.sqrt(m)).reshape(H, d, m)
    return W1.contiguous(), W3.contiguous(), W2.contiguous()


def gate_weight(seed: int, D: int) -> torch.Tensor:
    """Output-gate weight W_g ~ N(0, 1/D), fp32 [D, D] (row j produces gate j)."""
    return normal_rows(seed, TID_GATE, 0, D, D, torch.float32, std=1.0 / math.sqrt(D)).contiguous()


def conv_taps(seed: int, C: int) -> torch.Tensor:
    """Depthwise 3x3 taps ~ N(0, 1/9), fp32 [C, 3, 3]."""
    return normal_rows(seed, TID_TAPS, 0, C, 9, torch.float32, std=1.0 / 3.0).reshape(C, 3, 3).contiguous()


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    heads: int
    d: int
    m: int
    frames: int
    grid_h: int
    grid_w: int
    special: int = 0            # extra tokens per frame (ZipMap camera/register tokens)
    dtype: str = "bf16"         # "fp32" or "bf16": dtype of Q, K, V, O and MMA operands
    eta_kind: str = "scaled"
    steps: int = 1
    conv: bool = False
    chunk: int = 0              # 0: one bidirectional chunk
    order: int = 0              # chunked: 0 apply with the carried W, then update; 1 update, then apply
    query_tokens: int = 0       # >0: apply on separate query tokens instead of Q of the context
    gate: bool = False          # gated output o = RMSNorm(o') SiLU(W_g o') after the apply
    ns_iters: int = 5
    ns_a: float = 3.4445
    ns_b: float = -4.7750
    ns_c: float = 2.0315
    ns_eps: float = 1e-7
    lr: float = 1.0
    renorm: int = 1

    @property
    def tokens(self) -> int:
        return self.frames * (self.grid_h * self.grid_w + self.special)

    @property
    def model_dim(self) -> int:
        return self.heads * self.d

    @property
    def apply_tokens(self) -> int:
        return self.query_tokens if self.query_tokens else self.tokens

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def update_flops(self) -> float:
        """12*H*d*m flops per context token per inner step (forward + gradient GEMMs)."""
        return 12.0 * self.heads * self.d * self.m * self.tokens * self.steps

    def apply_flops(self) -> float:
        """6*H*d*m flops per query token, plus the gate's 2*D^2 when it is on."""
        gate = 2.0 * self.model_dim * self.model_dim * self.apply_tokens if self.gate else 0.0
        return 6.0 * self.heads * self.d * self.m * self.apply_tokens + gate

    def ns_flops(self) -> float:
        """Newton-Schulz flops per layer: 3H matrices, per iteration 2 r^2 c + 2 r^3 + 2 r^2 c."""
        r, c = min(self.d, self.m), max(self.d, self.m)
        per_iter = 2 * r * r * c + 2 * r * r * r + 2 * r * r * c
        return 3.0 * self.heads * self.ns_iters * per_iter * self.steps * max(1, self.n_chunks)

    @property
    def n_chunks(self) -> int:
        return (self.tokens + self.chunk - 1) // self.chunk if self.chunk else 1

    def with_frames(self, frames: int, chunk: int | None = None, query_tokens: int | None = None) -> "Workload":
        return dataclasses.replace(self, frames=frames,
                                   chunk=self.chunk if chunk is None else chunk,
                                   query_tokens=self.query_tokens if query_tokens is None else query_tokens)


WORKLOADS = {
    "tiny": Workload("tiny", 1000, heads=1, d=64, m=128, frames=2, grid_h=8, grid_w=8, dtype="fp32"),
    "object": Workload("object", 1001, heads=4, d=192, m=768, frames=8, grid_h=32, grid_w=32,
                       query_tokens=8 * 1024),
    "zipmap": Workload("zipmap", 1002, heads=4, d=192, m=768, frames=750, grid_h=37, grid_w=37,
                       special=5, eta_kind="linear"),
    "vggt3": Workload("vggt3", 1003, heads=4, d=192, m=768, frames=1000, grid_h=37, grid_w=37,
                      steps=2, conv=True),
    "loger": Workload("loger", 1004, heads=4, d=192, m=768, frames=2048, grid_h=32, grid_w=32,
                      chunk=128 * 1024),
    "stream": Workload("stream", 1005, heads=4, d=192, m=768, frames=750, grid_h=37, grid_w=37,
                       special=5, eta_kind="linear", chunk=37 * 37 + 5, order=1),
    "zipmap1024": Workload("zipmap1024", 1006, heads=1, d=1024, m=2048, frames=750, grid_h=37, grid_w=37,
                           special=5, eta_kind="linear", gate=True),
}


class Inputs:
    """Lazily generated inputs of one workload; every accessor takes a row range."""

    def __init__(self, cfg: Workload):
        self.cfg = cfg

    def q(self, t0=0, t1=None):
        t1 = self.cfg.apply_tokens if t1 is None else t1
        tid = TID_Q + 10 if self.cfg.query_tokens else TID_Q
        return normal_rows(self.cfg.seed, tid, t0, t1, self.cfg.model_dim, self.cfg.torch_dtype)

    def k(self, t0=0, t1=None):
        t1 = self.cfg.tokens if t1 is None else t1
        return normal_rows(self.cfg.seed, TID_K, t0, t1, self.cfg.model_dim, self.cfg.torch_dtype)

    def v(self, t0=0, t1=None):
        t1 = self.cfg.tokens if t1 is None else t1
        return normal_rows(self.cfg.seed, TID_V, t0, t1, self.cfg.model_dim, self.cfg.torch_dtype)

    def eta(self, t0=0, t1=None):
        t1 = self.cfg.tokens if t1 is None else t1
        return eta_rows(self.cfg, t0, t1)

    def weights(self):
        return init_weights(self.cfg.seed, self.cfg.heads, self.cfg.d, self.cfg.m)

    def taps(self):
        return conv_taps(self.cfg.seed, self.cfg.model_dim)

    def gate_weight(self):
        return gate_weight(self.cfg.seed, self.cfg.model_dim)
