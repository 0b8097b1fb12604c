"""Token-sharded layer across devices: Global Context Synchronization.

Each rank holds a shard of the tokens (whole frames).  Per update step every
rank computes the gradient of the dot-product loss on its shard, the gradients
are summed across ranks (the loss is a sum over tokens, so the sum of shard
gradients is the gradient of the whole sequence), and every rank takes the
same Muon step, so all ranks keep identical fast weights.  This follows
Scal3R's scheme 2 (gradients computed per GPU, summed and shared) and tttLRM's
sequence parallelism.

This module only sequences the calls; the arithmetic is done by the callables
it is given (the CUDA library in the bench, the oracle in the CPU tests).
"""
from __future__ import annotations

from typing import Callable, Optional


def sharded_layer(n_tokens: int, steps: int, grad: Callable[[int, int], object],
                  allreduce: Callable[[object], None], step: Callable[[object], None],
                  apply: Optional[Callable[[int, int], None]] = None, chunk: int = 0, order: int = 0,
                  grad_again: Optional[Callable[[int, int], object]] = None) -> None:
    """Run one layer over this rank's `n_tokens` tokens.

    grad(t0, t1) -> G: gradient of the loss over local tokens [t0, t1) at the current weights.
    allreduce(G): in-place sum of G over all ranks (every rank calls it in the same order).
    step(G): Muon step of the local weights from the summed gradient.
    apply(t0, t1): outputs for local query rows [t0, t1) with the current weights.
    chunk > 0: causal carry over chunks of `chunk` local tokens (each chunk of the
    whole sequence is the union of the ranks' chunk c); order 0 applies before the
    chunk's update, order 1 after.  chunk = 0: one bidirectional chunk, apply after.
    grad_again(t0, t1), if given, is used for the second and later inner steps of a
    chunk: the same gradient, reusing what the first call prepared for those tokens.
    All ranks must pass the same n_tokens, chunk and steps so the collectives line up.
    """
    size = chunk if chunk > 0 else n_tokens
    for c0 in range(0, max(n_tokens, 1), max(size, 1)):
        c1 = min(n_tokens, c0 + size)
        if chunk > 0 and order == 0 and apply is not None:
            apply(c0, c1)
        for st in range(steps):
            G = grad(c0, c1) if st == 0 or grad_again is None else grad_again(c0, c1)
            allreduce(G)
            step(G)
        if chunk > 0 and order == 1 and apply is not None:
            apply(c0, c1)
    if chunk <= 0 and apply is not None:
        apply(0, n_tokens)
