"""Helpers shared by the GPU parity tests: device setup, oracle conversions, error metrics."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from test_weight_layers_b200 import build as B
from test_weight_layers_b200 import ttt as T

# relative Frobenius tolerances: fp32 mode and bf16 mode (fast weights and outputs)
TOL_FP32 = 1e-4
TOL_BF16 = 3e-2


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    T.lib()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_fro(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def rand_tokens(T_, H, d, dtype, seed, ld=None, scale=1.0):
    """CPU tensor [T][ld] (ld >= H*d) with N(0, scale^2) in the first H*d columns, rounded to dtype."""
    g = torch.Generator().manual_seed(seed)
    ld = ld or H * d
    x = torch.zeros((T_, ld), dtype=torch.float32)
    x[:, :H * d] = torch.randn((T_, H * d), generator=g) * scale
    return x.to(dtype)


def rand_weights(H, d, m, seed):
    g = torch.Generator().manual_seed(seed)
    W1 = torch.randn((H, m, d), generator=g) / d ** 0.5
    W3 = torch.randn((H, m, d), generator=g) / d ** 0.5
    W2 = torch.randn((H, d, m), generator=g) / m ** 0.5
    return W1, W3, W2


def rand_eta(T_, H, seed, scale=0.01):
    g = torch.Generator().manual_seed(seed)
    return (scale * torch.nn.functional.softplus(torch.randn((T_, H), generator=g, dtype=torch.float64))).float()


class DevWeights:
    """fp32 fast weights on the device plus their ABI struct."""

    def __init__(self, W1, W3, W2):
        self.W1, self.W3, self.W2 = (w.float().contiguous().cuda() for w in (W1, W3, W2))
        self.abi = T.weights(self.W1, self.W3, self.W2)

    def oracle(self) -> O.FastWeights:
        return O.FastWeights(f64(self.W1), f64(self.W3), f64(self.W2))

    def numpy(self):
        return f64(self.W1), f64(self.W3), f64(self.W2)


def weight_errors(got: O.FastWeights, ref: O.FastWeights):
    """Relative Frobenius error per matrix and head."""
    out = []
    H = ref.W1.shape[0]
    for name in ("W1", "W3", "W2"):
        for h in range(H):
            out.append(rel_fro(getattr(got, name)[h], getattr(ref, name)[h]))
    return out


def check_status(ws):
    assert T.ttt_poll_status(ws) == T.TTT_OK, "device-side wait timed out"
