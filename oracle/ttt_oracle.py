"""CPU fp64 oracle for the large-chunk test-time-training (TTT) layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only the test suite, the package's smoke check and the bench's CPU-baseline
and reference legs use it.  It shares no code with the CUDA library.

Plain numpy in float64.  A matmul is the only library primitive used; every
other step is written out in the order and notation of the pages:

* fast weights  f_W(x) = W2 (SiLU(W1 x) o (W3 x)),  W = {W1, W2, W3} per head
  -- ZipMap: Linear-Time Stateful 3D Reconstruction via Test-Time Training,
     key design 1 (large-chunk TTT layer).
* loss          L = sum_i eta_i * ( - f_W(k_i)^T v_i )
  -- Scal3R: Scalable Test-Time Training for Large-Scale 3D Reconstruction,
     "Test-time training as memory", scheme 1, eq. (9); ZipMap key design 1.
* one gradient  g = grad_W sum_i eta_i L_i over every token of the chunk
  -- ZipMap key design 1; Scal3R scheme 1.
* Muon step     Delta <- NewtonSchulz(g);  W^ <- ||W|| (W - Delta)/||W - Delta||
  -- ZipMap key design 3 (Newton-Schulz + per-token learning rate).
* apply         o_i = f_W^(q_i)
  -- Scal3R eq. (4); ZipMap key design 1 and 4 (query tokens).
* L2-normalised Q/K and ShortConv2D on V, 1 or 2 inner steps
  -- VGG-T3: Offline Feed-Forward 3D Reconstruction at Scale, key designs 1-3.
* causal chunk carry  W^(t) <- TTTUpdate(W^(t-1); {k, v} of chunk t)
  -- ZipMap key design 4 (streaming); LoGeR: Long-Context Geometric
     Reconstruction with Hybrid Memory, method overview (chunk-wise TTT).
* gradient additivity over token shards (sum of per-shard gradients)
  -- Scal3R scheme 2 (Global Context Synchronization); VGG-T3 key finding 2.
* gated output  o_i = RMSNorm(o'_i) * SiLU(W_g o'_i)
  -- ZipMap key design 3 (the gated unit, second of the three stabilisers).

Readings where the pages are silent or disagree (each is listed again in the
design notes): minus sign on the dot-product loss; plain sum over tokens (no
1/T); Newton-Schulz per 2-D matrix per head, quintic with 5 iterations and
(a, b, c) = (3.4445, -4.7750, 2.0315), input scaled by ||G||_F + eps, run on
the wide orientation; renorm with the Frobenius norm per matrix per head; a
step size lr applied after Newton-Schulz (lr = 1 by default); no momentum;
a second inner step recomputes the gradient at the updated weights; depthwise
3x3 zero-padded cross-correlation per frame, no bias, optional SiLU; L2 norm
with max(||x||, 1e-12); chunked order apply-then-update by default; the
gate's RMSNorm has no learnable scale and eps = 1e-6, and W_g acts on the
token's whole output (all heads concatenated), without bias.

Layouts (all numpy float64 here):
  W1, W3: [H, m, d];  W2: [H, d, m]
  Q, K, V: [T, H*d], head h in columns h*d:(h+1)*d;  eta: [T, H]
"""
from __future__ import annotations

import dataclasses

import numpy as np

L2_EPS = 1e-12


# ---------------------------------------------------------------------------
# elementwise pieces


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def silu(x):
    """SiLU(x) = x * sigmoid(x)."""
    return x * sigmoid(x)


def silu_prime(x):
    """d/dx [x sigmoid(x)] = sigmoid(x) (1 + x (1 - sigmoid(x)))."""
    s = sigmoid(x)
    return s * (1.0 + x * (1.0 - s))


# ---------------------------------------------------------------------------
# Q/K preprocessing (VGG-T3 key design 1) and ShortConv2D (VGG-T3 key design 2)


def l2norm_heads(X: np.ndarray, H: int, d: int, eps: float = L2_EPS) -> np.ndarray:
    """x^ = x / max(||x||_2, eps) per token and per head (parameter-free L2 norm)."""
    T = X.shape[0]
    Xh = np.asarray(X, dtype=np.float64)[:, :H * d].reshape(T, H, d)
    n = np.sqrt(np.sum(Xh * Xh, axis=2, keepdims=True))
    return (Xh / np.maximum(n, eps)).reshape(T, H * d)


def shortconv2d(V: np.ndarray, taps: np.ndarray, N: int, h: int, w: int, act: int = 0) -> np.ndarray:
    """Depthwise 3x3 spatial mixing of V on the per-frame patch grid.

    V is viewed as (N, h, w, C) (token t = (n*h + y)*w + x); each channel c is
    cross-correlated with taps[c] (3x3) with zero padding inside each frame:
        V'[n,y,x,c] = sum_{dy,dx in {-1,0,1}} taps[c, dy+1, dx+1] * V[n, y+dy, x+dx, c]
    then flattened back to tokens.  act=1 applies SiLU afterwards.
    """
    C = taps.shape[0]
    G = np.asarray(V, dtype=np.float64)[:, :C].reshape(N, h, w, C)
    P = np.zeros((N, h + 2, w + 2, C))
    P[:, 1:h + 1, 1:w + 1, :] = G
    out = np.zeros((N, h, w, C))
    tp = np.asarray(taps, dtype=np.float64)
    for dy in (-1, 0, 1):
        for dx in (-1, 0, 1):
            out += tp[:, dy + 1, dx + 1] * P[:, 1 + dy:1 + dy + h, 1 + dx:1 + dx + w, :]
    if act == 1:
        out = silu(out)
    return out.reshape(N * h * w, C)


# ---------------------------------------------------------------------------
# fast-weight function, loss and its gradient (Scal3R eq. (9); ZipMap key design 1)


@dataclasses.dataclass
class FastWeights:
    W1: np.ndarray  # [H, m, d]
    W3: np.ndarray  # [H, m, d]
    W2: np.ndarray  # [H, d, m]

    @staticmethod
    def of(W1, W3, W2) -> "FastWeights":
        return FastWeights(np.array(W1, dtype=np.float64), np.array(W3, dtype=np.float64),
                           np.array(W2, dtype=np.float64))

    def copy(self) -> "FastWeights":
        return FastWeights(self.W1.copy(), self.W3.copy(), self.W2.copy())

    @property
    def dims(self):
        H, m, d = self.W1.shape
        return H, d, m


def head(X: np.ndarray, h: int, d: int) -> np.ndarray:
    return np.asarray(X, dtype=np.float64)[:, h * d:(h + 1) * d]


def fast_forward(W: FastWeights, X: np.ndarray) -> np.ndarray:
    """f_W(x) = W2 (SiLU(W1 x) o (W3 x)) for every row x of X, per head; returns [T, H*d]."""
    H, d, m = W.dims
    out = np.zeros((X.shape[0], H * d))
    for h in range(H):
        x = head(X, h, d)
        h1 = x @ W.W1[h].T          # rows: (W1 x)^T
        h3 = x @ W.W3[h].T
        u = silu(h1) * h3
        out[:, h * d:(h + 1) * d] = u @ W.W2[h].T
    return out


def loss(W: FastWeights, K: np.ndarray, V: np.ndarray, eta: np.ndarray) -> float:
    """L = sum_i eta_i * (-f_W(k_i)^T v_i), summed over heads and tokens (no 1/T)."""
    H, d, m = W.dims
    F = fast_forward(W, K)
    total = 0.0
    for h in range(H):
        total += float(np.sum(-np.asarray(eta, dtype=np.float64)[:, h]
                              * np.sum(F[:, h * d:(h + 1) * d] * head(V, h, d), axis=1)))
    return total


def grad(W: FastWeights, K: np.ndarray, V: np.ndarray, eta: np.ndarray) -> FastWeights:
    """Analytic gradient of L w.r.t. (W1, W3, W2), written out by the chain rule.

    Per token i and head: h1 = W1 k, h3 = W3 k, a = SiLU(h1), u = a o h3, f = W2 u,
    L_i = -eta_i f.v.  Then
        dL/dW2 = -eta_i v u^T
        du     = -eta_i W2^T v
        dL/dh3 = du o a                         -> dL/dW3 = (du o a) k^T
        dL/dh1 = du o h3 o SiLU'(h1)            -> dL/dW1 = (du o h3 o SiLU'(h1)) k^T
    summed over all tokens of the chunk.
    """
    H, d, m = W.dims
    E = np.asarray(eta, dtype=np.float64)
    g1 = np.zeros_like(W.W1)
    g3 = np.zeros_like(W.W3)
    g2 = np.zeros_like(W.W2)
    for h in range(H):
        k = head(K, h, d)
        v = head(V, h, d)
        e = E[:, h:h + 1]
        h1 = k @ W.W1[h].T
        h3 = k @ W.W3[h].T
        a = silu(h1)
        u = a * h3
        g2[h] = (-e * v).T @ u
        du = -e * (v @ W.W2[h])
        dh3 = du * a
        dh1 = du * h3 * silu_prime(h1)
        g3[h] = dh3.T @ k
        g1[h] = dh1.T @ k
    return FastWeights(g1, g3, g2)


def add(A: FastWeights, B: FastWeights) -> FastWeights:
    return FastWeights(A.W1 + B.W1, A.W3 + B.W3, A.W2 + B.W2)


def zeros_like(W: FastWeights) -> FastWeights:
    return FastWeights(np.zeros_like(W.W1), np.zeros_like(W.W3), np.zeros_like(W.W2))


# ---------------------------------------------------------------------------
# Muon step (ZipMap key design 3)


@dataclasses.dataclass
class NSConfig:
    iters: int = 5
    a: float = 3.4445
    b: float = -4.7750
    c: float = 2.0315
    eps: float = 1e-7
    lr: float = 1.0
    renorm: int = 1


def newton_schulz(G: np.ndarray, cfg: NSConfig) -> np.ndarray:
    """Quintic Newton-Schulz orthogonalisation of one matrix.

    X = G / (||G||_F + eps); work on the wide orientation (rows <= cols); then
    ``iters`` times  A = X X^T,  X <- a X + (b A + c A A) X.  iters = 0 returns G
    unchanged (a plain gradient step).
    """
    if cfg.iters == 0:
        return np.array(G, dtype=np.float64)
    X = np.array(G, dtype=np.float64) / (np.linalg.norm(G) + cfg.eps)
    tall = X.shape[0] > X.shape[1]
    if tall:
        X = X.T
    for _ in range(cfg.iters):
        A = X @ X.T
        B = cfg.b * A + cfg.c * (A @ A)
        X = cfg.a * X + B @ X
    return X.T if tall else X


def weight_step(W: np.ndarray, Delta: np.ndarray, cfg: NSConfig) -> np.ndarray:
    """W^ = ||W||_F (W - lr Delta) / ||W - lr Delta||_F  (renorm=0: W - lr Delta)."""
    Wn = W - cfg.lr * Delta
    if not cfg.renorm:
        return Wn
    return np.linalg.norm(W) * Wn / np.linalg.norm(Wn)


def muon_step(W: FastWeights, G: FastWeights, cfg: NSConfig) -> FastWeights:
    """Orthogonalise each per-head gradient matrix (g1, g3, g2 separately) and step."""
    out = W.copy()
    H = W.W1.shape[0]
    for h in range(H):
        out.W1[h] = weight_step(W.W1[h], newton_schulz(G.W1[h], cfg), cfg)
        out.W3[h] = weight_step(W.W3[h], newton_schulz(G.W3[h], cfg), cfg)
        out.W2[h] = weight_step(W.W2[h], newton_schulz(G.W2[h], cfg), cfg)
    return out


# ---------------------------------------------------------------------------
# the layer: update, apply, chunked carry


def prepare_kv(K, V, H, d, qk_l2norm=True, conv=None):
    """K^ (optionally L2-normalised) and V' (optionally ShortConv2D'd), fp64 [T, H*d].

    conv: None or (taps [C,3,3], N, h, w, act).
    """
    Kh = l2norm_heads(K, H, d) if qk_l2norm else np.asarray(K, dtype=np.float64)[:, :H * d]
    if conv is not None:
        taps, N, gh, gw, act = conv
        Vp = shortconv2d(V, taps, N, gh, gw, act)
    else:
        Vp = np.asarray(V, dtype=np.float64)[:, :H * d]
    return Kh, Vp


def update(W: FastWeights, K, V, eta, steps: int, cfg: NSConfig, qk_l2norm=True, conv=None) -> FastWeights:
    """TTTUpdate: ``steps`` times, one gradient over every token, then a Muon step."""
    H, d, m = W.dims
    Kh, Vp = prepare_kv(K, V, H, d, qk_l2norm, conv)
    for _ in range(steps):
        W = muon_step(W, grad(W, Kh, Vp, eta), cfg)
    return W


def apply(W: FastWeights, Q, qk_l2norm=True) -> np.ndarray:
    """o_i = f_W(q^_i) for every query row."""
    H, d, m = W.dims
    Qh = l2norm_heads(Q, H, d) if qk_l2norm else np.asarray(Q, dtype=np.float64)[:, :H * d]
    return fast_forward(W, Qh)


def chunked(W: FastWeights, Q, K, V, eta, chunk: int, steps: int, cfg: NSConfig,
            order: int = 0, qk_l2norm=True):
    """Causal chunk carry.  order 0: O_c = f_{W_(c-1)}(Q_c) then W_c = update(W_(c-1), chunk c);
    order 1: update first, then apply with W_c.  Returns (W_final, O)."""
    T = np.asarray(K).shape[0]
    H, d, m = W.dims
    O = np.zeros((T, H * d))
    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        if order == 0:
            O[c0:c1] = apply(W, Q[c0:c1], qk_l2norm)
            W = update(W, K[c0:c1], V[c0:c1], eta[c0:c1], steps, cfg, qk_l2norm)
        else:
            W = update(W, K[c0:c1], V[c0:c1], eta[c0:c1], steps, cfg, qk_l2norm)
            O[c0:c1] = apply(W, Q[c0:c1], qk_l2norm)
    return W, O


# ---------------------------------------------------------------------------
# ZipMap's gated output (key design 3, second stabiliser)

RMS_EPS = 1e-6


def rmsnorm(X, eps: float = RMS_EPS) -> np.ndarray:
    """RMSNorm(x) = x / sqrt(mean(x^2) + eps) over the last axis, no learnable scale."""
    X = np.asarray(X, dtype=np.float64)
    return X / np.sqrt(np.mean(X * X, axis=-1, keepdims=True) + eps)


def output_gate(Oprime, Wg, eps: float = RMS_EPS) -> np.ndarray:
    """o_i = RMSNorm(o'_i) * SiLU(W_g o'_i) per token; o' [T, D], W_g [D, D] (no bias)."""
    Oprime = np.asarray(Oprime, dtype=np.float64)
    Wg = np.asarray(Wg, dtype=np.float64)
    return rmsnorm(Oprime, eps) * silu(Oprime @ Wg.T)


# ---------------------------------------------------------------------------
# streaming helpers for large token counts (gradient additivity over shards)


def grad_streamed(W: FastWeights, blocks) -> FastWeights:
    """Sum of per-block gradients; ``blocks`` yields (K^, V', eta) row blocks.

    The loss is a sum over tokens, so its gradient is the sum of the gradients
    of any partition of the tokens (Scal3R scheme 2; VGG-T3 key finding 2)."""
    G = zeros_like(W)
    for Kb, Vb, eb in blocks:
        G = add(G, grad(W, Kb, Vb, eb))
    return G


def grad_rows(W: FastWeights, blocks, rows) -> dict:
    """Selected rows of the gradient, by the same chain rule restricted to those rows.

    ``rows`` is a list of (h, j): returns for each the fp64 vectors
    g1[h, j, :] (d), g3[h, j, :] (d) and the column g2[h, :, j] (d).  Each entry needs
    only W1[h, j], W3[h, j] and W2[h, :, j], so this is cheap for any token count."""
    H, d, m = W.dims
    acc = {r: [np.zeros(d), np.zeros(d), np.zeros(d)] for r in rows}
    for Kb, Vb, eb in blocks:
        E = np.asarray(eb, dtype=np.float64)
        for (h, j) in rows:
            k = head(Kb, h, d)
            v = head(Vb, h, d)
            e = E[:, h]
            h1 = k @ W.W1[h, j]
            h3 = k @ W.W3[h, j]
            a = silu(h1)
            u = a * h3
            du = -e * (v @ W.W2[h, :, j])
            acc[(h, j)][0] += (du * h3 * silu_prime(h1)) @ k
            acc[(h, j)][1] += (du * a) @ k
            acc[(h, j)][2] += (-e * u) @ v
    return acc
