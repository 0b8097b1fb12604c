"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test checks one part of the oracle against a hand-worked value, a closed
form, a library routine, or an invariant of the mathematics, chosen so that a
dropped term, a wrong sign, a swapped operand or a transposition fails.
"""
import numpy as np
import pytest
import torch

import oracle as O

RNG = np.random.default_rng(12345)


def rand_weights(H, d, m, rng=RNG, scale=1.0):
    return O.FastWeights(rng.normal(size=(H, m, d)) * scale / np.sqrt(d),
                         rng.normal(size=(H, m, d)) * scale / np.sqrt(d),
                         rng.normal(size=(H, d, m)) * scale / np.sqrt(m))


def nums(s):
    return np.array([float(x) for x in s.split()])


# ---------------------------------------------------------------- f_W and loss


def test_swiglu_hand_values(golden):
    for name, dims, w1, w3, w2, x, exp, _ in golden("swiglu_hand.txt"):
        H, d, m = (int(v) for v in dims.split())
        W = O.FastWeights(nums(w1).reshape(H, m, d), nums(w3).reshape(H, m, d), nums(w2).reshape(H, d, m))
        f = O.fast_forward(W, nums(x).reshape(1, H * d))
        np.testing.assert_allclose(f.ravel(), nums(exp), rtol=1e-14, atol=1e-14, err_msg=name)


def test_loss_sign_hand_values(golden):
    W = O.FastWeights(np.array([[[1.0, 0.0]]]), np.array([[[0.0, 1.0]]]), np.array([[[1.0], [-1.0]]]))
    k = np.array([[1.0, 2.0]])
    for v, eta, exp in golden("loss_hand.txt"):
        L = O.loss(W, k, nums(v).reshape(1, 2), np.array([[float(eta)]]))
        assert abs(L - float(exp)) < 1e-14


def test_loss_negative_when_values_align_with_outputs():
    # v = f_W(k) makes each term -eta ||f||^2 < 0: the minimised loss rewards alignment.
    W = rand_weights(2, 5, 7)
    K = RNG.normal(size=(9, 10))
    V = O.fast_forward(W, K)
    eta = RNG.uniform(0.1, 1.0, size=(9, 2))
    assert O.loss(W, K, V, eta) < 0
    assert O.loss(W, K, -V, eta) > 0


# ---------------------------------------------------------------- gradient


def _fd_grad(W, K, V, eta, h=1e-6):
    out = []
    for name in ("W1", "W3", "W2"):
        A = getattr(W, name)
        G = np.zeros_like(A)
        it = np.nditer(A, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            Wp, Wm = W.copy(), W.copy()
            getattr(Wp, name)[idx] += h
            getattr(Wm, name)[idx] -= h
            G[idx] = (O.loss(Wp, K, V, eta) - O.loss(Wm, K, V, eta)) / (2 * h)
        out.append(G)
    return out


@pytest.mark.parametrize("H,d,m,T", [(1, 3, 4, 5), (2, 4, 3, 6)])
def test_gradient_matches_central_differences(H, d, m, T):
    W = rand_weights(H, d, m, scale=1.5)
    K = RNG.normal(size=(T, H * d))
    V = RNG.normal(size=(T, H * d))
    eta = RNG.uniform(0.05, 2.0, size=(T, H))
    G = O.grad(W, K, V, eta)
    fd1, fd3, fd2 = _fd_grad(W, K, V, eta)
    for an, fd in ((G.W1, fd1), (G.W3, fd3), (G.W2, fd2)):
        err = np.linalg.norm(an - fd) / np.linalg.norm(fd)
        assert err < 1e-7, err


def test_plain_small_step_decreases_loss():
    W = rand_weights(2, 6, 8)
    K = RNG.normal(size=(20, 12))
    V = RNG.normal(size=(20, 12))
    eta = RNG.uniform(0.1, 1.0, size=(20, 2))
    G = O.grad(W, K, V, eta)
    cfg = O.NSConfig(iters=0, lr=1e-3, renorm=0)
    W2 = O.muon_step(W, G, cfg)
    assert O.loss(W2, K, V, eta) < O.loss(W, K, V, eta)


def test_gradient_additive_over_token_shards():
    W = rand_weights(2, 5, 6)
    K = RNG.normal(size=(30, 10))
    V = RNG.normal(size=(30, 10))
    eta = RNG.uniform(0.1, 1.0, size=(30, 2))
    full = O.grad(W, K, V, eta)
    parts = O.grad_streamed(W, [(K[a:b], V[a:b], eta[a:b]) for a, b in ((0, 7), (7, 19), (19, 30))])
    for x, y in ((full.W1, parts.W1), (full.W3, parts.W3), (full.W2, parts.W2)):
        np.testing.assert_allclose(x, y, rtol=1e-12, atol=1e-12)


def test_gradient_rows_agree_with_full_gradient():
    W = rand_weights(2, 5, 6)
    K = RNG.normal(size=(25, 10))
    V = RNG.normal(size=(25, 10))
    eta = RNG.uniform(0.1, 1.0, size=(25, 2))
    full = O.grad(W, K, V, eta)
    rows = [(0, 0), (1, 5), (1, 2)]
    got = O.grad_rows(W, [(K[:10], V[:10], eta[:10]), (K[10:], V[10:], eta[10:])], rows)
    for (h, j) in rows:
        np.testing.assert_allclose(got[(h, j)][0], full.W1[h, j], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(got[(h, j)][1], full.W3[h, j], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(got[(h, j)][2], full.W2[h, :, j], rtol=1e-12, atol=1e-13)


def test_head_independence():
    W = rand_weights(2, 4, 5)
    K = RNG.normal(size=(11, 8))
    V = RNG.normal(size=(11, 8))
    eta = RNG.uniform(0.1, 1.0, size=(11, 2))
    G = O.grad(W, K, V, eta)
    for h in range(2):
        Wh = O.FastWeights(W.W1[h:h + 1], W.W3[h:h + 1], W.W2[h:h + 1])
        Gh = O.grad(Wh, K[:, 4 * h:4 * h + 4], V[:, 4 * h:4 * h + 4], eta[:, h:h + 1])
        np.testing.assert_allclose(G.W1[h], Gh.W1[0], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(G.W2[h], Gh.W2[0], rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- Newton-Schulz


def _scalar_phi(x, cfg):
    for _ in range(cfg.iters):
        x = cfg.a * x + cfg.b * x ** 3 + cfg.c * x ** 5
    return x


def test_ns_scalar_iterates(golden):
    cfg = O.NSConfig()
    x = 1.0
    for step, val in golden("ns_scalar.txt"):
        x = cfg.a * x + cfg.b * x ** 3 + cfg.c * x ** 5
        assert abs(x - float(val)) < 2e-6, (step, x)


@pytest.mark.parametrize("shape", [(12, 40), (40, 12), (16, 16)])
def test_ns_closed_form_on_known_svd(shape):
    # G = U diag(s) V^T  =>  NS(G) = U diag(phi(s / (||s|| + eps))) V^T, phi = p o p o p o p o p
    r = min(shape)
    U, _ = np.linalg.qr(RNG.normal(size=(shape[0], r)))
    Vt, _ = np.linalg.qr(RNG.normal(size=(shape[1], r)))
    s = np.exp(RNG.uniform(-3, 1, size=r))
    G = U @ np.diag(s) @ Vt.T
    cfg = O.NSConfig()
    expected = U @ np.diag(_scalar_phi(s / (np.linalg.norm(s) + cfg.eps), cfg)) @ Vt.T
    np.testing.assert_allclose(O.newton_schulz(G, cfg), expected, rtol=0, atol=1e-12)


def test_ns_output_band():
    cfg = O.NSConfig()
    xs = np.linspace(1e-4, 1.0, 200001)
    phi = _scalar_phi(xs, cfg)
    hi = phi.max()
    lo01 = phi[xs >= 0.01].min()
    G = RNG.normal(size=(48, 192))
    S_in = np.linalg.svd(G, compute_uv=False) / np.linalg.norm(G)
    S_out = np.linalg.svd(O.newton_schulz(G, cfg), compute_uv=False)
    assert S_out.max() <= hi + 1e-9
    assert np.all(S_out[S_in >= 0.01] >= lo01 - 1e-9)
    assert 0.6 < lo01 < 0.7 and 1.1 < hi < 1.25


def test_single_token_rank_one_closed_form(golden):
    # T = 1: every gradient matrix is rank 1, so NS(g) = phi(1) g / ||g|| (up to eps).
    W = rand_weights(1, 6, 10)
    K = RNG.normal(size=(1, 6))
    V = RNG.normal(size=(1, 6))
    eta = np.array([[0.7]])
    G = O.grad(W, K, V, eta)
    cfg = O.NSConfig()
    phi1 = float(golden("ns_scalar.txt")[-1][1])
    for g in (G.W1[0], G.W3[0], G.W2[0]):
        n = np.linalg.norm(g)
        np.testing.assert_allclose(O.newton_schulz(g, cfg), phi1 * g / n, rtol=0, atol=2e-6)


def test_ns_step_is_a_descent_direction():
    W = rand_weights(1, 8, 16)
    K = RNG.normal(size=(40, 8))
    V = RNG.normal(size=(40, 8))
    eta = RNG.uniform(0.1, 1.0, size=(40, 1))
    G = O.grad(W, K, V, eta)
    cfg = O.NSConfig()
    for g in (G.W1[0], G.W3[0], G.W2[0]):
        assert np.sum(g * O.newton_schulz(g, cfg)) > 0


# ---------------------------------------------------------------- weight step


def test_weight_step_special_cases():
    W = RNG.normal(size=(6, 9))
    cfg = O.NSConfig()
    np.testing.assert_allclose(O.weight_step(W, 0.5 * W, cfg), W, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(O.weight_step(W, 2.0 * W, cfg), -W, rtol=1e-14, atol=1e-14)
    D = RNG.normal(size=(6, 9))
    out = O.weight_step(W, D, cfg)
    assert abs(np.linalg.norm(out) - np.linalg.norm(W)) < 1e-12
    plain = O.weight_step(W, D, O.NSConfig(renorm=0, lr=0.25))
    np.testing.assert_allclose(plain, W - 0.25 * D, rtol=1e-15, atol=1e-15)


# ---------------------------------------------------------------- update invariants


def _update_inputs(H=2, d=6, m=8, T=24, rng=RNG):
    W = rand_weights(H, d, m, rng)
    K = rng.normal(size=(T, H * d))
    V = rng.normal(size=(T, H * d))
    eta = rng.uniform(0.05, 1.0, size=(T, H))
    return W, K, V, eta


def test_update_eta_zero_leaves_weights():
    W, K, V, eta = _update_inputs()
    out = O.update(W, K, V, 0 * eta, 1, O.NSConfig())
    for a, b in ((out.W1, W.W1), (out.W3, W.W3), (out.W2, W.W2)):
        np.testing.assert_allclose(a, b, rtol=1e-14, atol=1e-14)


def test_update_value_zero_leaves_weights():
    W, K, V, eta = _update_inputs()
    out = O.update(W, K, 0 * V, eta, 1, O.NSConfig())
    np.testing.assert_allclose(out.W2, W.W2, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(out.W1, W.W1, rtol=1e-14, atol=1e-14)


def test_update_eta_scale_invariant():
    W, K, V, eta = _update_inputs()
    a = O.update(W, K, V, eta, 1, O.NSConfig())
    b = O.update(W, K, V, 37.0 * eta, 1, O.NSConfig())
    np.testing.assert_allclose(a.W1, b.W1, rtol=0, atol=1e-6)
    np.testing.assert_allclose(a.W2, b.W2, rtol=0, atol=1e-6)


def test_update_token_permutation_invariant():
    W, K, V, eta = _update_inputs()
    p = RNG.permutation(K.shape[0])
    a = O.update(W, K, V, eta, 2, O.NSConfig())
    b = O.update(W, K[p], V[p], eta[p], 2, O.NSConfig())
    np.testing.assert_allclose(a.W1, b.W1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(a.W3, b.W3, rtol=0, atol=1e-12)
    np.testing.assert_allclose(a.W2, b.W2, rtol=0, atol=1e-12)


def test_update_writes_memory_of_a_single_token():
    # One step on (k, v) raises f(k).v: the key-value pair is stored in W.
    W = rand_weights(1, 8, 32)
    k = RNG.normal(size=(1, 8))
    v = RNG.normal(size=(1, 8))
    eta = np.array([[1.0]])
    before = float((O.apply(W, k, qk_l2norm=True) @ v.T)[0, 0])
    Wn = O.update(W, k, v, eta, 1, O.NSConfig())
    after = float((O.apply(Wn, k, qk_l2norm=True) @ v.T)[0, 0])
    assert after > before


# ---------------------------------------------------------------- L2 norm and ShortConv2D


def test_l2norm_rows():
    X = RNG.normal(size=(7, 12)) * RNG.uniform(0.01, 50, size=(7, 1))
    X[3, 6:] = 0.0
    Y = O.l2norm_heads(X, 2, 6)
    n = np.linalg.norm(Y.reshape(7, 2, 6), axis=2)
    assert np.allclose(np.delete(n.ravel(), 3 * 2 + 1), 1.0, atol=1e-14)
    assert n[3, 1] == 0.0
    cos = np.sum(Y[:, :6] * X[:, :6], axis=1) / np.linalg.norm(X[:, :6], axis=1)
    np.testing.assert_allclose(cos, 1.0, atol=1e-14)


def test_shortconv_matches_torch_conv2d():
    N, h, w, C = 3, 5, 7, 6
    V = RNG.normal(size=(N * h * w, C))
    taps = RNG.normal(size=(C, 3, 3))
    got = O.shortconv2d(V, taps, N, h, w)
    x = torch.from_numpy(V.reshape(N, h, w, C)).permute(0, 3, 1, 2)
    ref = torch.nn.functional.conv2d(x, torch.from_numpy(taps).unsqueeze(1), padding=1, groups=C)
    ref = ref.permute(0, 2, 3, 1).reshape(N * h * w, C).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)
    got_act = O.shortconv2d(V, taps, N, h, w, act=1)
    np.testing.assert_allclose(got_act, ref / (1 + np.exp(-ref)), rtol=1e-13, atol=1e-13)


def test_shortconv_impulse_returns_flipped_taps_and_frames_do_not_mix():
    N, h, w, C = 2, 5, 5, 3
    taps = RNG.normal(size=(C, 3, 3))
    V = np.zeros((N * h * w, C))
    V[(0 * h + 2) * w + 2] = 1.0             # impulse in frame 0 at (2, 2)
    out = O.shortconv2d(V, taps, N, h, w).reshape(N, h, w, C)
    for c in range(C):
        np.testing.assert_allclose(out[0, 1:4, 1:4, c], taps[c, ::-1, ::-1], atol=0)
    assert np.all(out[1] == 0)
    # constant interior: sum of taps
    Vc = np.ones((N * h * w, C))
    oc = O.shortconv2d(Vc, taps, N, h, w).reshape(N, h, w, C)
    np.testing.assert_allclose(oc[:, 2, 2, :], np.broadcast_to(taps.sum(axis=(1, 2)), (N, C)), atol=1e-14)


# ---------------------------------------------------------------- apply and chunked carry


def test_apply_rows_independent_and_normalised():
    W = rand_weights(2, 5, 7)
    Q = RNG.normal(size=(9, 10))
    full = O.apply(W, Q)
    for i in (0, 4, 8):
        np.testing.assert_allclose(O.apply(W, Q[i:i + 1]), full[i:i + 1], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(O.apply(W, 3.0 * Q), full, rtol=1e-13, atol=1e-13)


def test_chunked_single_chunk_equals_bidirectional_update():
    W, K, V, eta = _update_inputs(T=30)
    Q = RNG.normal(size=K.shape)
    cfg = O.NSConfig()
    Wc, Oc = O.chunked(W, Q, K, V, eta, chunk=30, steps=1, cfg=cfg, order=0)
    Wu = O.update(W, K, V, eta, 1, cfg)
    np.testing.assert_allclose(Wc.W1, Wu.W1, rtol=0, atol=1e-14)
    np.testing.assert_allclose(Oc, O.apply(W, Q), rtol=0, atol=1e-14)
    Wc1, Oc1 = O.chunked(W, Q, K, V, eta, chunk=30, steps=1, cfg=cfg, order=1)
    np.testing.assert_allclose(Oc1, O.apply(Wu, Q), rtol=0, atol=1e-14)


def test_chunked_carry_resumes():
    W, K, V, eta = _update_inputs(T=40)
    Q = RNG.normal(size=K.shape)
    cfg = O.NSConfig()
    Wall, Oall = O.chunked(W, Q, K, V, eta, chunk=10, steps=1, cfg=cfg)
    Wa, Oa = O.chunked(W, Q[:20], K[:20], V[:20], eta[:20], chunk=10, steps=1, cfg=cfg)
    Wb, Ob = O.chunked(Wa, Q[20:], K[20:], V[20:], eta[20:], chunk=10, steps=1, cfg=cfg)
    np.testing.assert_allclose(Wb.W2, Wall.W2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(np.vstack([Oa, Ob]), Oall, rtol=0, atol=1e-14)
    # chunk c's output uses only chunks < c: changing the last chunk's K leaves earlier O
    K2 = K.copy()
    K2[30:] = RNG.normal(size=(10, K.shape[1]))
    _, O2 = O.chunked(W, Q, K2, V, eta, chunk=10, steps=1, cfg=cfg)
    np.testing.assert_allclose(O2[:40], Oall[:40], rtol=0, atol=0)
    V2 = V.copy()
    V2[0:10] *= -1.0
    _, O3 = O.chunked(W, Q, K, V2, eta, chunk=10, steps=1, cfg=cfg)
    np.testing.assert_allclose(O3[:10], Oall[:10], atol=0)
    assert np.abs(O3[10:] - Oall[10:]).max() > 1e-6


# ---------------------------------------------------------------------------
# ZipMap's gated output o = RMSNorm(o') * SiLU(W_g o') (key design 3)

def test_output_gate_hand_worked_identity_gate():
    # x = [1, -2, 3]: mean(x^2) = 14/3, so RMSNorm(x) = x sqrt(3/14) (eps shifts it by ~1e-7);
    # logistic values sigma(1), sigma(-2), sigma(3) from tables
    r = 0.4629100498862757  # sqrt(3/14)
    s1, sm2, s3 = 0.7310585786300049, 0.11920292202211755, 0.9525741268224334
    x = np.array([[1.0, -2.0, 3.0]])
    want = np.array([1.0 * r * (1.0 * s1), -2.0 * r * (-2.0 * sm2), 3.0 * r * (3.0 * s3)])
    got = O.output_gate(x, np.eye(3))[0]
    assert np.allclose(got, want, rtol=1e-6, atol=0)


def test_output_gate_zero_gate_and_orientation():
    rng = np.random.default_rng(70)
    x = rng.standard_normal((5, 6))
    assert np.array_equal(O.output_gate(x, np.zeros((6, 6))), np.zeros((5, 6)))
    # W_g maps component 1 to component 0 only: W_g x = [x1, 0, ...] (a transposed
    # gate would give [0, x0, 0, ...])
    Wg = np.zeros((6, 6))
    Wg[0, 1] = 1.0
    got = O.output_gate(x, Wg)
    rms = O.rmsnorm(x)
    assert np.all(got[:, 1:] == 0.0)
    assert np.allclose(got[:, 0], rms[:, 0] * x[:, 1] / (1.0 + np.exp(-x[:, 1])), rtol=1e-12)


def test_output_gate_rmsnorm_is_per_token_and_scale_free():
    rng = np.random.default_rng(71)
    x = rng.standard_normal((7, 8))
    Wg = rng.standard_normal((8, 8))
    c = np.exp(rng.standard_normal((7, 1)))  # a different positive scale per token
    # RMSNorm(c x) = RMSNorm(x) per row and W_g/c (c x) = W_g x, up to the eps term
    a = O.output_gate(x, Wg, eps=0.0)
    b = np.stack([O.output_gate(c[i] * x[i:i + 1], Wg / c[i], eps=0.0)[0] for i in range(7)])
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)
    # each normalised row has mean square 1
    assert np.allclose(np.mean(O.rmsnorm(x, eps=0.0) ** 2, axis=1), 1.0, rtol=1e-12)


# ---------------------------------------------------------------------------
# which orthogonalised gradient goes to which matrix (ZipMap key design 3),
# the second inner step (VGG-T3 key design 3), and which tensor ShortConv2D
# acts on (VGG-T3 key design 2)


def _rank1(rng, r, c):
    return np.outer(rng.normal(size=r), rng.normal(size=c))


def test_muon_step_pairs_each_gradient_with_its_own_matrix(golden):
    # Rank-1 gradients have the closed form NS(g) = phi(1) g / ||g|| (phi(1) from the
    # scalar iterates), so each updated matrix follows from its own gradient alone.
    rng = np.random.default_rng(81)
    H, d, m = 2, 5, 9
    W = rand_weights(H, d, m, rng)
    G = O.FastWeights(np.stack([_rank1(rng, m, d) for _ in range(H)]),
                      np.stack([_rank1(rng, m, d) for _ in range(H)]),
                      np.stack([_rank1(rng, d, m) for _ in range(H)]))
    cfg = O.NSConfig()
    phi1 = float(golden("ns_scalar.txt")[-1][1])
    out = O.muon_step(W, G, cfg)
    for name in ("W1", "W3", "W2"):
        for h in range(H):
            w = getattr(W, name)[h]
            g = getattr(G, name)[h]
            step = w - phi1 * g / np.linalg.norm(g)
            want = np.linalg.norm(w) * step / np.linalg.norm(step)
            np.testing.assert_allclose(getattr(out, name)[h], want, rtol=0, atol=2e-6, err_msg=f"{name}[{h}]")
    # a gradient in one matrix moves that matrix only: NS(0) = 0 leaves the others as they were
    for only in ("W1", "W3", "W2"):
        Z = O.FastWeights(np.zeros_like(W.W1), np.zeros_like(W.W3), np.zeros_like(W.W2))
        getattr(Z, only)[:] = getattr(G, only)
        res = O.muon_step(W, Z, cfg)
        for name in ("W1", "W3", "W2"):
            same = np.allclose(getattr(res, name), getattr(W, name), rtol=0, atol=1e-14)
            assert same == (name != only), (only, name)


def test_two_inner_steps_recompute_the_gradient_at_the_updated_weights():
    # steps = 2 is one step, then another from the weights the first produced; reusing the
    # first gradient for the second step gives a different result.
    W, K, V, eta = _update_inputs(H=2, d=6, m=8, T=24, rng=np.random.default_rng(82))
    cfg = O.NSConfig()
    two = O.update(W, K, V, eta, 2, cfg)
    once = O.update(W, K, V, eta, 1, cfg)
    twice = O.update(once, K, V, eta, 1, cfg)
    for name in ("W1", "W3", "W2"):
        np.testing.assert_allclose(getattr(two, name), getattr(twice, name), rtol=0, atol=1e-13)
    Kh = O.l2norm_heads(K, 2, 6)
    g0 = O.grad(W, Kh, V, eta)
    stale = O.muon_step(O.muon_step(W, g0, cfg), g0, cfg)
    assert np.abs(stale.W1 - two.W1).max() > 1e-3
    # the second step's gradient is the gradient at the once-updated weights
    g1 = O.grad(once, Kh, V, eta)
    assert np.abs(g1.W2 - g0.W2).max() > 1e-3 * np.abs(g0.W2).max()


def test_shortconv_acts_on_values_only():
    # VGG-T3 key design 2: the regression target becomes K -> V' = ShortConv2D(V); K is only
    # L2-normalised.  So the update with the conv equals the update on a pre-convolved V.
    rng = np.random.default_rng(83)
    H, d, m, N, gh, gw = 2, 4, 8, 2, 3, 4
    T = N * gh * gw
    W = rand_weights(H, d, m, rng)
    K = rng.normal(size=(T, H * d))
    V = rng.normal(size=(T, H * d))
    eta = rng.uniform(0.05, 1.0, size=(T, H))
    taps = rng.normal(size=(H * d, 3, 3)) / 3.0
    cfg = O.NSConfig()
    for act in (0, 1):
        with_conv = O.update(W, K, V, eta, 1, cfg, conv=(taps, N, gh, gw, act))
        Vp = O.shortconv2d(V, taps, N, gh, gw, act)
        pre = O.update(W, K, Vp, eta, 1, cfg)
        for name in ("W1", "W3", "W2"):
            np.testing.assert_allclose(getattr(with_conv, name), getattr(pre, name), rtol=0, atol=1e-13)
        # and the conv does change the result (it is not a no-op on these inputs)
        plain = O.update(W, K, V, eta, 1, cfg)
        assert np.abs(plain.W2 - with_conv.W2).max() > 1e-3
    Kh, Vh = O.prepare_kv(K, V, H, d, True, (taps, N, gh, gw, 0))
    np.testing.assert_allclose(Kh, O.l2norm_heads(K, H, d), rtol=0, atol=0)
