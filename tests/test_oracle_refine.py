"""Pins of the stacked-refinement oracle (SequenceO1 Sec. 3.3, eqs. (12)-(16))
against closed forms, the already pinned single-block SA oracle, and explicit
loops on tiny inputs."""
import math

import numpy as np
import pytest

import oracle
from sa_inputs import gauss, refine_layers, rng_for


def _tiny(seed, n=5, k=3, d=4, n_iter=1, affine=True):
    rng = rng_for(seed)
    X = gauss(rng, (n, d), 0.7).astype(np.float64)
    P0 = gauss(rng, (k, d), 1.0).astype(np.float64)
    return X, P0, refine_layers(rng, n_iter, d, affine)


# ------------------------------------------------------------------ LayerNorm
def test_layer_norm_closed_form():
    # y = [1, 2, 3, 4]: mean 5/2, biased variance 5/4
    y = np.array([[1.0, 2.0, 3.0, 4.0]])
    eps = 1e-3
    ref = (y - 2.5) / math.sqrt(1.25 + eps)
    np.testing.assert_allclose(oracle.layer_norm(y, eps=eps), ref, rtol=1e-14)
    g, b = np.array([2.0, -1.0, 0.5, 3.0]), np.array([0.1, 0.2, 0.3, 0.4])
    np.testing.assert_allclose(oracle.layer_norm(y, g, b, eps), ref * g + b, rtol=1e-14)


def test_layer_norm_row_statistics_and_invariance():
    Y = gauss(rng_for(3), (7, 16), 2.0).astype(np.float64)
    out = oracle.layer_norm(Y, eps=0.0)
    np.testing.assert_allclose(out.mean(axis=1), 0.0, atol=1e-12)
    np.testing.assert_allclose((out ** 2).mean(axis=1), 1.0, rtol=1e-12)
    # shift and positive scale of a row do not change its normalised value
    np.testing.assert_allclose(oracle.layer_norm(3.0 * Y - 5.0, eps=0.0), out, atol=1e-12)


# ------------------------------------------------------------------ SwiGLU FFN
def test_swiglu_against_loops():
    rng = rng_for(5)
    Y = gauss(rng, (3, 4), 1.0).astype(np.float64)
    W1 = gauss(rng, (4, 8), 0.5).astype(np.float64)
    W3 = gauss(rng, (4, 8), 0.5).astype(np.float64)
    W2 = gauss(rng, (8, 4), 0.5).astype(np.float64)
    ref = np.zeros((3, 4))
    for r in range(3):
        for f in range(8):
            a = sum(Y[r, c] * W1[c, f] for c in range(4))
            lin = sum(Y[r, c] * W3[c, f] for c in range(4))
            silu = a / (1.0 + math.exp(-a))
            for o in range(4):
                ref[r, o] += silu * lin * W2[f, o]
    np.testing.assert_allclose(oracle.swiglu_ffn(Y, W1, W3, W2), ref, rtol=1e-12)


def test_swiglu_special_values():
    Y = np.eye(2)
    W1 = np.array([[0.0, 40.0], [0.0, 0.0]])
    W3 = np.ones((2, 2))
    W2 = np.eye(2)
    out = oracle.swiglu_ffn(Y, W1, W3, W2)
    assert out[0, 0] == 0.0                      # SiLU(0) = 0
    assert abs(out[0, 1] - 40.0) < 1e-12         # SiLU(x) -> x for large x
    assert np.all(oracle.swiglu_ffn(Y, W1, np.zeros((2, 2)), W2) == 0.0)


# ------------------------------------------------------------------ refinement
def test_one_iteration_is_ln_of_prototypes_plus_sa_aggregate():
    """With FFN = 0, unit gains and zero biases, one iteration is LN(LN(P0 + A X)),
    where A X is the pinned SA oracle's H (and LN is pinned above)."""
    X, P0, layers = _tiny(11, affine=False)
    L = layers[0]
    L["W2"] = np.zeros_like(L["W2"])
    eps = 1e-6
    _, _, H = oracle.sa_user(X, P0, L["W_Q"], L["W_K"], np.eye(P0.shape[1]), 0.0)
    ref = oracle.layer_norm(oracle.layer_norm(P0 + H, eps=eps), eps=eps)
    np.testing.assert_allclose(oracle.sa_refine_user(X, P0, [L], eps), ref, rtol=1e-12, atol=1e-12)
    # LN is idempotent up to eps: the same within a few eps of LN(P0 + H)
    np.testing.assert_allclose(ref, oracle.layer_norm(P0 + H, eps=eps), atol=10 * eps)


def test_refinement_against_loops():
    """Every step written out with loops over tokens, prototypes and features."""
    X, P0, layers = _tiny(13, n=4, k=3, d=4, n_iter=2)
    eps = 1e-5
    Xt = P0.copy()
    n, d = X.shape
    k = P0.shape[0]
    for L in layers:
        Q = [[sum(Xt[j, c] * L["W_Q"][c, e] for c in range(d)) for e in range(d)] for j in range(k)]
        K = [[sum(X[i, c] * L["W_K"][c, e] for c in range(d)) for e in range(d)] for i in range(n)]
        S = [[sum(Q[j][e] * K[i][e] for e in range(d)) / math.sqrt(d) for i in range(n)] for j in range(k)]
        A = [[0.0] * n for _ in range(k)]
        for i in range(n):
            col = [math.exp(S[j][i]) for j in range(k)]
            for j in range(k):
                A[j][i] = col[j] / sum(col)          # softmax over prototypes
        Xhat = np.array([[sum(A[j][i] * X[i, c] for i in range(n)) for c in range(d)] for j in range(k)])

        def ln(v, g, b):
            mu = sum(v) / len(v)
            var = sum((x - mu) ** 2 for x in v) / len(v)
            return [(x - mu) / math.sqrt(var + eps) * g[c] + b[c] for c, x in enumerate(v)]

        Xbar = np.array([ln(list(Xt[j] + Xhat[j]), L["ln1_g"], L["ln1_b"]) for j in range(k)])
        F = np.zeros((k, d))
        for j in range(k):
            for f in range(2 * d):
                a = sum(Xbar[j, c] * L["W1"][c, f] for c in range(d))
                lin = sum(Xbar[j, c] * L["W3"][c, f] for c in range(d))
                for o in range(d):
                    F[j, o] += a / (1.0 + math.exp(-a)) * lin * L["W2"][f, o]
        Xt = np.array([ln(list(Xbar[j] + F[j]), L["ln2_g"], L["ln2_b"]) for j in range(k)])
    np.testing.assert_allclose(oracle.sa_refine_user(X, P0, layers, eps), Xt, rtol=1e-10, atol=1e-12)


def test_second_iteration_uses_the_users_own_prototypes():
    X, P0, layers = _tiny(17, n=6, k=3, d=4, n_iter=2)
    first = oracle.sa_refine_user(X, P0, layers[:1])
    both = oracle.sa_refine_user(X, P0, layers)
    np.testing.assert_allclose(both, oracle.sa_refine_user(X, first, layers[1:]), rtol=1e-13)
    # and they differ between users: a second user's history changes its prototypes
    X2 = X[::-1] * 1.5
    assert np.max(np.abs(oracle.sa_refine_user(X2, P0, layers) - both)) > 1e-3


def test_token_order_does_not_matter():
    X, P0, layers = _tiny(19, n=7, n_iter=2)
    perm = np.random.default_rng(0).permutation(len(X))
    np.testing.assert_allclose(oracle.sa_refine_user(X[perm], P0, layers),
                               oracle.sa_refine_user(X, P0, layers), rtol=1e-12, atol=1e-13)


def test_batch_matches_users_and_empty_user():
    rng = rng_for(23)
    d, k = 4, 3
    X = gauss(rng, (9, d), 1.0).astype(np.float64)
    P0 = gauss(rng, (k, d), 1.0).astype(np.float64)
    layers = refine_layers(rng, 2, d)
    off = [0, 4, 4, 9]
    out = oracle.sa_refine(X, off, P0, layers)
    np.testing.assert_allclose(out[0], oracle.sa_refine_user(X[0:4], P0, layers), rtol=1e-14)
    np.testing.assert_allclose(out[2], oracle.sa_refine_user(X[4:9], P0, layers), rtol=1e-14)
    # no events: X^ = 0 in every iteration
    Xt = P0
    for L in layers:
        Xbar = oracle.layer_norm(Xt, L["ln1_g"], L["ln1_b"])
        Xt = oracle.layer_norm(Xbar + oracle.swiglu_ffn(Xbar, L["W1"], L["W3"], L["W2"]),
                               L["ln2_g"], L["ln2_b"])
    np.testing.assert_allclose(out[1], Xt, rtol=1e-13)
