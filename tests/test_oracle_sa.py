"""Pins of the SA oracle against what the SequenceO1 pages and the mathematics
fix (no GPU).  Each test would fail under a plausible slip in the oracle: a
softmax over the wrong axis, a dropped 1/sqrt(d), a transposed projection, a
missing normalisation or value projection, a wrong gradient term."""
import math

import numpy as np
import pytest

import oracle
from sa_inputs import make_sa_problem


def _prob(lengths=(37, 0, 19), k=5, d=8, seed=7, **kw):
    return make_sa_problem(lengths, k, d, "f32", seed, **kw)


def test_columns_sum_to_one_and_total_mass():
    """eq. (7): every token's weights over the k prototypes sum to one, so the
    total mass of a user equals its number of tokens."""
    p = _prob(lengths=(50, 13), k=7, d=6, p_scale=4.0)
    for u in range(p.B):
        X = p.x_f64(p.offsets[u], p.offsets[u + 1])
        A = oracle.assignment(X, p.P, p.W_Q, p.W_K)
        assert A.shape == (7, X.shape[0])
        np.testing.assert_allclose(A.sum(axis=0), 1.0, atol=1e-13)
        assert (A >= 0).all()
    S, m, H = oracle.sa_forward(p.x_f64(), p.offsets, p.P, p.W_Q, p.W_K, p.W_V, p.eps)
    np.testing.assert_allclose(m.sum(axis=1), np.diff(p.offsets), rtol=1e-12)


def test_token_permutation_invariance():
    """The sketch is a sum over tokens, so it does not depend on their order."""
    p = _prob(lengths=(41,), k=6, d=5, p_scale=3.0)
    X = p.x_f64()
    perm = np.random.default_rng(0).permutation(X.shape[0])
    a = oracle.sa_forward(X, p.offsets, p.P, p.W_Q, p.W_K, p.W_V, p.eps)
    b = oracle.sa_forward(X[perm], p.offsets, p.P, p.W_Q, p.W_K, p.W_V, p.eps)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-12, atol=1e-14)


def test_single_prototype_is_the_mean():
    """k = 1: A = 1 everywhere, m = n and S = n/(n+eps) mean(X) W_V."""
    p = _prob(lengths=(23, 4), k=1, d=6)
    S, m, H = oracle.sa_forward(p.x_f64(), p.offsets, p.P, p.W_Q, p.W_K, p.W_V, p.eps)
    for u in range(p.B):
        X = p.x_f64(p.offsets[u], p.offsets[u + 1])
        n = X.shape[0]
        mean = X.mean(axis=0)
        want = np.array([sum(n / (n + p.eps) * mean[a] * p.W_V[a, b] for a in range(6))
                         for b in range(6)])
        np.testing.assert_allclose(m[u], [n], rtol=1e-14)
        np.testing.assert_allclose(S[u, 0], want, rtol=1e-11, atol=1e-14)
        np.testing.assert_allclose(H[u, 0], X.sum(axis=0), rtol=1e-12)


def test_zero_logits_give_uniform_assignment():
    """P = 0 makes every affinity zero; each token then spreads 1/k to every
    prototype and all sketch rows are equal."""
    p = _prob(lengths=(30,), k=4, d=5)
    P0 = np.zeros_like(p.P)
    X = p.x_f64()
    S, m, H = oracle.sa_forward(X, p.offsets, P0, p.W_Q, p.W_K, p.W_V, p.eps)
    np.testing.assert_allclose(m[0], 30 / 4, rtol=1e-14)
    row = (X.sum(axis=0) / 4) / (30 / 4 + p.eps) @ p.W_V.astype(np.float64)
    for j in range(4):
        np.testing.assert_allclose(S[0, j], row, rtol=1e-12)


def test_identical_tokens():
    """All tokens equal to x: every sketch row is x W_V m_j/(m_j+eps), for any P."""
    p = _prob(lengths=(17,), k=5, d=4, p_scale=5.0)
    x = np.array([0.3, -1.2, 0.7, 2.0])
    X = np.tile(x, (17, 1))
    S, m, H = oracle.sa_forward(X, p.offsets, p.P, p.W_Q, p.W_K, p.W_V, p.eps)
    xw = x @ p.W_V.astype(np.float64)
    for j in range(5):
        np.testing.assert_allclose(S[0, j], xw * m[0, j] / (m[0, j] + p.eps), rtol=1e-12)
    np.testing.assert_allclose(m[0].sum(), 17, rtol=1e-14)


def test_two_prototype_closed_form_fixes_scale_and_operand_order():
    """d = 2, W_Q = I, W_K = [[0,1],[0,0]] (not symmetric), x = e_1, P = [[0,s],[0,0]].
    x W_K = e_2, so S_11 = s/sqrt(2) and S_21 = 0 (eq. 6), hence
    A_11 = logistic(s/sqrt(2)).  A transposed W_K gives A_11 = 1/2 and a
    missing 1/sqrt(d) gives logistic(s)."""
    s = 1.7
    P = np.array([[0.0, s], [0.0, 0.0]])
    W_Q = np.eye(2)
    W_K = np.array([[0.0, 1.0], [0.0, 0.0]])
    W_V = np.array([[2.0, -1.0], [0.5, 3.0]])
    X = np.array([[1.0, 0.0]])
    A = oracle.assignment(X, P, W_Q, W_K)
    a1 = 1.0 / (1.0 + math.exp(-s / math.sqrt(2.0)))
    np.testing.assert_allclose(A[:, 0], [a1, 1 - a1], rtol=1e-14)
    S, m, H = oracle.sa_forward(X, [0, 1], P, W_Q, W_K, W_V, 0.25)
    np.testing.assert_allclose(m[0], [a1, 1 - a1], rtol=1e-14)
    np.testing.assert_allclose(H[0], [[a1, 0.0], [1 - a1, 0.0]], rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(S[0, 0], a1 / (a1 + 0.25) * np.array([2.0, -1.0]), rtol=1e-14)
    np.testing.assert_allclose(S[0, 1], (1 - a1) / (1 - a1 + 0.25) * np.array([2.0, -1.0]), rtol=1e-14)


def test_token_lse_closed_forms():
    """k = 1: the log-sum-exp is the single affinity; P = 0: ln k; two
    prototypes with the closed-form affinities above: ln(e^{s/sqrt 2} + 1)."""
    rng = np.random.default_rng(12)
    d = 5
    X = rng.standard_normal((9, d))
    P1, WQ, WK = rng.standard_normal((1, d)), rng.standard_normal((d, d)), rng.standard_normal((d, d))
    z = ((P1 @ WQ) @ (X @ WK).T / math.sqrt(d))[0]
    np.testing.assert_allclose(oracle.token_lse(X, P1, WQ, WK), z, rtol=1e-13)
    np.testing.assert_allclose(oracle.token_lse(X, np.zeros((7, d)), WQ, WK), np.log(7.0), rtol=1e-15)
    s = 1.7
    P = np.array([[0.0, s], [0.0, 0.0]])
    lse = oracle.token_lse(np.array([[1.0, 0.0]]), P, np.eye(2), np.array([[0.0, 1.0], [0.0, 0.0]]))
    np.testing.assert_allclose(lse, [math.log(math.exp(s / math.sqrt(2.0)) + 1.0)], rtol=1e-14)
    # the assignment is exp(S - lse)
    A = oracle.assignment(X, P1, WQ, WK)
    np.testing.assert_allclose(A, 1.0, rtol=1e-15)


def test_hard_assignment_limit():
    """Scaling every affinity up drives the prototype-wise softmax to a one-hot
    argmax, so H_j becomes the sum of the tokens whose best prototype is j and
    m_j their count (the k-means style assignment-aggregation of App. E)."""
    rng = np.random.default_rng(3)
    k, d, n = 4, 3, 40
    P = rng.standard_normal((k, d))
    W_Q, W_K = np.eye(d), np.eye(d)
    W_V = rng.standard_normal((d, d))
    X = rng.standard_normal((n, d))
    best = np.argmax(P @ X.T, axis=0)
    gap = np.sort(P @ X.T, axis=0)
    assert (gap[-1] - gap[-2]).min() > 1e-3
    scale = 1e6
    S, m, H = oracle.sa_forward(X, [0, n], P * scale, W_Q, W_K, W_V, 0.0)
    for j in range(k):
        sel = X[best == j]
        np.testing.assert_allclose(m[0, j], len(sel), atol=1e-9)
        np.testing.assert_allclose(H[0, j], sel.sum(axis=0), atol=1e-9)
        if len(sel):
            np.testing.assert_allclose(S[0, j], sel.mean(axis=0) @ W_V, rtol=1e-9, atol=1e-12)


def _brute(X, P, W_Q, W_K, W_V, eps):
    """Independent triple-loop evaluation in extended precision."""
    ld = np.longdouble
    k, d = P.shape
    n = X.shape[0]
    Q = [[sum(ld(P[j, a]) * ld(W_Q[a, b]) for a in range(d)) for b in range(d)] for j in range(k)]
    K = [[sum(ld(X[i, a]) * ld(W_K[a, b]) for a in range(d)) for b in range(d)] for i in range(n)]
    A = [[ld(0)] * n for _ in range(k)]
    for i in range(n):
        z = [sum(Q[j][b] * K[i][b] for b in range(d)) / np.sqrt(ld(d)) for j in range(k)]
        zmax = max(z)
        e = [np.exp(v - zmax) for v in z]
        tot = sum(e)
        for j in range(k):
            A[j][i] = e[j] / tot
    S = np.zeros((k, d), dtype=ld)
    m = np.zeros(k, dtype=ld)
    for j in range(k):
        m[j] = sum(A[j])
        Hj = [sum(A[j][i] * ld(X[i, b]) for i in range(n)) for b in range(d)]
        for c in range(d):
            S[j, c] = sum(Hj[b] * ld(W_V[b, c]) for b in range(d)) / (m[j] + ld(eps))
    return S, m


def test_brute_force_tiny():
    p = _prob(lengths=(6,), k=3, d=4, p_scale=2.0)
    X = p.x_f64()
    S, m, _ = oracle.sa_forward(X, p.offsets, p.P, p.W_Q, p.W_K, p.W_V, p.eps)
    Sb, mb = _brute(X, p.P, p.W_Q, p.W_K, p.W_V, p.eps)
    np.testing.assert_allclose(S[0], Sb.astype(np.float64), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(m[0], mb.astype(np.float64), rtol=1e-13)


def test_empty_user_gives_zero():
    p = _prob(lengths=(0, 5, 0), k=3, d=4)
    S, m, H = oracle.sa_forward(p.x_f64(), p.offsets, p.P, p.W_Q, p.W_K, p.W_V, p.eps)
    assert np.all(S[0] == 0) and np.all(m[0] == 0) and np.all(S[2] == 0)
    assert np.abs(S[1]).sum() > 0


# --------------------------------------------------------------------------
# backward: central finite differences of the forward
# --------------------------------------------------------------------------
def _loss(X, offsets, P, W_Q, W_K, W_V, eps, G, Gm):
    S, m, _ = oracle.sa_forward(X, offsets, P, W_Q, W_K, W_V, eps)
    out = float(np.sum(S * G))
    if Gm is not None:
        out += float(np.sum(m * Gm))
    return out


@pytest.mark.parametrize("with_dmass", [False, True])
def test_backward_matches_finite_differences(with_dmass):
    rng = np.random.default_rng(11)
    k, d = 3, 4
    offsets = np.array([0, 5, 5, 8])
    X = rng.standard_normal((8, d))
    P = rng.standard_normal((k, d)) * 1.5
    W_Q = rng.standard_normal((d, d))
    W_K = rng.standard_normal((d, d))
    W_V = rng.standard_normal((d, d))
    eps = 0.05
    G = rng.standard_normal((3, k, d))
    Gm = rng.standard_normal((3, k)) if with_dmass else None
    grads = oracle.sa_backward(X, offsets, P, W_Q, W_K, W_V, eps, G, Gm)
    params = [X, P, W_Q, W_K, W_V]
    h = 1e-6
    for which, (arr, g) in enumerate(zip(params, grads)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            save = arr[idx]
            arr[idx] = save + h
            lp = _loss(*params[:1], offsets, *params[1:], eps, G, Gm)
            arr[idx] = save - h
            lm = _loss(*params[:1], offsets, *params[1:], eps, G, Gm)
            arr[idx] = save
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=2e-6, atol=2e-7,
                                   err_msg=f"gradient {['dX','dP','dW_Q','dW_K','dW_V'][which]}")


def test_backward_permutes_with_tokens():
    rng = np.random.default_rng(5)
    k, d, n = 4, 3, 9
    X = rng.standard_normal((n, d))
    P, W_Q, W_K, W_V = (rng.standard_normal(s) for s in [(k, d), (d, d), (d, d), (d, d)])
    G = rng.standard_normal((1, k, d))
    perm = rng.permutation(n)
    a = oracle.sa_backward(X, [0, n], P, W_Q, W_K, W_V, 1e-6, G)
    b = oracle.sa_backward(X[perm], [0, n], P, W_Q, W_K, W_V, 1e-6, G)
    np.testing.assert_allclose(a[0][perm], b[0], rtol=1e-10, atol=1e-12)
    for x, y in zip(a[1:], b[1:]):
        np.testing.assert_allclose(x, y, rtol=1e-10, atol=1e-12)
