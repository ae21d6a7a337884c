"""Pins of the token-wise normalisation variant's oracle: closed forms, a
library attention routine in fp64, and the symmetry SA's prototype-wise
softmax does not have."""
import math

import numpy as np
import torch

import oracle
from sa_inputs import gauss, rng_for


def _case(seed, n=9, k=5, d=6):
    rng = rng_for(seed)
    return (gauss(rng, (n, d), 1.0).astype(np.float64), gauss(rng, (k, d), 1.0).astype(np.float64),
            gauss(rng, (d, d), 1 / math.sqrt(d)).astype(np.float64),
            gauss(rng, (d, d), 1 / math.sqrt(d)).astype(np.float64),
            gauss(rng, (d, d), 1 / math.sqrt(d)).astype(np.float64))


def test_rows_sum_to_one_and_mass_is_one():
    X, P, WQ, WK, WV = _case(1)
    S, m, H = oracle.tokenwise_user(X, P, WQ, WK, WV, 1e-6)
    np.testing.assert_allclose(m, 1.0, rtol=1e-14)
    # each prototype's H is a convex combination of the tokens: inside their bounding box
    assert np.all(H <= X.max(axis=0) + 1e-12) and np.all(H >= X.min(axis=0) - 1e-12)
    np.testing.assert_allclose(S, (H / (1 + 1e-6)) @ WV, rtol=1e-13)


def test_single_token_and_identical_tokens():
    X, P, WQ, WK, WV = _case(2, n=1)
    _, _, H = oracle.tokenwise_user(X, P, WQ, WK, WV, 0.0)
    np.testing.assert_allclose(H, np.repeat(X, P.shape[0], axis=0), rtol=1e-14)
    Xs = np.repeat(X, 7, axis=0)
    _, _, H7 = oracle.tokenwise_user(Xs, P, WQ, WK, WV, 0.0)
    np.testing.assert_allclose(H7, H, rtol=1e-13)


def test_matches_torch_attention_fp64():
    X, P, WQ, WK, WV = _case(3, n=40, k=7, d=8)
    Q = torch.from_numpy(P @ WQ)[None, None]
    K = torch.from_numpy(X @ WK)[None, None]
    V = torch.from_numpy(X)[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V)[0, 0].numpy()
    _, _, H = oracle.tokenwise_user(X, P, WQ, WK, WV, 0.0)
    np.testing.assert_allclose(H, ref, rtol=1e-12, atol=1e-13)


def test_prototypes_do_not_compete():
    """Token-wise: a prototype's output does not depend on the other prototypes
    (prototype-wise SA's does, through the softmax over prototypes)."""
    X, P, WQ, WK, WV = _case(4)
    _, _, H = oracle.tokenwise_user(X, P, WQ, WK, WV, 0.0)
    _, _, H0 = oracle.tokenwise_user(X, P[:1], WQ, WK, WV, 0.0)
    np.testing.assert_allclose(H[0], H0[0], rtol=1e-13)
    _, _, Hsa = oracle.sa_user(X, P, WQ, WK, WV, 0.0)
    _, _, Hsa0 = oracle.sa_user(X, P[:1], WQ, WK, WV, 0.0)
    assert np.max(np.abs(Hsa[0] - Hsa0[0])) > 1e-3


def test_batch_and_empty_user():
    X, P, WQ, WK, WV = _case(5, n=10)
    S, m, H = oracle.sa_forward_tokenwise(X, [0, 4, 4, 10], P, WQ, WK, WV, 1e-6)
    assert np.all(S[1] == 0) and np.all(m[1] == 0) and np.all(H[1] == 0)
    np.testing.assert_allclose(H[2], oracle.tokenwise_user(X[4:], P, WQ, WK, WV, 1e-6)[2], rtol=1e-14)
