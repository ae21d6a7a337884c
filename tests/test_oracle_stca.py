"""Pins of the STCA and fusion oracle (no GPU)."""
import math

import numpy as np
import pytest
import torch

import oracle
from sa_inputs import STCALayer


def _layers(rng, n, D, heads, d_h, with_wo=True):
    out = []
    for _ in range(n):
        out.append(STCALayer(rng.standard_normal((heads, D, d_h)) / math.sqrt(D),
                             rng.standard_normal((heads, D, d_h)) / math.sqrt(D),
                             rng.standard_normal((heads, D, d_h)) / math.sqrt(D),
                             rng.standard_normal((heads * d_h, D)) / math.sqrt(D) if with_wo else None))
    return out


def _closed_form_const_keys(q, x, layers, heads, d_h):
    """With every key equal to x, every softmax weight is uniform and each
    head's output is x W_V^h whatever the query: each layer adds the same
    vector concat_h(x W_V^h) W_O to the query."""
    out = q.copy()
    for lay in layers:
        o = np.concatenate([x @ lay.W_V[h] for h in range(heads)])
        out = out + (o if lay.W_O is None else o @ lay.W_O)
    return out


@pytest.mark.parametrize("L", [1, 6])
def test_constant_keys_closed_form(L):
    rng = np.random.default_rng(1)
    D, heads, d_h = 8, 2, 4
    layers = _layers(rng, 2, D, heads, d_h)
    q = rng.standard_normal((5, D))
    x = rng.standard_normal(D)
    kv = np.tile(x, (L, 1))
    out = oracle.stca_branch(q, [0, 5], kv, [0], [L], layers, heads, d_h)
    for c in range(5):
        np.testing.assert_allclose(out[c], _closed_form_const_keys(q[c], x, layers, heads, d_h),
                                   rtol=1e-12, atol=1e-14)


def test_matches_torch_sdpa_fp64():
    """One head, one layer: the attention is torch's scaled_dot_product_attention
    on the projected query/keys/values, then W_O and the residual."""
    rng = np.random.default_rng(2)
    D, d_h, L, C = 12, 12, 30, 7
    lay = _layers(rng, 1, D, 1, d_h)
    q = rng.standard_normal((C, D))
    X = rng.standard_normal((L, D))
    out = oracle.stca_branch(q, [0, C], X, [0], [L], lay, 1, d_h)
    tq = torch.from_numpy(q @ lay[0].W_Q[0])[None, None]
    tk = torch.from_numpy(X @ lay[0].W_K[0])[None, None]
    tv = torch.from_numpy(X @ lay[0].W_V[0])[None, None]
    att = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0, 0].numpy()
    np.testing.assert_allclose(out, q + att @ lay[0].W_O, rtol=1e-12, atol=1e-13)


def test_multi_head_matches_sdpa_per_head():
    rng = np.random.default_rng(4)
    D, heads, d_h, L, C = 16, 4, 4, 19, 6
    lay = _layers(rng, 1, D, heads, d_h)
    q = rng.standard_normal((C, D))
    X = rng.standard_normal((L, D))
    out = oracle.stca_branch(q, [0, C], X, [0], [L], lay, heads, d_h)
    heads_out = []
    for h in range(heads):
        tq = torch.from_numpy(q @ lay[0].W_Q[h])[None, None]
        tk = torch.from_numpy(X @ lay[0].W_K[h])[None, None]
        tv = torch.from_numpy(X @ lay[0].W_V[h])[None, None]
        heads_out.append(torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0, 0].numpy())
    np.testing.assert_allclose(out, q + np.concatenate(heads_out, axis=1) @ lay[0].W_O,
                               rtol=1e-12, atol=1e-13)


def test_reordered_form_eq24_equals_direct():
    rng = np.random.default_rng(3)
    D, heads, d_h = 16, 4, 4
    layers = _layers(rng, 2, D, heads, d_h)
    cand = np.array([0, 3, 3, 8])
    q = rng.standard_normal((8, D))
    kv = rng.standard_normal((40, D))
    b, e = np.array([0, 10, 25]), np.array([10, 10, 40])
    a = oracle.stca_branch(q, cand, kv, b, e, layers, heads, d_h)
    r = oracle.stca_branch_reordered(q, cand, kv, b, e, layers, heads, d_h)
    np.testing.assert_allclose(a, r, rtol=1e-11, atol=1e-12)


def test_key_permutation_invariance_and_empty_range():
    rng = np.random.default_rng(6)
    D, heads, d_h = 8, 2, 4
    layers = _layers(rng, 2, D, heads, d_h, with_wo=False)
    q = rng.standard_normal((4, D))
    kv = rng.standard_normal((11, D))
    perm = rng.permutation(11)
    a = oracle.stca_branch(q, [0, 4], kv, [0], [11], layers, heads, d_h)
    b = oracle.stca_branch(q, [0, 4], kv[perm], [0], [11], layers, heads, d_h)
    np.testing.assert_allclose(a, b, rtol=1e-12)
    empty = oracle.stca_branch(q, [0, 4], kv, [3], [3], layers, heads, d_h)
    np.testing.assert_array_equal(empty, q)


def test_fuse_linear_blocks():
    rng = np.random.default_rng(8)
    D = 6
    zr, zu = rng.standard_normal((5, D)), rng.standard_normal((5, D))
    b = rng.standard_normal(D)
    I, O = np.eye(D), np.zeros((D, D))
    np.testing.assert_allclose(oracle.stca_fuse(zr, zu, np.vstack([I, I]), b), zr + zu + b, rtol=1e-15)
    np.testing.assert_allclose(oracle.stca_fuse(zr, zu, np.vstack([O, I])), zu, rtol=1e-15)
    np.testing.assert_allclose(oracle.stca_fuse(zr, zu, np.vstack([2 * I, O])), 2 * zr, rtol=1e-15)
