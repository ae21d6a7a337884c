"""Pins of the full STCA layer in the oracle (Sec. 5.1, eqs. (26)-(28)): the
history-side SwiGLU FFN before each layer's attention and the query-side
SwiGLU FFN after the W_O residual (no GPU)."""
import copy
import math

import numpy as np
import torch

import oracle
from sa_inputs import STCALayer, add_stca_ffns


def _layers(rng, n, D, heads, d_h, hist=True, query=True):
    out = []
    for _ in range(n):
        out.append(STCALayer(rng.standard_normal((heads, D, d_h)) / math.sqrt(D),
                             rng.standard_normal((heads, D, d_h)) / math.sqrt(D),
                             rng.standard_normal((heads, D, d_h)) / math.sqrt(D),
                             rng.standard_normal((heads * d_h, D)) / math.sqrt(D)))
    return add_stca_ffns(rng, out, D, hist, query)


def _torch_swiglu(x, W1, W3, W2):
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    return (torch.nn.functional.silu(x @ t(W1)) * (x @ t(W3))) @ t(W2)


def test_one_layer_matches_torch_silu_and_sdpa():
    """One head, one layer with both FFNs, written with torch's SiLU and
    scaled_dot_product_attention in fp64: the history FFN transforms the keys
    and values before the attention, the query FFN follows the W_O residual."""
    rng = np.random.default_rng(11)
    D, d_h, L, C = 10, 10, 23, 6
    lay = _layers(rng, 1, D, 1, d_h)[0]
    q = rng.standard_normal((C, D))
    X = rng.standard_normal((L, D))
    out = oracle.stca_branch(q, [0, C], X, [0], [L], [lay], 1, d_h)
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    Xh = t(X) + _torch_swiglu(t(X), lay.hist_W1, lay.hist_W3, lay.hist_W2)
    att = torch.nn.functional.scaled_dot_product_attention(
        (t(q) @ t(lay.W_Q[0]))[None, None], (Xh @ t(lay.W_K[0]))[None, None],
        (Xh @ t(lay.W_V[0]))[None, None])[0, 0]
    q1 = t(q) + att @ t(lay.W_O)
    ref = q1 + _torch_swiglu(q1, lay.q_W1, lay.q_W3, lay.q_W2)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_history_ffn_chains_across_layers():
    """Two layers = two one-layer calls, the second over the once-transformed
    keys: layer 2 attends over X2 = X1 + FFN_2(X1), X1 = X + FFN_1(X)."""
    rng = np.random.default_rng(12)
    D, heads, d_h, L, C = 8, 2, 4, 17, 5
    layers = _layers(rng, 2, D, heads, d_h)
    q = rng.standard_normal((C, D))
    X = rng.standard_normal((L, D))
    both = oracle.stca_branch(q, [0, C], X, [0], [L], layers, heads, d_h)
    l1 = copy.copy(layers[0])
    q1 = oracle.stca_branch(q, [0, C], X, [0], [L], [l1], heads, d_h)
    X1 = X + oracle.swiglu_ffn(X, l1.hist_W1, l1.hist_W3, l1.hist_W2)
    q2 = oracle.stca_branch(q1, [0, C], X1, [0], [L], [layers[1]], heads, d_h)
    np.testing.assert_allclose(both, q2, rtol=1e-12, atol=1e-12)


def test_zero_output_weights_remove_the_ffns():
    """W2 = 0 in both FFNs gives exactly the attention-only layer."""
    rng = np.random.default_rng(13)
    D, heads, d_h, L, C = 8, 2, 4, 9, 4
    layers = _layers(rng, 2, D, heads, d_h)
    plain = [STCALayer(l.W_Q, l.W_K, l.W_V, l.W_O) for l in layers]
    for l in layers:
        l.hist_W2 = np.zeros_like(l.hist_W2)
        l.q_W2 = np.zeros_like(l.q_W2)
    q = rng.standard_normal((C, D))
    X = rng.standard_normal((L, D))
    np.testing.assert_array_equal(oracle.stca_branch(q, [0, C], X, [0], [L], layers, heads, d_h),
                                  oracle.stca_branch(q, [0, C], X, [0], [L], plain, heads, d_h))


def test_key_permutation_invariance():
    """The history FFN acts on each row alone and the attention is a sum over
    keys, so permuting a user's keys changes nothing (up to rounding)."""
    rng = np.random.default_rng(14)
    D, heads, d_h, L, C = 8, 2, 4, 31, 6
    layers = _layers(rng, 2, D, heads, d_h)
    q = rng.standard_normal((C, D))
    X = rng.standard_normal((L, D))
    a = oracle.stca_branch(q, [0, C], X, [0], [L], layers, heads, d_h)
    b = oracle.stca_branch(q, [0, C], X[rng.permutation(L)], [0], [L], layers, heads, d_h)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def test_constant_keys_closed_form():
    """All keys equal to x: they stay equal through the history FFN, every
    softmax weight is uniform, and layer l adds concat_h(x_l W_V^h) W_O with
    x_l = x_{l-1} + FFN_l(x_{l-1}); the query FFN then acts on that sum."""
    rng = np.random.default_rng(15)
    D, heads, d_h, L = 8, 2, 4, 7
    layers = _layers(rng, 2, D, heads, d_h)
    q = rng.standard_normal((3, D))
    x = rng.standard_normal(D)
    out = oracle.stca_branch(q, [0, 3], np.tile(x, (L, 1)), [0], [L], layers, heads, d_h)
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    ref, xl = t(q), t(x)[None]
    for lay in layers:
        xl = xl + _torch_swiglu(xl, lay.hist_W1, lay.hist_W3, lay.hist_W2)
        o = torch.cat([xl @ t(lay.W_V[h]) for h in range(heads)], dim=1)
        ref = ref + o @ t(lay.W_O)
        ref = ref + _torch_swiglu(ref, lay.q_W1, lay.q_W3, lay.q_W2)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_reordering_with_ffns():
    """The eq. (24) reordering gives the same layers with both FFNs, over
    ragged users with an empty key range and a user without candidates."""
    rng = np.random.default_rng(16)
    D, heads, d_h = 8, 2, 4
    layers = _layers(rng, 2, D, heads, d_h)
    q = rng.standard_normal((9, D))
    kv = rng.standard_normal((40, D))
    cand = [0, 4, 4, 9, 9]
    kb, ke = [0, 10, 12, 12], [10, 12, 12, 40]
    a = oracle.stca_branch(q, cand, kv, kb, ke, layers, heads, d_h)
    b = oracle.stca_branch_reordered(q, cand, kv, kb, ke, layers, heads, d_h)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)
    # user 2 has candidates 4..8 and an empty key range: attention adds 0, the query FFN still acts
    q2 = q[4:9]
    for lay in layers:
        q2 = q2 + oracle.swiglu_ffn(q2, lay.q_W1, lay.q_W3, lay.q_W2)
    np.testing.assert_allclose(a[4:9], q2, rtol=1e-12, atol=1e-12)
