"""Pins of the stacked refinement's backward in the oracle (no GPU): the reverse-mode
gradients of oracle.sa_refine_grads against central finite differences of the numpy
forward oracle.sa_refine, for every input and weight entry of a small ragged batch
(two iterations, affine LayerNorms, a user without events), and the permutation of
dX with the tokens."""
import numpy as np
import pytest

import oracle
from sa_inputs import gauss, refine_layers, rng_for


def _problem(seed=900, lengths=(5, 0, 3), k=3, d=4, n_iter=2):
    rng = rng_for(seed)
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    X = gauss(rng, (int(offsets[-1]), d), 1.0).astype(np.float64)
    P0 = gauss(rng, (k, d), 1.0).astype(np.float64)
    layers = [{n: (None if v is None else np.asarray(v, np.float64)) for n, v in L.items()}
              for L in refine_layers(rng, n_iter, d)]
    # logits of order one, so the softmax over prototypes is not flat
    for L in layers:
        L["W_Q"] = L["W_Q"] * 2.0
    dout = gauss(rng, (len(lengths), k, d), 1.0).astype(np.float64)
    return X, offsets, P0, layers, dout


def _loss(X, offsets, P0, layers, dout):
    return float((oracle.sa_refine(X, offsets, P0, layers) * dout).sum())


def _fd(f, a, h=1e-6):
    g = np.zeros_like(a)
    for idx in np.ndindex(a.shape):
        old = a[idx]
        a[idx] = old + h
        fp = f()
        a[idx] = old - h
        fm = f()
        a[idx] = old
        g[idx] = (fp - fm) / (2 * h)
    return g


def test_refine_grads_match_finite_differences():
    X, offsets, P0, layers, dout = _problem()
    got = oracle.sa_refine_grads(X, offsets, P0, layers, dout)
    f = lambda: _loss(X, offsets, P0, layers, dout)
    for name, arr, g in [("dX", X, got["dX"]), ("dP0", P0, got["dP0"])]:
        ref = _fd(f, arr)
        np.testing.assert_allclose(g, ref, rtol=1e-6, atol=1e-8, err_msg=name)
    for i, L in enumerate(layers):
        for name, v in L.items():
            if v is None:
                assert got["layers"][i][name] is None
                continue
            ref = _fd(f, v)
            np.testing.assert_allclose(got["layers"][i][name], ref, rtol=1e-6, atol=1e-8,
                                       err_msg=f"iteration {i} {name}")


def test_refine_grads_user_without_events_and_permutation():
    X, offsets, P0, layers, dout = _problem(seed=901, lengths=(6, 0, 4))
    got = oracle.sa_refine_grads(X, offsets, P0, layers, dout)
    # permuting a user's tokens permutes its rows of dX and leaves the rest unchanged
    perm = np.arange(X.shape[0])
    perm[0:6] = perm[0:6][::-1]
    got_p = oracle.sa_refine_grads(X[perm], offsets, P0, layers, dout)
    np.testing.assert_allclose(got_p["dX"], got["dX"][perm], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(got_p["dP0"], got["dP0"], rtol=1e-10, atol=1e-12)
    # the user without events still sends a gradient to P0 (its sketch is LN(LN(P0) + ...))
    only_empty = np.zeros_like(dout)
    only_empty[1] = dout[1]
    g1 = oracle.sa_refine_grads(X, offsets, P0, layers, only_empty)
    assert np.abs(g1["dP0"]).max() > 1e-3 and np.abs(g1["dX"]).max() == 0.0
