"""Pins of the STCA backward in the oracle: reverse-mode gradients of the full
STCA layer (Sec. 2.3 eq. (4), Sec. 5.1 eqs. (26)-(27)) against central finite
differences of the numpy forward, on tiny ragged problems (no GPU)."""
import math

import numpy as np
import pytest

import oracle
from sa_inputs import STCALayer, add_stca_ffns


def _layers(rng, n, D, heads, d_h, with_wo=True, hist=True, query=True):
    out = []
    for _ in range(n):
        out.append(STCALayer(rng.standard_normal((heads, D, d_h)) / math.sqrt(D),
                             rng.standard_normal((heads, D, d_h)) / math.sqrt(D),
                             rng.standard_normal((heads, D, d_h)) / math.sqrt(D),
                             rng.standard_normal((heads * d_h, D)) / math.sqrt(D) if with_wo else None))
    add_stca_ffns(rng, out, D, hist, query)
    # fp64 copies: a finite-difference step must not be rounded to fp32
    for lay in out:
        for name in oracle.STCA_WEIGHTS:
            if getattr(lay, name) is not None:
                setattr(lay, name, np.asarray(getattr(lay, name), np.float64))
    return out


PROBLEMS = [
    # D, heads, d_h, layers, W_O, history FFN, query FFN
    (6, 2, 3, 2, True, True, True),
    (4, 2, 2, 1, False, False, False),
    (6, 3, 2, 2, True, False, True),
    (4, 1, 4, 2, False, True, False),
]

# two users with overlapping key ranges, one user without candidates, one with no keys
CAND = [0, 3, 3, 5, 7]
KB, KE = [0, 4, 0, 9], [6, 9, 0, 11]


def _objective(q, kv, layers, heads, d_h, dout):
    return float((oracle.stca_branch(q, CAND, kv, KB, KE, layers, heads, d_h) * dout).sum())


def _fd(f, x, idx, h=1e-6):
    old = x[idx]
    x[idx] = old + h
    fp = f()
    x[idx] = old - h
    fm = f()
    x[idx] = old
    return (fp - fm) / (2 * h)


@pytest.mark.parametrize("prob", PROBLEMS, ids=[f"D{p[0]}_h{p[1]}_L{p[3]}_wo{p[4]}_hf{p[5]}_qf{p[6]}" for p in PROBLEMS])
def test_gradients_match_finite_differences(prob):
    D, heads, d_h, n_layers, wo, hist, query = prob
    rng = np.random.default_rng(100 + D + heads + n_layers)
    layers = _layers(rng, n_layers, D, heads, d_h, wo, hist, query)
    q = rng.standard_normal((CAND[-1], D))
    kv = rng.standard_normal((12, D))
    dout = rng.standard_normal((CAND[-1], D))
    g = oracle.stca_branch_grads(q, CAND, kv, KB, KE, layers, heads, d_h, dout)
    f = lambda: _objective(q, kv, layers, heads, d_h, dout)
    checks = [("dq", q, g["dq"]), ("dkv", kv, g["dkv"])]
    for li, lay in enumerate(layers):
        for name in oracle.STCA_WEIGHTS:
            w = getattr(lay, name)
            if w is not None:
                checks.append((f"layers[{li}].{name}", w, g["layers"][li][name]))
    for name, x, grad in checks:
        assert grad.shape == x.shape, name
        flat = list(np.ndindex(x.shape))
        for idx in [flat[i] for i in rng.choice(len(flat), size=min(6, len(flat)), replace=False)]:
            num = _fd(f, x, idx)
            assert abs(num - grad[idx]) <= 1e-6 * max(1.0, abs(num)), (name, idx, num, grad[idx])


def test_rows_outside_every_range_get_zero_and_shared_rows_sum():
    """Row 11 lies in no user's range: its gradient is exactly 0.  Rows 4-5 are keys
    of users 0 and 1: their gradient is the sum of the two users' contributions."""
    D, heads, d_h = 4, 2, 2
    rng = np.random.default_rng(7)
    layers = _layers(rng, 1, D, heads, d_h, hist=False, query=False)
    q = rng.standard_normal((CAND[-1], D))
    kv = rng.standard_normal((12, D))
    dout = rng.standard_normal((CAND[-1], D))
    cand, kb, ke = [0, 3, 5], [0, 4], [6, 9]
    g = oracle.stca_branch_grads(q[:5], cand, kv, kb, ke, layers, heads, d_h, dout[:5])
    assert np.all(g["dkv"][9:] == 0.0)
    g0 = oracle.stca_branch_grads(q[:3], [0, 3], kv, [0], [6], layers, heads, d_h, dout[:3])
    g1 = oracle.stca_branch_grads(q[3:5], [0, 2], kv, [4], [9], layers, heads, d_h, dout[3:5])
    np.testing.assert_allclose(g["dkv"], g0["dkv"] + g1["dkv"], rtol=1e-12, atol=1e-14)


def test_query_without_keys_or_query_ffn_passes_the_gradient_through():
    """A user whose key range is empty adds 0 in every attention; without query FFNs
    its output is its query, so dq = dout on its rows, exactly, and it contributes
    nothing to the attention weights' gradients."""
    D, heads, d_h = 6, 2, 3
    rng = np.random.default_rng(9)
    layers = _layers(rng, 2, D, heads, d_h, query=False)
    q = rng.standard_normal((4, D))
    kv = rng.standard_normal((5, D))
    dout = rng.standard_normal((4, D))
    g = oracle.stca_branch_grads(q, [0, 4], kv, [2], [2], layers, heads, d_h, dout)
    np.testing.assert_array_equal(g["dq"], dout)
    assert np.all(g["dkv"] == 0.0)
    for lg in g["layers"]:
        for name in ("W_Q", "W_K", "W_V", "W_O", "hist_W1", "hist_W3", "hist_W2"):
            assert np.all(lg[name] == 0.0), name
