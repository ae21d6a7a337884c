"""Pins of the event-embedding rows in the oracle (no GPU)."""
import numpy as np

import oracle
from sa_inputs import bf16_bits, sa_workload


def test_structured_tables_closed_form():
    """Item v's row holds v in column 0, action a's row holds a in column 1: the
    event row reads back its own ids (a swapped table or index fails)."""
    vocab, n_act, d = 50, 8, 4
    item = np.zeros((vocab, d)); item[:, 0] = np.arange(vocab); item[:, 2] = 1.0
    action = np.zeros((n_act, d)); action[:, 1] = np.arange(n_act); action[:, 3] = -1.0
    ids = np.array([3, 49, 0, 7, 7]); acts = np.array([0, 7, 2, 2, 5])
    x = oracle.event_rows(item, action, ids, acts)
    np.testing.assert_array_equal(x[:, 0], ids)
    np.testing.assert_array_equal(x[:, 1], acts)
    np.testing.assert_array_equal(x[:, 2], 1.0)
    np.testing.assert_array_equal(x[:, 3], -1.0)


def test_workload_rows_are_event_rows():
    """The SA workloads' X is the bf16 rounding of the event rows of the ids they drew."""
    p, tables, _ = sa_workload(2, users=1, vocab=4096, with_tables=True, keep_ids=True)
    n = min(5000, p.n_total)
    x = oracle.event_rows(tables.item, tables.action, p.item_ids[:n], p.action_ids[:n])
    np.testing.assert_array_equal(bf16_bits(x.astype(np.float32)), p.X[:n])


def _fused_weights(rng, d, wf):
    return (rng.standard_normal((2 * d, wf)) / np.sqrt(2 * d), rng.standard_normal((2 * d, wf)) / np.sqrt(2 * d),
            rng.standard_normal((wf, d)) / np.sqrt(wf))


def test_fused_rows_scalar_closed_form():
    """d = 1, w_f = 1: x = e + SiLU(u e + v a) (s e + t a) w, written out with the
    logistic function (a dropped residual, a swapped gate or table fails)."""
    import math
    item = np.array([[0.3], [-1.2], [2.0]]); action = np.array([[0.5], [-0.25]])
    u, v, s_, t, w = 0.7, -1.1, 0.4, 0.9, -0.6
    W1 = np.array([[u], [v]]); W3 = np.array([[s_], [t]]); W2 = np.array([[w]])
    ids = np.array([2, 0, 1, 2]); acts = np.array([1, 0, 1, 0])
    x = oracle.event_rows_fused(item, action, ids, acts, W1, W3, W2)
    for r, (i, k) in enumerate(zip(ids, acts)):
        e, a = item[i, 0], action[k, 0]
        g = u * e + v * a
        want = e + g / (1.0 + math.exp(-g)) * (s_ * e + t * a) * w
        assert abs(x[r, 0] - want) < 1e-15


def test_fused_rows_without_ffn_are_item_rows():
    """W2 = 0 removes the FFN term: x = e (the action enters only through the FFN)."""
    rng = np.random.default_rng(7)
    d, wf = 8, 16
    item, action = rng.standard_normal((20, d)), rng.standard_normal((8, d))
    W1, W3, _ = _fused_weights(rng, d, wf)
    ids, acts = rng.integers(0, 20, 30), rng.integers(0, 8, 30)
    x = oracle.event_rows_fused(item, action, ids, acts, W1, W3, np.zeros((wf, d)))
    np.testing.assert_array_equal(x, item[ids])


def test_fused_rows_match_torch_silu():
    """Against torch's SiLU and matmuls in fp64 on the concatenated features."""
    import torch
    rng = np.random.default_rng(8)
    d, wf = 16, 32
    item, action = rng.standard_normal((50, d)) * 0.02, rng.standard_normal((8, d)) * 0.02
    W1, W3, W2 = _fused_weights(rng, d, wf)
    ids, acts = rng.integers(0, 50, 64), rng.integers(0, 8, 64)
    x = oracle.event_rows_fused(item, action, ids, acts, W1, W3, W2)
    e = torch.from_numpy(item[ids]); a = torch.from_numpy(action[acts])
    z = torch.cat([e, a], dim=1)
    t1, t3, t2 = (torch.from_numpy(w) for w in (W1, W3, W2))
    want = e + (torch.nn.functional.silu(z @ t1) * (z @ t3)) @ t2
    np.testing.assert_allclose(x, want.numpy(), rtol=1e-12, atol=1e-15)


def test_fused_rows_depend_on_the_action():
    """The same item under two feedback types gives rows that differ by exactly the
    difference of the two FFN terms (eq. (20)'s purpose: one item, different contributions)."""
    rng = np.random.default_rng(9)
    d, wf = 8, 16
    item, action = rng.standard_normal((5, d)), rng.standard_normal((8, d))
    W1, W3, W2 = _fused_weights(rng, d, wf)
    x = oracle.event_rows_fused(item, action, [3, 3], [1, 6], W1, W3, W2)
    f = lambda z: oracle.swiglu_ffn(z[None, :], W1, W3, W2)[0]
    np.testing.assert_allclose(x[0] - x[1], f(np.concatenate([item[3], action[1]])) -
                               f(np.concatenate([item[3], action[6]])), rtol=1e-12, atol=1e-14)
    assert np.abs(x[0] - x[1]).max() > 1e-3
