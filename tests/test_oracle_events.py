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
