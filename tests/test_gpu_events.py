"""GPU checks of sa_gather_events (the events' rows built on the device from item
and action ids), through the C ABI: bit-exact rows, the out-of-range guard, and the
SA forward over gathered rows against the oracle on the exact event rows."""
import numpy as np
import pytest
import torch

import oracle
from helpers import compare, dev_f32, tol_for
from sa_inputs import bf16_bits, bf16_to_f32, bf16_to_f64, event_problem, make_sa_problem

pytestmark = pytest.mark.gpu


def _dev(item, action, ids, acts):
    t = lambda b: torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16)
    return t(item), t(action), torch.from_numpy(ids).cuda(), torch.from_numpy(acts).cuda()


@pytest.mark.parametrize("n,vocab", [(1, 10), (1000, 4096), (100_003, 1_000_000)])
def test_gather_bit_exact(lib, n, vocab):
    item, action, ids, acts = event_problem(n, vocab, 128, seed=700 + n)
    X = lib.sa_gather_events(*_dev(item, action, ids, acts))
    torch.cuda.synchronize()
    lib.poll_device_status()
    ref = bf16_bits(bf16_to_f32(item)[ids] + bf16_to_f32(action)[acts])
    got = X.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_gather_out_of_range_id_zeroes_the_row_and_reports(lib):
    item, action, ids, acts = event_problem(64, 100, 128, seed=710)
    ids = ids.copy(); acts = acts.copy()
    ids[5] = 100          # one past the table
    acts[9] = 8           # one past the action table
    X = lib.sa_gather_events(*_dev(item, action, ids, acts))
    torch.cuda.synchronize()
    with pytest.raises(lib.SAError):
        lib.poll_device_status()
    lib.poll_device_status()   # the word was cleared
    got = X.float().cpu().numpy()
    assert np.all(got[5] == 0) and np.all(got[9] == 0)
    ok = [i for i in range(64) if i not in (5, 9)]
    ref = bf16_to_f32(bf16_bits(bf16_to_f32(item)[ids[ok]] + bf16_to_f32(action)[acts[ok]]))
    np.testing.assert_array_equal(got[ok], ref)


def test_sa_forward_over_gathered_rows(lib):
    """Three users (one empty) of events: gather, then sa_forward; the oracle runs on
    the exact event rows (the bf16 rounding of each row counts as error)."""
    lengths = (3000, 0, 1300)
    n = sum(lengths)
    item, action, ids, acts = event_problem(n, 50_000, 128, seed=720)
    p = make_sa_problem(lengths, 256, 128, "bf16", seed=721)
    X = lib.sa_gather_events(*_dev(item, action, ids, acts))
    out = lib.sa_forward(X, p.offsets, dev_f32(p.P), dev_f32(p.W_Q), dev_f32(p.W_K), dev_f32(p.W_V), p.eps)
    torch.cuda.synchronize()
    rows = oracle.event_rows(bf16_to_f64(item), bf16_to_f64(action), ids, acts)
    S, mass = oracle.sa_forward(rows, p.offsets, p.P, p.W_Q, p.W_K, p.W_V, p.eps)[:2]
    compare("S", out["S"], S, tol_for("bf16"))
    compare("mass", out["mass"], mass, tol_for("bf16"))


@pytest.mark.parametrize("n,vocab,scale", [(1, 10, 1.0), (1000, 4096, 1.0), (5003, 4096, 40.0),
                                           (100_003, 1_000_000, 1.0)])
def test_fused_rows_against_the_oracle(lib, n, vocab, scale):
    """sa_gather_events_fused (eq. (20)) against oracle.event_rows_fused on the same
    bf16 tables and fp32 weights; scale 40 makes the FFN term larger than the item
    row itself (with the workloads' std-0.02 tables it is a few percent of it), and
    the FFN term alone is compared as well."""
    from sa_inputs import event_ffn_weights, rng_for
    item, action, ids, acts = event_problem(n, vocab, 128, seed=730 + n)
    W1, W3, W2 = event_ffn_weights(rng_for(731 + n), 128, scale=scale)
    X = lib.sa_gather_events_fused(*_dev(item, action, ids, acts), dev_f32(W1), dev_f32(W3), dev_f32(W2))
    torch.cuda.synchronize()
    lib.poll_device_status()
    ref = oracle.event_rows_fused(bf16_to_f64(item), bf16_to_f64(action), ids, acts, W1, W3, W2)
    compare("fused rows", X, ref, tol_for("bf16"))
    e = bf16_to_f64(item)[ids]
    if scale > 1.0:
        compare("FFN term", X.double().cpu().numpy() - e, ref - e, tol_for("bf16"))


def test_fused_rows_out_of_range_zero_and_report(lib):
    from sa_inputs import event_ffn_weights, rng_for
    item, action, ids, acts = event_problem(300, 100, 128, seed=740)
    ids = ids.copy(); acts = acts.copy()
    ids[7] = -1
    ids[130] = 100
    acts[200] = 8
    W1, W3, W2 = event_ffn_weights(rng_for(741), 128)
    X = lib.sa_gather_events_fused(*_dev(item, action, ids, acts), dev_f32(W1), dev_f32(W3), dev_f32(W2))
    torch.cuda.synchronize()
    with pytest.raises(lib.SAError) as ei:
        lib.poll_device_status()
    assert ei.value.status == 1
    got = X.double().cpu().numpy()
    bad = (7, 130, 200)
    assert all(np.all(got[i] == 0) for i in bad)
    ok = [i for i in range(300) if i not in bad]
    ref = oracle.event_rows_fused(bf16_to_f64(item), bf16_to_f64(action), ids[ok], acts[ok], W1, W3, W2)
    compare("fused rows beside the bad ones", got[ok], ref, tol_for("bf16"))
