"""GPU parity of stca_forward_full (the full STCA layer of Sec. 5.1, eqs.
(26)-(28): history-side SwiGLU FFN before each attention, query-side SwiGLU
FFN after the W_O residual) against the fp64 oracle, through the C ABI.
Small ragged cases cover empty key ranges, users without candidates, FFNs on
some layers only, both dtypes and both branches; the sketch branch (N(0,1)
rows) and a rescaled recent history make the FFN terms as large as the rows
themselves; a config-4-sized problem compares sampled users."""
import numpy as np
import pytest
import torch

import oracle
from helpers import compare, dev_f32, dev_x, tol_for
from sa_inputs import add_stca_ffns, bf16_bits, make_stca_problem, rng_for, stca_workload

pytestmark = pytest.mark.gpu

FFN_KEYS = ("hist_W1", "hist_W3", "hist_W2", "q_W1", "q_W3", "q_W2")


def _layers_dev(layers):
    out = []
    for L in layers:
        d = dict(W_Q=dev_f32(L.W_Q), W_K=dev_f32(L.W_K), W_V=dev_f32(L.W_V),
                 W_O=None if L.W_O is None else dev_f32(L.W_O))
        for k in FFN_KEYS:
            v = getattr(L, k)
            d[k] = None if v is None else dev_f32(v)
        out.append(d)
    return out


def _with_ffns(prob, seed, hist=True, query=True, only_layer=None):
    rng = rng_for(seed)
    for layers in (prob.layers_r, prob.layers_u):
        for i, lay in enumerate(layers):
            if only_layer is None or i == only_layer:
                add_stca_ffns(rng, [lay], prob.D, hist, query)
    return prob


def _branch(prob, which):
    br = prob.recent if which == "recent" else prob.sketch
    layers = prob.layers_r if which == "recent" else prob.layers_u
    return br, layers


def _run(lib, prob, which, kv=None):
    br, layers = _branch(prob, which)
    kv = br.kv if kv is None else kv
    out = lib.stca_forward_full(dev_x(br.q, prob.dtype), br.cand_offsets, dev_x(kv, prob.dtype),
                                br.kv_begin, br.kv_end, _layers_dev(layers), prob.heads, prob.d_h)
    torch.cuda.synchronize()
    lib.poll_device_status()
    return out


def _ref(prob, which, kv=None, users=None):
    br, layers = _branch(prob, which)
    q = prob.widen(br.q)
    kvf = prob.widen(br.kv if kv is None else kv)
    if users is None:
        return oracle.stca_branch(q, br.cand_offsets, kvf, br.kv_begin, br.kv_end, layers,
                                  prob.heads, prob.d_h)
    res = {}
    for u in users:
        c0, c1 = int(br.cand_offsets[u]), int(br.cand_offsets[u + 1])
        res[u] = oracle.stca_branch(q[c0:c1], [0, c1 - c0], kvf, br.kv_begin[u:u + 1],
                                    br.kv_end[u:u + 1], layers, prob.heads, prob.d_h)
    return res


SMALL = [
    # B, cands, recent lengths, k, heads, d_h, layers, dtype, FFNs ("both", "hist", "query", "first")
    (3, (5, 0, 37), (1, 200, 130), 64, 4, 32, 2, "bf16", "both"),
    (2, (129, 3), (1000, 0), 16, 4, 32, 1, "bf16", "hist"),
    (4, (1, 2, 3, 300), (40, 41, 42, 257), 128, 2, 64, 2, "f32", "both"),
    (2, (7, 9), (300, 129), 128, 4, 32, 2, "bf16", "query"),
    (2, (7, 9), (300, 129), 256, 4, 32, 2, "bf16", "first"),
    (1, (64,), (5000,), 1024, 4, 32, 2, "bf16", "both"),
    (3, (4, 4, 4), (10, 0, 77), 32, 4, 32, 2, "f32", "first"),
]


def _make(case, seed):
    B, cands, rec, k, heads, d_h, n_layers, dtype, ffn = case
    prob = make_stca_problem(B, cands, rec, k, 128, heads, d_h, n_layers, dtype, seed=seed)
    if ffn == "first":
        return _with_ffns(prob, seed + 1, only_layer=0)
    return _with_ffns(prob, seed + 1, hist=ffn in ("both", "hist"), query=ffn in ("both", "query"))


@pytest.mark.parametrize("case", SMALL, ids=[f"B{c[0]}_k{c[3]}_{c[7]}_{c[8]}" for c in SMALL])
@pytest.mark.parametrize("which", ["recent", "sketch"])
def test_stca_full_small(lib, case, which):
    prob = _make(case, 300 + case[3])
    e = compare(f"stca_full {which}", _run(lib, prob, which), _ref(prob, which), tol_for(prob.dtype))
    print(f"stca_full {which} {case}: {e}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_stca_full_large_history_values(lib, dtype):
    """The recent rows scaled to unit size, so the history FFN's output is as
    large as the row it is added to (the event embeddings alone give an FFN
    term of about 1% of the row)."""
    prob = _make((2, (40, 33), (700, 1300), 64, 4, 32, 2, dtype, "both"), 410)
    kv = prob.widen(prob.recent.kv) * 40.0
    kv_in = bf16_bits(kv.astype(np.float32)) if dtype == "bf16" else kv.astype(np.float32)
    got = _run(lib, prob, "recent", kv=kv_in)
    ref = _ref(prob, "recent", kv=kv_in)
    print("stca_full recent x40", dtype, compare("stca_full recent x40", got, ref, tol_for(dtype)))


def test_stca_full_all_ranges_empty(lib):
    """No key rows at all with history FFNs: every attention adds 0 and only the
    query FFNs act."""
    prob = _make((2, (3, 4), (10, 10), 8, 4, 32, 2, "bf16", "both"), 420)
    br, layers = _branch(prob, "recent")
    kb = np.zeros(2, np.int64); ke = np.zeros(2, np.int64)
    out = lib.stca_forward_full(dev_x(br.q, "bf16"), br.cand_offsets, dev_x(br.kv, "bf16"), kb, ke,
                                _layers_dev(layers), prob.heads, prob.d_h)
    torch.cuda.synchronize()
    ref = oracle.stca_branch(prob.widen(br.q), br.cand_offsets, prob.widen(br.kv), kb, ke, layers,
                             prob.heads, prob.d_h)
    compare("stca_full no keys", out, ref, tol_for("f32"))


def test_stca_full_without_ffns_equals_stca_forward(lib):
    prob = make_stca_problem(3, (5, 0, 37), (1, 200, 130), 64, 128, 4, 32, 2, "bf16", seed=430)
    for which in ("recent", "sketch"):
        br, layers = _branch(prob, which)
        q, kv = dev_x(br.q, "bf16"), dev_x(br.kv, "bf16")
        a = lib.stca_forward_full(q, br.cand_offsets, kv, br.kv_begin, br.kv_end, _layers_dev(layers),
                                  prob.heads, prob.d_h)
        b = lib.stca_forward(q, br.cand_offsets, kv, br.kv_begin, br.kv_end, _layers_dev(layers),
                             prob.heads, prob.d_h)
        torch.cuda.synchronize()
        assert torch.equal(a, b)


def test_stca_full_deterministic(lib):
    prob = _make((2, (130, 7), (900, 300), 64, 4, 32, 2, "bf16", "both"), 440)
    a = _run(lib, prob, "recent")
    b = _run(lib, prob, "recent")
    assert torch.equal(a, b)


def test_stca_full_rejects_partial_ffn(lib):
    prob = _make((1, (3,), (10,), 8, 4, 32, 1, "bf16", "both"), 450)
    br, layers = _branch(prob, "recent")
    L = _layers_dev(layers)
    L[0]["hist_W3"] = None
    with pytest.raises(lib.SAError):
        lib.stca_forward_full(dev_x(br.q, "bf16"), br.cand_offsets, dev_x(br.kv, "bf16"), br.kv_begin,
                              br.kv_end, L, prob.heads, prob.d_h)


@pytest.fixture(scope="module")
def w4full():
    prob = stca_workload()
    return _with_ffns(prob, 460)


@pytest.mark.parametrize("which", ["recent", "sketch"])
def test_stca_full_workload4_sampled(lib, w4full, which):
    """16 users x 512 candidates, 10K suffixes and 1024-row sketches, two full
    layers: users 0 and 15 against the oracle."""
    got = _run(lib, w4full, which)
    br, _ = _branch(w4full, which)
    for u, ref in _ref(w4full, which, users=(0, 15)).items():
        c0, c1 = int(br.cand_offsets[u]), int(br.cand_offsets[u + 1])
        print(which, u, compare(f"stca_full {which}[{u}]", got[c0:c1], ref, tol_for("bf16")))


def test_stca_full_reports_fp16_range(lib):
    """bf16 rows beyond the fp16 range (|x| > 65504) cannot be held by the full
    layer's fp16 key copy: the call's status poll reports SA_ERR_UNSUPPORTED,
    and the next call on normal rows runs clean."""
    prob = _make((2, (5, 6), (50, 70), 16, 4, 32, 1, "bf16", "hist"), 470)
    br, layers = _branch(prob, "sketch")
    big = bf16_bits((prob.widen(br.kv) * 1e5).astype(np.float32))
    lib.stca_forward_full(dev_x(br.q, "bf16"), br.cand_offsets, dev_x(big, "bf16"), br.kv_begin, br.kv_end,
                          _layers_dev(layers), prob.heads, prob.d_h)
    torch.cuda.synchronize()
    with pytest.raises(lib.SAError) as ei:
        lib.poll_device_status()
    assert ei.value.status == 2 and "fp16" in str(ei.value)
    out = _run(lib, prob, "sketch")
    compare("stca_full after a range error", out, _ref(prob, "sketch"), tol_for("bf16"))
