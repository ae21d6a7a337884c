"""GPU parity of stca_forward and stca_fuse against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from helpers import compare, dev_f32, dev_x, stca_branch_dev, stca_layers_dev, tol_for
from sa_inputs import make_stca_problem, stca_workload

pytestmark = pytest.mark.gpu

SMALL = [
    # B, cands, recent lengths, k, heads, d_h, layers, dtype, with W_O
    (3, (5, 0, 37), (1, 200, 130), 64, 4, 32, 2, "bf16", True),
    (2, (129, 3), (1000, 0), 16, 4, 32, 1, "bf16", False),
    (4, (1, 2, 3, 300), (40, 41, 42, 257), 128, 2, 64, 2, "f32", True),
    (1, (64,), (5000,), 1024, 4, 32, 2, "bf16", True),
]


def _run_branch(lib, prob, which):
    br = prob.recent if which == "recent" else prob.sketch
    layers = prob.layers_r if which == "recent" else prob.layers_u
    q, kv = stca_branch_dev(br, prob.dtype)
    out = lib.stca_forward(q, br.cand_offsets, kv, br.kv_begin, br.kv_end,
                           stca_layers_dev(layers), prob.heads, prob.d_h)
    torch.cuda.synchronize()
    return out


def _ref_branch(prob, which, users=None):
    br = prob.recent if which == "recent" else prob.sketch
    layers = prob.layers_r if which == "recent" else prob.layers_u
    q = prob.widen(br.q)
    kv = prob.widen(br.kv)
    if users is None:
        return oracle.stca_branch(q, br.cand_offsets, kv, br.kv_begin, br.kv_end, layers,
                                  prob.heads, prob.d_h)
    res = {}
    for u in users:
        c0, c1 = int(br.cand_offsets[u]), int(br.cand_offsets[u + 1])
        res[u] = oracle.stca_branch(q[c0:c1], [0, c1 - c0], kv, br.kv_begin[u:u + 1],
                                    br.kv_end[u:u + 1], layers, prob.heads, prob.d_h)
    return res


@pytest.mark.parametrize("case", SMALL, ids=[f"B{c[0]}_k{c[3]}_h{c[4]}_{c[7]}_wo{c[8]}" for c in SMALL])
@pytest.mark.parametrize("which", ["recent", "sketch"])
def test_stca_small(lib, case, which):
    B, cands, rec, k, heads, d_h, n_layers, dtype, wo = case
    prob = make_stca_problem(B, cands, rec, k, 128, heads, d_h, n_layers, dtype, seed=77 + k,
                             with_wo=wo)
    got = _run_branch(lib, prob, which)
    compare(f"stca {which}", got, _ref_branch(prob, which), tol_for(dtype))


def test_stca_empty_key_range_keeps_query(lib):
    prob = make_stca_problem(2, (3, 4), (10, 10), 8, 128, 4, 32, 2, "bf16", seed=5)
    br = prob.recent
    q, kv = stca_branch_dev(br, "bf16")
    kb = np.array([0, 10]); ke = np.array([0, 10])
    out = lib.stca_forward(q, br.cand_offsets, kv, kb, ke, stca_layers_dev(prob.layers_r), 4, 32)
    torch.cuda.synchronize()
    assert torch.equal(out[:3], q[:3].float())


@pytest.fixture(scope="module")
def w4():
    return stca_workload()


@pytest.mark.parametrize("which", ["recent", "sketch"])
def test_stca_workload4_sampled(lib, w4, which):
    got = _run_branch(lib, w4, which)
    br = w4.recent if which == "recent" else w4.sketch
    for u, ref in _ref_branch(w4, which, users=(0, 15)).items():
        c0, c1 = int(br.cand_offsets[u]), int(br.cand_offsets[u + 1])
        compare(f"stca {which}[{u}]", got[c0:c1], ref, tol_for("bf16"))


def test_stca_fuse(lib):
    rng = np.random.default_rng(2)
    C, D = 300, 128
    zr, zu = rng.standard_normal((C, D)), rng.standard_normal((C, D))
    W = rng.standard_normal((2 * D, D)) / np.sqrt(2 * D)
    b = rng.standard_normal(D)
    got = lib.stca_fuse(dev_f32(zr), dev_f32(zu), dev_f32(W), dev_f32(b))
    nob = lib.stca_fuse(dev_f32(zr), dev_f32(zu), dev_f32(W))
    torch.cuda.synchronize()
    f32 = lambda a: a.astype(np.float32).astype(np.float64)
    compare("fuse", got, oracle.stca_fuse(f32(zr), f32(zu), f32(W), f32(b)), tol_for("f32"))
    compare("fuse no bias", nob, oracle.stca_fuse(f32(zr), f32(zu), f32(W)), tol_for("f32"))
