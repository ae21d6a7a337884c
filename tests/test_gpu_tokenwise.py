"""GPU parity of sa_forward_tokenwise (the token-wise normalisation variant)
against the fp64 oracle, through the C ABI: ragged users including an empty
one, k not a multiple of 128, and sampled users of a large workload."""
import numpy as np
import pytest
import torch

import oracle
from helpers import compare, sa_device_inputs, tol_for
from sa_inputs import make_sa_problem, sa_workload

pytestmark = pytest.mark.gpu

CASES = [
    # lengths, k, kind, p_scale
    ((130, 0, 700, 5), 256, "events", 1.0),
    ((1, 2000), 100, "gauss", 4.0),
    ((3000, 129), 1024, "gauss", 2.0),
]


def _check(lib, p, users=None):
    dv = sa_device_inputs(p)
    out = lib.sa_forward_tokenwise(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps,
                                   want_H=True, want_bf16=True)
    torch.cuda.synchronize()
    lib.poll_device_status()
    tol = tol_for(p.dtype)
    for u in (range(p.B) if users is None else users):
        lo, hi = int(p.offsets[u]), int(p.offsets[u + 1])
        S, m, H = oracle.tokenwise_user(p.x_f64(lo, hi), p.P, p.W_Q, p.W_K, p.W_V, p.eps)
        compare(f"S[{u}]", out["S"][u], S, tol)
        compare(f"H[{u}]", out["H"][u], H, tol)
        assert torch.equal(out["mass"][u].cpu(), torch.from_numpy(m.astype(np.float32)))


@pytest.mark.parametrize("case", CASES, ids=[f"n{'-'.join(map(str, c[0]))}_k{c[1]}" for c in CASES])
def test_tokenwise_small(lib, case):
    lengths, k, kind, ps = case
    _check(lib, make_sa_problem(lengths, k, 128, "bf16", seed=40 + k, x_kind=kind, p_scale=ps))


def test_tokenwise_workload2_sampled(lib):
    _check(lib, sa_workload(2), users=(0, 7))
