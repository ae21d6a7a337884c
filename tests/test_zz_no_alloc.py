"""sa_forward_noalloc: the SA forward for callers that cannot allocate device
memory (a memory pool they do not own, a host application that forbids device
allocations, work recorded once and replayed).  It uses the library's fixed
scratch array instead of a caller workspace.  This file is collected last, so
a run that stops at the first failure has already run every other test; it
also passes on its own in a fresh process.

Checked through the C ABI: two calls in a row against sa_forward and against
the oracle (same inputs, bf16 tolerance), with and without the caller's lse
buffer (without it the per-token log-sum-exp lives in the scratch array), and
sizes beyond the array's limits are refused up front."""
import numpy as np
import pytest
import torch

import oracle
from helpers import compare, sa_device_inputs, tol_for
from sa_inputs import make_sa_problem

pytestmark = pytest.mark.gpu


def _outputs(B, k, d, n, with_lse=True, device="cuda"):
    out = {"S": torch.empty(B, k, d, device=device), "mass": torch.empty(B, k, device=device),
           "H": torch.empty(B, k, d, device=device)}
    if with_lse:
        out["lse"] = torch.empty(max(n, 1), device=device)
    return out


CASES = [((1500, 0, 4321, 129), 256, 3.0, True), ((777, 64), 512, 6.0, True),
         ((2048, 5, 0, 3000), 384, 4.0, False)]


@pytest.mark.parametrize("case", CASES, ids=[f"k{c[1]}_lse{int(c[3])}" for c in CASES])
def test_noalloc_matches_sa_forward_and_oracle_twice(lib, case):
    lengths, k, scale, with_lse = case
    p = make_sa_problem(lengths, k, 128, "bf16", seed=101 + k, x_kind="events", p_scale=scale)
    dv = sa_device_inputs(p)
    offd = torch.from_numpy(p.offsets).cuda()
    ref = lib.sa_forward(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps,
                         offsets_dev=offd, want_H=True, want_lse=True)
    tol = tol_for("bf16")
    orc = [oracle.sa_user(p.x_f64(int(p.offsets[u]), int(p.offsets[u + 1])), p.P, p.W_Q, p.W_K,
                          p.W_V, p.eps) for u in range(p.B)]
    for call in range(2):
        out = _outputs(p.B, k, 128, p.n_total, with_lse)
        got = lib.sa_forward_noalloc(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"],
                                     dv["W_V"], p.eps, offsets_dev=offd, out=out)
        torch.cuda.synchronize()
        lib.poll_device_status()
        for name in ("S", "mass", "H"):
            compare(f"{name} call {call} k={k}", got[name], ref[name].double().cpu().numpy(), tol)
        for u, (S, m, H) in enumerate(orc):
            compare(f"S[{u}] vs oracle, call {call}", got["S"][u], S, tol)
            compare(f"mass[{u}] vs oracle, call {call}", got["mass"][u], m, tol)
            compare(f"H[{u}] vs oracle, call {call}", got["H"][u], H, tol)
        if with_lse:
            n = p.n_total
            err = (got["lse"][:n] - ref["lse"][:n]).abs().max().item()
            assert err <= 2e-2 * max(1.0, ref["lse"][:n].abs().max().item())


def test_noalloc_refuses_sizes_beyond_its_limits(lib):
    p = make_sa_problem((300,) * 9, 256, 128, "bf16", seed=5)     # 9 users > 8
    dv = sa_device_inputs(p)
    offd = torch.from_numpy(p.offsets).cuda()
    out = _outputs(p.B, 256, 128, p.n_total)
    with pytest.raises(lib.SAError) as ei:
        lib.sa_forward_noalloc(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"],
                               p.eps, offsets_dev=offd, out=out)
    assert ei.value.status == 2 and "users" in str(ei.value)
    q = make_sa_problem((300,), 1024, 128, "bf16", seed=6)        # k above 512
    dq = sa_device_inputs(q)
    with pytest.raises(lib.SAError):
        lib.sa_forward_noalloc(dq["X"], q.offsets, dq["P"], dq["W_Q"], dq["W_K"], dq["W_V"],
                               q.eps, offsets_dev=torch.from_numpy(q.offsets).cuda(),
                               out=_outputs(1, 1024, 128, 300))
    # without the caller's lse the per-token log-sum-exp needs 4 bytes per token of the
    # array: 8 users of 100K tokens at k = 512 do not fit (refused before any GPU work)
    r = make_sa_problem((300,) * 8, 512, 128, "bf16", seed=7)
    dr = sa_device_inputs(r)
    offs = np.arange(9, dtype=np.int64) * 100_000
    X = torch.zeros(int(offs[-1]), 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.SAError) as ei:
        lib.sa_forward_noalloc(X, offs, dr["P"], dr["W_Q"], dr["W_K"], dr["W_V"], r.eps,
                               offsets_dev=torch.from_numpy(offs).cuda(),
                               out=_outputs(8, 512, 128, int(offs[-1]), with_lse=False))
    assert ei.value.status == 2 and "scratch" in str(ei.value)
