"""sa_forward_noalloc: the SA forward for callers that cannot allocate device
memory (a memory pool they do not own, a host application that forbids device
allocations, work recorded once and replayed).  It uses the library's fixed
scratch array instead of a caller workspace.  This file is collected last, so
a run that stops at the first failure has already run every other test; it
also passes on its own in a fresh process.

Checked through the C ABI: two calls in a row against sa_forward (same inputs,
bf16 tolerance), and sizes beyond the array's limits are refused up front."""
import numpy as np
import pytest
import torch

from helpers import compare, sa_device_inputs, tol_for
from sa_inputs import make_sa_problem

pytestmark = pytest.mark.gpu


def _outputs(B, k, d, n, device="cuda"):
    return {"S": torch.empty(B, k, d, device=device), "mass": torch.empty(B, k, device=device),
            "H": torch.empty(B, k, d, device=device), "lse": torch.empty(max(n, 1), device=device)}


def test_noalloc_matches_sa_forward_twice(lib):
    cases = [((1500, 0, 4321, 129), 256, 3.0), ((777, 64), 512, 6.0)]
    for lengths, k, scale in cases:
        p = make_sa_problem(lengths, k, 128, "bf16", seed=101 + k, x_kind="events", p_scale=scale)
        dv = sa_device_inputs(p)
        offd = torch.from_numpy(p.offsets).cuda()
        ref = lib.sa_forward(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps,
                             offsets_dev=offd, want_H=True, want_lse=True)
        for call in range(2):
            out = _outputs(p.B, k, 128, p.n_total)
            got = lib.sa_forward_noalloc(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"],
                                         dv["W_V"], p.eps, offsets_dev=offd, out=out)
            torch.cuda.synchronize()
            lib.poll_device_status()
            tol = tol_for("bf16")
            for name in ("S", "mass", "H"):
                compare(f"{name} call {call} k={k}", got[name], ref[name].double().cpu().numpy(), tol)
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
