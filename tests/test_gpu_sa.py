"""GPU parity of sa_forward / sa_backward against the fp64 oracle, through the
C ABI (Python binding).  Small ragged cases span several 128-token tiles, a
ragged tail and empty users; the full-size workloads compare sampled users in
the same launch the benchmark times."""
import numpy as np
import pytest
import torch

import oracle
from helpers import compare, dev_f32, sa_device_inputs, tol_for
from sa_inputs import make_sa_problem, sa_workload

pytestmark = pytest.mark.gpu

SMALL = [
    # lengths, k, d, dtype, kind, p_scale
    ((0, 1, 127, 128, 129, 1000), 64, 64, "f32", "gauss", 1.0),
    ((3001, 0, 17), 100, 128, "f32", "gauss", 3.0),
    ((129, 513), 1, 64, "f32", "gauss", 1.0),
    ((130, 257, 1, 0), 256, 128, "bf16", "events", 1.0),
    ((1000, 0, 3000), 512, 128, "bf16", "gauss", 30.0),
    ((700, 5), 1024, 128, "bf16", "gauss", 8.0),
    ((64, 200), 2, 128, "bf16", "gauss", 5.0),
    ((333,), 384, 64, "bf16", "gauss", 4.0),
]


def _ids(c):
    return f"n{'-'.join(map(str, c[0]))}_k{c[1]}_d{c[2]}_{c[3]}_{c[4]}_x{c[5]:g}"


def _check_forward(lib, p, users=None):
    dv = sa_device_inputs(p)
    out = lib.sa_forward(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps,
                         want_H=True, want_bf16=True, want_lse=True)
    torch.cuda.synchronize()
    lib.poll_device_status()
    tol = tol_for(p.dtype)
    users = range(p.B) if users is None else users
    stats = {}
    for u in users:
        lo, hi = int(p.offsets[u]), int(p.offsets[u + 1])
        S, m, H = oracle.sa_user(p.x_f64(lo, hi), p.P, p.W_Q, p.W_K, p.W_V, p.eps)
        stats[f"S[{u}]"] = compare(f"S[{u}]", out["S"][u], S, tol)
        stats[f"mass[{u}]"] = compare(f"mass[{u}]", out["mass"][u], m, tol)
        stats[f"H[{u}]"] = compare(f"H[{u}]", out["H"][u], H, tol)
        if hi > lo:
            # the log-sum-exp is an absolute quantity: compare errors in units of 1
            lse = oracle.token_lse(p.x_f64(lo, hi), p.P, p.W_Q, p.W_K)
            err = np.abs(out["lse"][lo:hi].double().cpu().numpy() - lse)
            assert err.max() <= (1e-4 if p.dtype == "f32" else 2e-2) * max(1.0, np.abs(lse).max()), err.max()
        # each token spreads unit mass over the prototypes (eq. 7)
        tot = float(out["mass"][u].double().sum())
        assert abs(tot - (hi - lo)) <= (1e-5 if p.dtype == "f32" else 1e-3) * max(hi - lo, 1)
    Sb = out["S_bf16"].float()
    assert torch.all((Sb - out["S"]).abs() <= out["S"].abs() * 2.0 ** -8 + 1e-30)
    return out, stats


@pytest.mark.parametrize("case", SMALL, ids=[_ids(c) for c in SMALL])
def test_sa_forward_small(lib, case):
    lengths, k, d, dtype, kind, scale = case
    p = make_sa_problem(lengths, k, d, dtype, seed=17 + k + d, x_kind=kind, p_scale=scale)
    _check_forward(lib, p)


def test_sa_forward_zero_tokens(lib):
    p = make_sa_problem((0, 0), 128, 128, "bf16", seed=3)
    dv = sa_device_inputs(p)
    out = lib.sa_forward(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps,
                         want_H=True)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out["S"]) == 0 and torch.count_nonzero(out["mass"]) == 0
    assert torch.count_nonzero(out["H"]) == 0


def test_sa_forward_is_deterministic(lib):
    p = make_sa_problem((5000, 17, 2222), 256, 128, "bf16", seed=5, x_kind="events")
    dv = sa_device_inputs(p)
    a = lib.sa_forward(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps)
    b = lib.sa_forward(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps)
    torch.cuda.synchronize()
    assert torch.equal(a["S"], b["S"]) and torch.equal(a["mass"], b["mass"])


def test_sa_forward_token_permutation(lib):
    """Permuting a user's tokens leaves its sketch unchanged (up to rounding)."""
    p = make_sa_problem((4000,), 512, 128, "bf16", seed=9, p_scale=10.0)
    dv = sa_device_inputs(p)
    perm = torch.randperm(4000, generator=torch.Generator().manual_seed(0)).cuda()
    a = lib.sa_forward(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps)
    b = lib.sa_forward(dv["X"][perm].contiguous(), p.offsets, dv["P"], dv["W_Q"], dv["W_K"],
                       dv["W_V"], p.eps)
    compare("S perm", b["S"], a["S"].double().cpu().numpy(), tol_for("bf16"))


# --------------------------------------------------------------------------
# full-size workloads (sampled users, the benchmark's launch)
# --------------------------------------------------------------------------
@pytest.fixture(scope="module")
def workload_cache():
    return {}


def _workload(cache, cfg):
    if cfg not in cache:
        cache[cfg] = sa_workload(cfg)
    return cache[cfg]


def test_sa_forward_workload1_full(lib, workload_cache):
    _check_forward(lib, _workload(workload_cache, 1))


@pytest.mark.parametrize("cfg,users", [(2, (0, 7)), (3, (0, 31))])
def test_sa_forward_workload_sampled(lib, workload_cache, cfg, users):
    p = _workload(workload_cache, cfg)
    _check_forward(lib, p, users=users)


# --------------------------------------------------------------------------
# backward
# --------------------------------------------------------------------------
BWD = [
    ((0, 1, 129, 700), 64, 64, "f32", 2.0, False),
    ((300, 45), 100, 128, "f32", 3.0, True),
    ((513, 0, 128), 256, 128, "bf16", 5.0, True),
    ((1000,), 1024, 128, "bf16", 2.0, False),
    ((1500, 77), 512, 128, "bf16", 6.0, True),
]


def _run_backward(lib, p, dS, dmass=None, pass_lse=True):
    dv = sa_device_inputs(p)
    fwd = lib.sa_forward(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps,
                         want_H=True, want_lse=True)
    g = lib.sa_backward(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps,
                        fwd["H"], fwd["mass"], dev_f32(dS),
                        None if dmass is None else dev_f32(dmass),
                        fwd["lse"] if pass_lse else None)
    torch.cuda.synchronize()
    lib.poll_device_status()
    return fwd, g


@pytest.mark.parametrize("case", BWD, ids=[_ids(c[:5] + (c[4],)) + f"_dm{c[5]}" for c in BWD])
def test_sa_backward_small(lib, case):
    lengths, k, d, dtype, scale, with_dm = case
    p = make_sa_problem(lengths, k, d, dtype, seed=31 + k, p_scale=scale, with_grad=True)
    rng = np.random.default_rng(4)
    dmass = rng.standard_normal((p.B, k)).astype(np.float32) if with_dm else None
    _, g = _run_backward(lib, p, p.dS, dmass, pass_lse=(k != 100))
    ref = oracle.sa_backward(p.x_f64(), p.offsets, p.P, p.W_Q, p.W_K, p.W_V, p.eps, p.dS, dmass)
    tol = tol_for(dtype)
    for name, r in zip(["dX", "dP", "dW_Q", "dW_K", "dW_V"], ref):
        compare(name, g[name], r, tol)


def test_sa_backward_workload5_sampled(lib, workload_cache):
    """Full-size training step (64 users, mean 85K): dX rows of sampled users
    against the oracle; weight gradients are sums over users, so the full
    launch must equal the sum of one-user launches, and the one-user launches
    of sampled users must match the oracle."""
    p = _workload(workload_cache, 5)
    dv = sa_device_inputs(p)
    dS = dev_f32(p.dS)
    fwd = lib.sa_forward(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps,
                         want_H=True, want_lse=True)
    g = lib.sa_backward(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps,
                        fwd["H"], fwd["mass"], dS, None, fwd["lse"])
    torch.cuda.synchronize()
    tol = tol_for("bf16")
    names = ["dP", "dW_Q", "dW_K", "dW_V"]
    total = {n: torch.zeros_like(g[n], dtype=torch.float64) for n in names}
    for u in range(p.B):
        lo, hi = int(p.offsets[u]), int(p.offsets[u + 1])
        gu = lib.sa_backward(dv["X"][lo:hi], [0, hi - lo], dv["P"], dv["W_Q"], dv["W_K"],
                             dv["W_V"], p.eps, fwd["H"][u:u + 1].contiguous(),
                             fwd["mass"][u:u + 1].contiguous(), dS[u:u + 1].contiguous(), None,
                             fwd["lse"][lo:hi].clone())   # the ABI wants 16-byte aligned buffers
        for n in names:
            total[n] += gu[n].double()
        if u in (0, p.B - 1):
            ref = oracle.sa_backward(p.x_f64(lo, hi), [0, hi - lo], p.P, p.W_Q, p.W_K, p.W_V,
                                     p.eps, p.dS[u:u + 1])
            compare(f"dX[{u}]", g["dX"][lo:hi], ref[0], tol)
            for n, r in zip(names, ref[1:]):
                compare(f"{n}[{u}]", gu[n], r, tol)
    torch.cuda.synchronize()
    for n in names:
        # the same sums in another order: fp32 reassociation of sums with cancellation
        compare(f"{n} full = sum of users", g[n], total[n].cpu().numpy(), dict(max_rel=1e-3, mean_rel=1e-3))


@pytest.mark.parametrize("dtype,k", [("f32", 100), ("bf16", 256)])
def test_sa_backward_accumulate_over_user_groups(lib, dtype, k):
    """Weight gradients are sums over users: a first group through sa_backward and
    a second through sa_backward_accumulate equal one call over the whole batch,
    and each group's dX rows equal the whole batch's."""
    p = make_sa_problem((700, 0, 129, 1500, 60), k, 128, dtype, seed=77, with_grad=True)
    dv = sa_device_inputs(p)
    fwd = lib.sa_forward(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps,
                         want_H=True, want_lse=True)
    dS = dev_f32(p.dS)
    full = lib.sa_backward(dv["X"], p.offsets, dv["P"], dv["W_Q"], dv["W_K"], dv["W_V"], p.eps,
                           fwd["H"], fwd["mass"], dS, None, fwd["lse"])
    names = ["dP", "dW_Q", "dW_K", "dW_V"]
    acc = {n: torch.empty_like(full[n]) for n in names}
    off = p.offsets
    for i, (u0, u1) in enumerate(((0, 2), (2, p.B))):
        lo, hi = int(off[u0]), int(off[u1])
        g = lib.sa_backward(dv["X"][lo:hi], off[u0:u1 + 1] - off[u0], dv["P"], dv["W_Q"], dv["W_K"],
                            dv["W_V"], p.eps, fwd["H"][u0:u1], fwd["mass"][u0:u1], dS[u0:u1], None,
                            fwd["lse"][lo:hi].clone(), out=dict(acc), accumulate=(i > 0))
        torch.cuda.synchronize()
        np.testing.assert_allclose(g["dX"].float().cpu().numpy(), full["dX"][lo:hi].float().cpu().numpy(),
                                   rtol=1e-2, atol=1e-2 * float(full["dX"].float().abs().max()))
    for n in names:
        np.testing.assert_allclose(acc[n].cpu().numpy(), full[n].cpu().numpy(), rtol=1e-3,
                                   atol=1e-4 * float(full[n].abs().max()))
    ref = oracle.sa_backward(p.x_f64(), p.offsets, p.P, p.W_Q, p.W_K, p.W_V, p.eps, p.dS)
    for name, r in zip(["dX", "dP", "dW_Q", "dW_K", "dW_V"], ref):
        if name != "dX":
            compare(name, acc[name], r, tol_for(dtype))
