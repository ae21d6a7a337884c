"""GPU parity of sa_refine_forward (stacked SA refinement, Sec. 3.3) against the
fp64 oracle, through the C ABI.  Small ragged cases span several 128-token
tiles, a ragged tail and an empty user; one iteration, two iterations (the
second with per-user prototypes), with and without LN gains and biases; a
larger workload compares sampled users."""
import numpy as np
import pytest
import torch

import oracle
from helpers import compare, dev_f32, dev_x, tol_for
from sa_inputs import make_sa_problem, refine_layers, rng_for, sa_workload

pytestmark = pytest.mark.gpu

CASES = [
    # lengths, k, iterations, affine, seed
    ((130, 0, 700, 5), 256, 2, True, 1),
    ((385,), 128, 1, False, 2),
    ((2000, 129), 1024, 2, True, 3),
    ((1, 260, 3000), 512, 3, True, 4),
    ((0, 0), 128, 2, True, 5),            # no events at all: X^ = 0 in every iteration
]


def _layers_dev(layers):
    return [{k: (dev_f32(v) if v is not None else None) for k, v in L.items()} for L in layers]


def _run(lib, p, layers, users=None):
    X = dev_x(p.X, p.dtype)
    out = lib.sa_refine_forward(X, p.offsets, dev_f32(p.P), _layers_dev(layers), 1e-5)
    torch.cuda.synchronize()
    lib.poll_device_status()
    tol = tol_for(p.dtype)
    for u in (range(p.B) if users is None else users):
        lo, hi = int(p.offsets[u]), int(p.offsets[u + 1])
        ref = oracle.sa_refine_user(p.x_f64(lo, hi), p.P, layers, 1e-5)
        compare(f"sketch[{u}]", out[u], ref, tol)
    return out


@pytest.mark.parametrize("case", CASES, ids=[f"n{'-'.join(map(str, c[0]))}_k{c[1]}_it{c[2]}" for c in CASES])
def test_refine_small(lib, case):
    lengths, k, n_iter, affine, seed = case
    p = make_sa_problem(lengths, k, 128, "bf16", seed=100 + seed, x_kind="events")
    layers = refine_layers(rng_for(200 + seed), n_iter, 128, affine)
    _run(lib, p, layers)


def test_refine_deterministic(lib):
    p = make_sa_problem((900, 300), 256, 128, "bf16", seed=7, x_kind="events")
    layers = _layers_dev(refine_layers(rng_for(8), 2, 128))
    X = dev_x(p.X, p.dtype)
    a = lib.sa_refine_forward(X, p.offsets, dev_f32(p.P), layers)
    b = lib.sa_refine_forward(X, p.offsets, dev_f32(p.P), layers)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_refine_rejects_unsupported(lib):
    p = make_sa_problem((10,), 100, 128, "bf16", seed=9)
    with pytest.raises(lib.SAError):
        lib.sa_refine_forward(dev_x(p.X, p.dtype), p.offsets, dev_f32(p.P),
                              _layers_dev(refine_layers(rng_for(9), 1, 128)))


def test_refine_workload2_sampled(lib):
    """8 users of 20K-100K events, k = 512: users 0 and 7 against the oracle."""
    p = sa_workload(2)
    layers = refine_layers(rng_for(31), 2, p.d)
    _run(lib, p, layers, users=(0, 7))
