"""GPU parity of sa_refine_backward (the backward of the stacked SA refinement,
Sec. 3.3, eqs. (12)-(16)) against the oracle's reverse-mode gradients in fp64,
through the C ABI: dX, dP0 and every parameter gradient of every iteration,
on ragged batches with an empty user, one to three iterations, with and
without LayerNorm gains and biases, and a user of a few thousand events at
k = 1024."""
import numpy as np
import pytest
import torch

import oracle
from helpers import compare, dev_f32, dev_x, tol_for
from sa_inputs import gauss, make_sa_problem, refine_layers, rng_for

pytestmark = pytest.mark.gpu

CASES = [
    # lengths, k, iterations, affine, prototype scale, seed
    ((130, 0, 700, 5), 256, 2, True, 3.0, 1),
    ((385,), 128, 1, False, 1.0, 2),
    ((1, 260, 1500), 128, 3, True, 4.0, 3),
    ((4000,), 1024, 2, True, 2.0, 4),
]


def _layers_dev(layers):
    return [{k: (dev_f32(v) if v is not None else None) for k, v in L.items()} for L in layers]


@pytest.mark.parametrize("case", CASES, ids=[f"n{'-'.join(map(str, c[0]))}_k{c[1]}_it{c[2]}" for c in CASES])
def test_refine_backward(lib, case):
    lengths, k, n_iter, affine, scale, seed = case
    p = make_sa_problem(lengths, k, 128, "bf16", seed=300 + seed, x_kind="gauss", p_scale=scale)
    layers = refine_layers(rng_for(400 + seed), n_iter, 128, affine)
    dsk = gauss(rng_for(500 + seed), (p.B, k, 128), 1.0)
    got = lib.sa_refine_backward(dev_x(p.X, p.dtype), p.offsets, dev_f32(p.P), _layers_dev(layers), dev_f32(dsk))
    torch.cuda.synchronize()
    lib.poll_device_status()
    ref = oracle.sa_refine_grads(p.x_f64(), p.offsets, p.P, layers, dsk.astype(np.float64))
    tol = tol_for("bf16")
    stats = {}
    if p.n_total > 0:
        stats["dX"] = compare("dX", got["dX"], ref["dX"], tol)
    stats["dP0"] = compare("dP0", got["dP0"], ref["dP0"], tol)
    for i, (g, r) in enumerate(zip(got["layers"], ref["layers"])):
        for name, rv in r.items():
            if rv is None:
                assert ("d" + name) not in g
                continue
            stats[f"{i}.{name}"] = compare(f"iteration {i} d{name}", g["d" + name], rv, tol)
    print(case, {k: round(v["mean_rel"], 5) for k, v in stats.items()})


def test_refine_backward_deterministic(lib):
    p = make_sa_problem((900, 300), 256, 128, "bf16", seed=7, x_kind="events", p_scale=3.0)
    layers = _layers_dev(refine_layers(rng_for(8), 2, 128))
    dsk = dev_f32(gauss(rng_for(9), (p.B, 256, 128), 1.0))
    X = dev_x(p.X, p.dtype)
    a = lib.sa_refine_backward(X, p.offsets, dev_f32(p.P), layers, dsk)
    b = lib.sa_refine_backward(X, p.offsets, dev_f32(p.P), layers, dsk)
    torch.cuda.synchronize()
    assert torch.equal(a["dX"], b["dX"]) and torch.equal(a["dP0"], b["dP0"])
    for ga, gb in zip(a["layers"], b["layers"]):
        for name in ga:
            assert torch.equal(ga[name], gb[name]), name
