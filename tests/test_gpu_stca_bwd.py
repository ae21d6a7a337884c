"""GPU parity of stca_backward_full (the STCA backward through the attention, W_O
and both SwiGLU FFNs of the full layer) against the fp64 oracle's reverse-mode
gradients, through the C ABI.  With fp32 inputs everything runs in fp32 and
every gradient tensor is held to the fp32 bound; with bf16 inputs the attention
products run on the tensor cores over hi + lo bf16 splits of their fp32 operands
and the bound derived for that arithmetic applies."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import TOL_SPLIT_BWD, compare, dev_f32, dev_x, tol_for
from sa_inputs import STCALayer, add_stca_ffns, bf16_bits, bf16_to_f64, gauss, rng_for

pytestmark = pytest.mark.gpu

GRAD_OF = {"dW_Q": "W_Q", "dW_K": "W_K", "dW_V": "W_V", "dW_O": "W_O", "hist_dW1": "hist_W1",
           "hist_dW3": "hist_W3", "hist_dW2": "hist_W2", "q_dW1": "q_W1", "q_dW3": "q_W3", "q_dW2": "q_W2"}


def _problem(seed, cands, kv_rows, kb, ke, D, heads, d_h, n_layers, dtype, wo=True, hist=True, query=True,
             kv_scale=1.0):
    rng = rng_for(seed)
    layers = []
    for _ in range(n_layers):
        layers.append(STCALayer(gauss(rng, (heads, D, d_h), 1 / math.sqrt(D)),
                                gauss(rng, (heads, D, d_h), 1 / math.sqrt(D)),
                                gauss(rng, (heads, D, d_h), 1 / math.sqrt(D)),
                                gauss(rng, (heads * d_h, D), 1 / math.sqrt(D)) if wo else None))
    add_stca_ffns(rng, layers, D, hist, query)
    cand = np.concatenate([[0], np.cumsum(cands)]).astype(np.int64)
    q = gauss(rng, (int(cand[-1]), D), 1.0)
    kv = gauss(rng, (kv_rows, D), kv_scale)
    dout = gauss(rng, (int(cand[-1]), D), 1.0)
    if dtype == "bf16":
        q, kv = bf16_bits(q), bf16_bits(kv)
    return dict(layers=layers, cand=cand, q=q, kv=kv, kb=np.asarray(kb, np.int64), ke=np.asarray(ke, np.int64),
                dout=dout, heads=heads, d_h=d_h, dtype=dtype)


def _widen(p, a):
    return bf16_to_f64(a) if p["dtype"] == "bf16" else a.astype(np.float64)


def _layers_dev(layers):
    out = []
    for L in layers:
        out.append({k: (None if getattr(L, k) is None else dev_f32(getattr(L, k))) for k in oracle.STCA_WEIGHTS})
    return out


def _run(lib, p):
    g = lib.stca_backward_full(dev_x(p["q"], p["dtype"]), p["cand"], dev_x(p["kv"], p["dtype"]), p["kb"], p["ke"],
                               _layers_dev(p["layers"]), p["heads"], p["d_h"], dev_f32(p["dout"]))
    torch.cuda.synchronize()
    lib.poll_device_status()
    return g


def _check(lib, p):
    got = _run(lib, p)
    ref = oracle.stca_branch_grads(_widen(p, p["q"]), p["cand"], _widen(p, p["kv"]), p["kb"], p["ke"],
                                   p["layers"], p["heads"], p["d_h"], p["dout"])
    tol = tol_for("f32") if p["dtype"] == "f32" else TOL_SPLIT_BWD
    errs = {"dq": compare("dq", got["dq"], ref["dq"], tol), "dkv": compare("dkv", got["dkv"], ref["dkv"], tol)}
    for li, (gl, rl) in enumerate(zip(got["layers"], ref["layers"])):
        for gk, buf in gl.items():
            errs[f"{li}.{gk}"] = compare(f"layers[{li}].{gk}", buf, rl[GRAD_OF[gk]], tol)
    return errs


CASES = [
    # cands, kv rows, begins, ends, D, heads, d_h, layers, dtype, W_O, hist FFN, query FFN
    ((5, 0, 37, 3), 900, (0, 10, 100, 700), (300, 10, 700, 900), 128, 4, 32, 2, "bf16", True, True, True),
    ((7, 9), 600, (0, 250), (300, 600), 128, 4, 32, 2, "f32", False, True, False),
    ((33, 2), 500, (0, 0), (500, 0), 128, 2, 64, 1, "bf16", True, False, True),
    ((4, 4, 4), 260, (0, 100, 200), (150, 250, 260), 128, 4, 32, 2, "f32", True, False, False),
    # key ranges of 1, 7 and 65 rows: tiles far past the matrix edges on the tensor cores
    ((1, 2, 3), 80, (0, 1, 8), (1, 8, 73), 128, 4, 32, 2, "bf16", True, True, True),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{len(c[0])}_L{c[7]}_{c[8]}_wo{c[9]}_hf{c[10]}_qf{c[11]}" for c in CASES])
def test_stca_backward_small(lib, case):
    cands, rows, kb, ke, D, heads, d_h, nl, dtype, wo, hist, query = case
    p = _problem(500 + rows, cands, rows, kb, ke, D, heads, d_h, nl, dtype, wo, hist, query)
    errs = _check(lib, p)
    print(case, {k: (round(v["max_rel"], 6), round(v["mean_rel"], 6)) for k, v in errs.items()})


def test_stca_backward_overlapping_ranges_and_unused_rows(lib):
    """Users 0 and 1 share rows 100-199; rows 400-499 belong to no user (zero gradient)."""
    p = _problem(611, (6, 5), 500, (0, 100), (200, 400), 128, 4, 32, 2, "bf16")
    got = _run(lib, p)
    assert torch.count_nonzero(got["dkv"][400:]).item() == 0
    _check(lib, p)


def test_stca_backward_deterministic(lib):
    p = _problem(612, (40, 9), 2000, (0, 900), (900, 2000), 128, 4, 32, 2, "bf16")
    a, b = _run(lib, p), _run(lib, p)
    assert torch.equal(a["dq"], b["dq"]) and torch.equal(a["dkv"], b["dkv"])
    for la, lb in zip(a["layers"], b["layers"]):
        for k in la:
            assert torch.equal(la[k], lb[k]), k


def test_stca_backward_larger(lib):
    """Two users with 2.5K and 4K keys and 128 / 64 candidates (1K and 512 query rows
    per head group), two full layers."""
    p = _problem(613, (128, 64), 6500, (0, 2500), (2500, 6500), 128, 4, 32, 2, "bf16", kv_scale=0.5)
    errs = _check(lib, p)
    print({k: (round(v["max_rel"], 6), round(v["mean_rel"], 6)) for k, v in errs.items()})


def test_stca_backward_rejects_missing_gradient_buffer(lib):
    """Every argument valid except the layer's gradient buffers (all NULL)."""
    p = _problem(614, (3,), 10, (0,), (10,), 128, 4, 32, 1, "bf16")
    layers = _layers_dev(p["layers"])
    q, kv = dev_x(p["q"], "bf16"), dev_x(p["kv"], "bf16")
    dout = dev_f32(p["dout"])
    cd, kbd, ked = (torch.from_numpy(a).cuda() for a in (p["cand"], p["kb"], p["ke"]))
    ws = torch.empty(lib.stca_backward_full_workspace(p["cand"], p["kb"], p["ke"], 128, 4, 32, 1, lib.SA_BF16),
                     dtype=torch.uint8, device="cuda")
    garr = (lib.StcaFullLayerGradC * 1)()
    st = lib.load().stca_backward_full(q.data_ptr(), lib.SA_BF16, p["cand"].ctypes.data, cd.data_ptr(), 1,
                                       kv.data_ptr(), 10, p["kb"].ctypes.data, p["ke"].ctypes.data, kbd.data_ptr(),
                                       ked.data_ptr(), 128, 4, 32, 1, lib._full_layers_c(layers), dout.data_ptr(),
                                       None, None, garr, ws.data_ptr(), ws.numel(), None)
    assert st == 1      # SA_ERR_INVALID_ARG
    assert b"gradient" in lib.load().sa_last_error()


@pytest.mark.parametrize("which", ["recent", "sketch"])
def test_stca_backward_full_size_one_user(lib, which):
    """The bench's STCA-backward shapes for one user (512 candidates x 4 heads, a 10K
    suffix or a 1024-row sketch, two full layers): every gradient against the oracle.
    The weight gradients of a batch are sums of such per-user terms."""
    from sa_inputs import make_stca_problem
    prob = make_stca_problem(1, (512,), (10_000,), 1024, 128, 4, 32, 2, "bf16", seed=620)
    add_stca_ffns(rng_for(621), prob.layers_r, 128)
    add_stca_ffns(rng_for(622), prob.layers_u, 128)
    br = prob.recent if which == "recent" else prob.sketch
    layers = prob.layers_r if which == "recent" else prob.layers_u
    dout = gauss(rng_for(623), (512, 128), 1.0)
    p = dict(layers=layers, cand=br.cand_offsets, q=br.q, kv=br.kv, kb=br.kv_begin, ke=br.kv_end, dout=dout,
             heads=4, d_h=32, dtype="bf16")
    errs = _check(lib, p)
    print(which, {k: (round(v["max_rel"], 6), round(v["mean_rel"], 6)) for k, v in errs.items()})
