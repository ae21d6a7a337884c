"""Shared helpers of the GPU parity tests: move seeded inputs to the device and
compare the library's outputs with the oracle under the stated tolerances.

Tolerances, per output tensor, normalised by that tensor's max |reference|:
  fp32 paths: max |err| <= 1e-4 max |ref|
  bf16 paths: max |err| <= 2e-2 max |ref|  and  sum |err| / sum |ref| <= 3e-3
  (the full STCA layer's bf16 path included: its computed tensor-core operands
  are fp16, so it meets the same bound)
"""
from __future__ import annotations

import numpy as np
import torch

from sa_inputs import SAProblem, STCABranch, STCAProblem

TOL_F32 = dict(max_rel=1e-4, mean_rel=None)
TOL_BF16 = dict(max_rel=2e-2, mean_rel=3e-3)



# The STCA backward with bf16 inputs: its attention and FFN products run on the bf16
# tensor cores with every fp32 operand split into hi + lo bf16 parts, so each operand
# is kept to 2^-16 ~ 1.5e-5 of its value and each product drops only lo x lo (also
# <= 2^-16 of |a| |b| per term): <= 3 x 2^-16 ~ 4.6e-5 of sum |a| |b| per product
# (pinned in test_split_arithmetic.py); the rest is fp32.  About ten chained products
# per layer over two layers give about 9e-4 in the worst case; the bound asks for a
# third of it.
TOL_SPLIT_BWD = dict(max_rel=3e-4, mean_rel=2e-4)


def tol_for(dtype: str) -> dict:
    return TOL_F32 if dtype == "f32" else TOL_BF16


def dev_x(X: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(X.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(X, np.float32)).to(device)


def dev_f32(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


def sa_device_inputs(p: SAProblem, device="cuda") -> dict:
    return dict(X=dev_x(p.X, p.dtype, device), P=dev_f32(p.P, device), W_Q=dev_f32(p.W_Q, device),
                W_K=dev_f32(p.W_K, device), W_V=dev_f32(p.W_V, device))


def compare(name: str, got, ref, tol: dict):
    got = got.detach().float().cpu().numpy().astype(np.float64) if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    err = np.abs(got - ref)
    scale = np.abs(ref).max() if ref.size else 0.0
    if scale == 0.0:
        assert err.max(initial=0.0) == 0.0, f"{name}: expected zeros, max |got| {err.max()}"
        return {"max_rel": 0.0, "mean_rel": 0.0}
    max_rel = err.max() / scale
    mean_rel = err.sum() / np.abs(ref).sum()
    assert max_rel <= tol["max_rel"], f"{name}: max|err|/max|ref| = {max_rel:.3e} > {tol['max_rel']:.1e}"
    if tol.get("mean_rel") is not None:
        assert mean_rel <= tol["mean_rel"], f"{name}: sum|err|/sum|ref| = {mean_rel:.3e} > {tol['mean_rel']:.1e}"
    return {"max_rel": float(max_rel), "mean_rel": float(mean_rel)}


def stca_layers_dev(layers, device="cuda"):
    out = []
    for L in layers:
        out.append(dict(W_Q=dev_f32(L.W_Q, device), W_K=dev_f32(L.W_K, device),
                        W_V=dev_f32(L.W_V, device),
                        W_O=None if L.W_O is None else dev_f32(L.W_O, device)))
    return out


def stca_branch_dev(br: STCABranch, dtype: str, device="cuda"):
    return dev_x(br.q, dtype, device), dev_x(br.kv, dtype, device)
