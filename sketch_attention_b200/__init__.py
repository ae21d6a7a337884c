"""Python binding of libsketchattn.so (include/sketch_attn.h).

Argument marshalling only: PyTorch supplies device memory and the current
stream; every step of SA and STCA runs in the library's CUDA kernels.  There
is no CPU fallback: if the library is missing or a call fails, an exception
is raised.

Entry points keep the C names: ``sa_forward``, ``sa_backward``,
``stca_forward``, ``stca_forward_full``, ``stca_fuse`` (plus the workspace queries).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsketchattn.so")

SA_F32, SA_BF16 = 0, 1
_STATUS = {0: "SA_OK", 1: "SA_ERR_INVALID_ARG", 2: "SA_ERR_UNSUPPORTED", 3: "SA_ERR_CUDA",
           4: "SA_ERR_TIMEOUT", 5: "SA_ERR_WORKSPACE"}

# Symbols include/sketch_attn.h declares.
EXPORTS = ("sa_version", "sa_last_error", "sa_poll_device_status", "sa_forward_workspace",
           "sa_forward", "sa_backward_workspace", "sa_backward", "stca_forward_workspace",
           "stca_forward", "stca_fuse", "sa_launch_count", "sa_profile", "sa_profile_read",
           "sa_forward_noalloc", "sa_refine_workspace", "sa_refine_forward",
           "sa_forward_tokenwise_workspace", "sa_forward_tokenwise", "sa_backward_accumulate",
           "stca_forward_full_workspace", "stca_forward_full", "stca_backward_full_workspace",
           "stca_backward_full", "sa_gather_events", "sa_gather_events_fused",
           "sa_gather_events_fused_workspace", "sa_measure_exp2_rate", "sa_selftest_bounded_wait",
           "sa_refine_backward_workspace", "sa_refine_backward")


class SAError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {_STATUS.get(status, status)}: {msg}")
        self.status = status


class StcaLayerC(ctypes.Structure):
    _fields_ = [("W_Q", ctypes.c_void_p), ("W_K", ctypes.c_void_p),
                ("W_V", ctypes.c_void_p), ("W_O", ctypes.c_void_p)]


STCA_FFN_KEYS = ("hist_W1", "hist_W3", "hist_W2", "q_W1", "q_W3", "q_W2")


class StcaFullLayerC(ctypes.Structure):
    _fields_ = [("attn", StcaLayerC)] + [(k, ctypes.c_void_p) for k in STCA_FFN_KEYS]


STCA_GRAD_KEYS = ("dW_Q", "dW_K", "dW_V", "dW_O", "hist_dW1", "hist_dW3", "hist_dW2", "q_dW1", "q_dW3", "q_dW2")


class StcaFullLayerGradC(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in STCA_GRAD_KEYS]


class RefineLayerC(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in ("W_Q", "W_K", "ln1_g", "ln1_b", "W1", "W3", "W2",
                                               "ln2_g", "ln2_b")]


REFINE_GRAD_KEYS = ("dW_Q", "dW_K", "dln1_g", "dln1_b", "dW1", "dW3", "dW2", "dln2_g", "dln2_b")


class RefineLayerGradC(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in REFINE_GRAD_KEYS]


_lib = None

_vp, _i, _i64, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


def load(path: Optional[str] = None):
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m sketch_attention_b200.build`")
    lib = ctypes.CDLL(path)
    lib.sa_version.restype = _i
    lib.sa_last_error.restype = ctypes.c_char_p
    lib.sa_poll_device_status.restype = _i
    lib.sa_poll_device_status.argtypes = [_vp]
    lib.sa_forward_workspace.restype = _sz
    lib.sa_forward_workspace.argtypes = [_i, _i64, _i, _i, _i]
    lib.sa_forward.restype = _i
    lib.sa_forward.argtypes = [_vp, _i, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _f,
                               _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.sa_backward_workspace.restype = _sz
    lib.sa_backward_workspace.argtypes = [_i, _i64, _i, _i, _i]
    lib.sa_backward.restype = _i
    lib.sa_backward.argtypes = [_vp, _i, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _f,
                                _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.sa_backward_accumulate.restype = _i
    lib.sa_backward_accumulate.argtypes = lib.sa_backward.argtypes
    lib.stca_forward_workspace.restype = _sz
    lib.stca_forward_workspace.argtypes = [_i, _i64, _i, _i, _i, _i]
    lib.stca_forward.restype = _i
    lib.stca_forward.argtypes = [_vp, _i, _vp, _vp, _i, _vp, _i64, _vp, _vp, _vp, _vp,
                                 _i, _i, _i, _i, ctypes.POINTER(StcaLayerC), _vp, _vp, _sz, _vp]
    lib.stca_forward_full_workspace.restype = _sz
    lib.stca_forward_full_workspace.argtypes = [_i, _i64, _i64, _i, _i, _i, _i]
    lib.stca_forward_full.restype = _i
    lib.stca_forward_full.argtypes = [_vp, _i, _vp, _vp, _i, _vp, _i64, _vp, _vp, _vp, _vp,
                                      _i, _i, _i, _i, ctypes.POINTER(StcaFullLayerC), _vp, _vp, _sz, _vp]
    lib.stca_backward_full_workspace.restype = _sz
    lib.stca_backward_full_workspace.argtypes = [_i, _vp, _vp, _vp, _i, _i, _i, _i, _i]
    lib.stca_backward_full.restype = _i
    lib.stca_backward_full.argtypes = [_vp, _i, _vp, _vp, _i, _vp, _i64, _vp, _vp, _vp, _vp,
                                       _i, _i, _i, _i, ctypes.POINTER(StcaFullLayerC), _vp, _vp, _vp,
                                       ctypes.POINTER(StcaFullLayerGradC), _vp, _sz, _vp]
    lib.sa_selftest_bounded_wait.restype = _i
    lib.sa_selftest_bounded_wait.argtypes = [ctypes.c_longlong, _vp]
    lib.sa_measure_exp2_rate.restype = _i
    lib.sa_measure_exp2_rate.argtypes = [_i, ctypes.POINTER(ctypes.c_double), _vp]
    lib.sa_gather_events.restype = _i
    lib.sa_gather_events.argtypes = [_vp, _i64, _vp, _i, _vp, _vp, _i64, _i, _vp, _vp]
    lib.sa_gather_events_fused_workspace.restype = _sz
    lib.sa_gather_events_fused_workspace.argtypes = [_i, _i, _i]
    lib.sa_gather_events_fused.restype = _i
    lib.sa_gather_events_fused.argtypes = [_vp, _i64, _vp, _i, _vp, _vp, _i64, _i, _vp, _vp, _vp, _i, _vp, _vp,
                                           _sz, _vp]
    lib.stca_fuse.restype = _i
    lib.stca_fuse.argtypes = [_vp, _vp, _vp, _vp, _i64, _i, _vp, _vp]
    lib.sa_forward_noalloc.restype = _i
    lib.sa_forward_noalloc.argtypes = [_vp, _i, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _f,
                                       _vp, _vp, _vp, _vp, _vp, _vp]
    lib.sa_forward_tokenwise_workspace.restype = _sz
    lib.sa_forward_tokenwise_workspace.argtypes = [_i, _i64, _i, _i, _i]
    lib.sa_forward_tokenwise.restype = _i
    lib.sa_forward_tokenwise.argtypes = [_vp, _i, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _f,
                                         _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.sa_refine_workspace.restype = _sz
    lib.sa_refine_workspace.argtypes = [_i, _i64, _i, _i, _i]
    lib.sa_refine_forward.restype = _i
    lib.sa_refine_forward.argtypes = [_vp, _i, _vp, _vp, _i, _i, _i, _vp, _i,
                                      ctypes.POINTER(RefineLayerC), _f, _vp, _vp, _sz, _vp]
    lib.sa_refine_backward_workspace.restype = _sz
    lib.sa_refine_backward_workspace.argtypes = [_i, _i64, _i, _i, _i, _i]
    lib.sa_refine_backward.restype = _i
    lib.sa_refine_backward.argtypes = [_vp, _i, _vp, _vp, _i, _i, _i, _vp, _i, ctypes.POINTER(RefineLayerC), _f,
                                       _vp, _vp, _vp, ctypes.POINTER(RefineLayerGradC), _vp, _sz, _vp]
    lib.sa_launch_count.restype = ctypes.c_longlong
    lib.sa_profile.restype = _i
    lib.sa_profile.argtypes = [_i]
    lib.sa_profile_read.restype = _i
    lib.sa_profile_read.argtypes = [_i, ctypes.c_char_p, _i, ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(ctypes.c_longlong)]
    _lib = lib
    return lib


def _check(fn: str, status: int):
    if status != 0:
        raise SAError(fn, status, load().sa_last_error().decode())


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SA_F32
    if t.dtype == torch.bfloat16:
        return SA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _host_i64(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def _hp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dev_i64(host: np.ndarray, device, given: Optional[torch.Tensor]) -> torch.Tensor:
    if given is not None:
        return given
    return torch.from_numpy(host).to(device, non_blocking=False)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


# --------------------------------------------------------------------------
def sa_forward_workspace(B: int, n_total: int, k: int, d: int, dtype: int) -> int:
    return int(load().sa_forward_workspace(B, n_total, k, d, dtype))


def sa_forward(X: torch.Tensor, offsets, P, W_Q, W_K, W_V, eps: float = 1e-6, *,
               offsets_dev: Optional[torch.Tensor] = None, want_H: bool = False,
               want_bf16: bool = False, want_lse: bool = False, out: Optional[dict] = None,
               workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """Sketches of a ragged batch.  Returns {"S", "mass"[, "H"][, "S_bf16"][, "lse"]}."""
    lib = load()
    _need_cuda(X, P, W_Q, W_K, W_V)
    off = _host_i64(offsets)
    B = len(off) - 1
    k, d = P.shape
    dev = X.device
    dt = _dtype_code(X)
    o = dict(out or {})
    S = o.get("S") if o.get("S") is not None else torch.empty(B, k, d, device=dev)
    mass = o.get("mass") if o.get("mass") is not None else torch.empty(B, k, device=dev)
    H = o.get("H") if o.get("H") is not None else (torch.empty(B, k, d, device=dev) if want_H else None)
    Sb = o.get("S_bf16") if o.get("S_bf16") is not None else (
        torch.empty(B, k, d, device=dev, dtype=torch.bfloat16) if want_bf16 else None)
    lse = o.get("lse") if o.get("lse") is not None else (
        torch.empty(max(int(off[-1]), 1), device=dev) if want_lse else None)
    ws_bytes = lib.sa_forward_workspace(B, int(off[-1]), k, d, dt)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    offd = _dev_i64(off, dev, offsets_dev)
    st = lib.sa_forward(_p(X), dt, _hp(off), _p(offd), B, k, d, _p(P), _p(W_Q), _p(W_K), _p(W_V),
                        float(eps), _p(S), _p(mass), _p(H), _p(Sb), _p(lse), _p(workspace),
                        workspace.numel(), _stream(stream))
    _check("sa_forward", st)
    res = {"S": S, "mass": mass}
    if H is not None:
        res["H"] = H
    if Sb is not None:
        res["S_bf16"] = Sb
    if lse is not None:
        res["lse"] = lse
    return res


def sa_forward_tokenwise_workspace(B: int, n_total: int, k: int, d: int, x_dtype: int) -> int:
    return int(load().sa_forward_tokenwise_workspace(B, n_total, k, d, x_dtype))


def sa_forward_tokenwise(X: torch.Tensor, offsets, P, W_Q, W_K, W_V, eps: float = 1e-6, *,
                         offsets_dev: Optional[torch.Tensor] = None, want_H: bool = False,
                         want_bf16: bool = False, out: Optional[dict] = None,
                         workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """The token-wise normalisation variant (softmax over each prototype's tokens).
    Returns {"S", "mass"[, "H"][, "S_bf16"]}."""
    lib = load()
    _need_cuda(X, P, W_Q, W_K, W_V)
    off = _host_i64(offsets)
    B = len(off) - 1
    k, d = P.shape
    dev = X.device
    dt = _dtype_code(X)
    o = dict(out or {})
    S = o.get("S") if o.get("S") is not None else torch.empty(B, k, d, device=dev)
    mass = o.get("mass") if o.get("mass") is not None else torch.empty(B, k, device=dev)
    H = o.get("H") if o.get("H") is not None else (torch.empty(B, k, d, device=dev) if want_H else None)
    Sb = o.get("S_bf16") if o.get("S_bf16") is not None else (
        torch.empty(B, k, d, device=dev, dtype=torch.bfloat16) if want_bf16 else None)
    ws_bytes = lib.sa_forward_tokenwise_workspace(B, int(off[-1]), k, d, dt)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    offd = _dev_i64(off, dev, offsets_dev)
    st = lib.sa_forward_tokenwise(_p(X), dt, _hp(off), _p(offd), B, k, d, _p(P), _p(W_Q), _p(W_K),
                                  _p(W_V), float(eps), _p(S), _p(mass), _p(H), _p(Sb),
                                  _p(workspace), workspace.numel(), _stream(stream))
    _check("sa_forward_tokenwise", st)
    res = {"S": S, "mass": mass}
    if H is not None:
        res["H"] = H
    if Sb is not None:
        res["S_bf16"] = Sb
    return res


def sa_forward_noalloc(X: torch.Tensor, offsets, P, W_Q, W_K, W_V, eps: float = 1e-6, *,
                       offsets_dev: torch.Tensor, out: dict, stream=None) -> dict:
    """sa_forward without a workspace, for callers that cannot allocate device
    memory: every buffer is the caller's (``out`` holds preallocated "S" and
    "mass", optionally "H", "S_bf16", "lse"; ``offsets_dev`` is a device copy of
    the offsets), and the library's fixed scratch array stands in for the
    workspace.  This wrapper allocates nothing on the device."""
    lib = load()
    _need_cuda(X, P, W_Q, W_K, W_V, offsets_dev)
    off = _host_i64(offsets)
    B = len(off) - 1
    k, d = P.shape
    o = {n: out.get(n) for n in ("S", "mass", "H", "S_bf16", "lse")}
    _need_cuda(*[t for t in o.values() if t is not None])
    st = lib.sa_forward_noalloc(_p(X), _dtype_code(X), _hp(off), _p(offsets_dev), B, k, d, _p(P),
                                _p(W_Q), _p(W_K), _p(W_V), float(eps), _p(o["S"]), _p(o["mass"]),
                                _p(o["H"]), _p(o["S_bf16"]), _p(o["lse"]), _stream(stream))
    _check("sa_forward_noalloc", st)
    return {n: t for n, t in o.items() if t is not None}


def sa_backward_workspace(B: int, n_total: int, k: int, d: int, dtype: int) -> int:
    return int(load().sa_backward_workspace(B, n_total, k, d, dtype))


def sa_backward(X: torch.Tensor, offsets, P, W_Q, W_K, W_V, eps: float, H, mass, dS,
                dmass=None, lse=None, *, offsets_dev: Optional[torch.Tensor] = None,
                out: Optional[dict] = None, workspace: Optional[torch.Tensor] = None,
                stream=None, accumulate: bool = False) -> dict:
    """Gradients {"dX", "dP", "dW_Q", "dW_K", "dW_V"} of <dS, S> + <dmass, mass>.
    With ``accumulate`` the weight gradients are added into out's dP, dW_Q, dW_K,
    dW_V (sa_backward_accumulate), e.g. one call per group of users."""
    lib = load()
    _need_cuda(X, P, W_Q, W_K, W_V, H, mass, dS, dmass, lse)
    off = _host_i64(offsets)
    B = len(off) - 1
    k, d = P.shape
    dev = X.device
    dt = _dtype_code(X)
    o = dict(out or {})
    dX = o.get("dX") if o.get("dX") is not None else torch.empty_like(X)
    dP = o.get("dP") if o.get("dP") is not None else torch.empty(k, d, device=dev)
    dWQ = o.get("dW_Q") if o.get("dW_Q") is not None else torch.empty(d, d, device=dev)
    dWK = o.get("dW_K") if o.get("dW_K") is not None else torch.empty(d, d, device=dev)
    dWV = o.get("dW_V") if o.get("dW_V") is not None else torch.empty(d, d, device=dev)
    ws_bytes = lib.sa_backward_workspace(B, int(off[-1]), k, d, dt)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    offd = _dev_i64(off, dev, offsets_dev)
    if accumulate and any(o.get(n) is None for n in ("dP", "dW_Q", "dW_K", "dW_V")):
        raise ValueError("accumulate needs out with dP, dW_Q, dW_K and dW_V")
    fn = lib.sa_backward_accumulate if accumulate else lib.sa_backward
    st = fn(_p(X), dt, _hp(off), _p(offd), B, k, d, _p(P), _p(W_Q), _p(W_K), _p(W_V),
            float(eps), _p(H), _p(mass), _p(dS), _p(dmass), _p(lse), _p(dX), _p(dP), _p(dWQ),
            _p(dWK), _p(dWV), _p(workspace), workspace.numel(), _stream(stream))
    _check("sa_backward_accumulate" if accumulate else "sa_backward", st)
    return {"dX": dX, "dP": dP, "dW_Q": dWQ, "dW_K": dWK, "dW_V": dWV}


def stca_forward_workspace(B: int, C_total: int, D: int, heads: int, d_h: int, dtype: int) -> int:
    return int(load().stca_forward_workspace(B, C_total, D, heads, d_h, dtype))


def stca_forward(q: torch.Tensor, cand_offsets, kv: torch.Tensor, kv_begin, kv_end,
                 layers: Sequence[dict], heads: int, d_h: int, *,
                 cand_offsets_dev=None, kv_begin_dev=None, kv_end_dev=None,
                 out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """One STCA branch.  ``layers``: dicts with W_Q, W_K, W_V [heads, D, d_h] and
    W_O [heads*d_h, D] or None (fp32 CUDA tensors).  Returns out [C_total, D] fp32."""
    lib = load()
    _need_cuda(q, kv)
    dt = _dtype_code(q)
    if kv.dtype != q.dtype:
        raise TypeError("q and kv must have the same dtype")
    cand = _host_i64(cand_offsets)
    kb, ke = _host_i64(kv_begin), _host_i64(kv_end)
    B = len(cand) - 1
    D = q.shape[1]
    dev = q.device
    C = int(cand[-1])
    res = out if out is not None else torch.empty(C, D, device=dev)
    arr = (StcaLayerC * len(layers))()
    for i, L in enumerate(layers):
        _need_cuda(L["W_Q"], L["W_K"], L["W_V"], L.get("W_O"))
        arr[i].W_Q = L["W_Q"].data_ptr()
        arr[i].W_K = L["W_K"].data_ptr()
        arr[i].W_V = L["W_V"].data_ptr()
        arr[i].W_O = L["W_O"].data_ptr() if L.get("W_O") is not None else None
    ws_bytes = lib.stca_forward_workspace(B, C, D, heads, d_h, dt)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    cd = _dev_i64(cand, dev, cand_offsets_dev)
    kbd = _dev_i64(kb, dev, kv_begin_dev)
    ked = _dev_i64(ke, dev, kv_end_dev)
    st = lib.stca_forward(_p(q), dt, _hp(cand), _p(cd), B, _p(kv), kv.shape[0], _hp(kb), _hp(ke),
                          _p(kbd), _p(ked), D, heads, d_h, len(layers), arr, _p(res),
                          _p(workspace), workspace.numel(), _stream(stream))
    _check("stca_forward", st)
    return res


def stca_forward_full_workspace(B: int, C_total: int, kv_total: int, D: int, heads: int, d_h: int,
                                dtype: int) -> int:
    return int(load().stca_forward_full_workspace(B, C_total, kv_total, D, heads, d_h, dtype))


def stca_forward_full(q: torch.Tensor, cand_offsets, kv: torch.Tensor, kv_begin, kv_end,
                      layers: Sequence[dict], heads: int, d_h: int, *,
                      cand_offsets_dev=None, kv_begin_dev=None, kv_end_dev=None,
                      out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """One STCA branch of full layers (the attention layer plus the history- and
    query-side SwiGLU FFNs).  ``layers``: dicts as for stca_forward plus, each
    optional (absent or None = no such FFN), hist_W1, hist_W3 [D, 2D], hist_W2
    [2D, D], q_W1, q_W3 [D, 2D], q_W2 [2D, D] (fp32 CUDA tensors).  Returns
    out [C_total, D] fp32."""
    lib = load()
    _need_cuda(q, kv)
    dt = _dtype_code(q)
    if kv.dtype != q.dtype:
        raise TypeError("q and kv must have the same dtype")
    cand = _host_i64(cand_offsets)
    kb, ke = _host_i64(kv_begin), _host_i64(kv_end)
    B = len(cand) - 1
    D = q.shape[1]
    dev = q.device
    C = int(cand[-1])
    kv_total = int((ke - kb).sum()) if B else 0
    res = out if out is not None else torch.empty(C, D, device=dev)
    arr = (StcaFullLayerC * len(layers))()
    for i, L in enumerate(layers):
        _need_cuda(L["W_Q"], L["W_K"], L["W_V"], L.get("W_O"), *(L.get(k) for k in STCA_FFN_KEYS))
        arr[i].attn.W_Q = L["W_Q"].data_ptr()
        arr[i].attn.W_K = L["W_K"].data_ptr()
        arr[i].attn.W_V = L["W_V"].data_ptr()
        arr[i].attn.W_O = L["W_O"].data_ptr() if L.get("W_O") is not None else None
        for k in STCA_FFN_KEYS:
            setattr(arr[i], k, L[k].data_ptr() if L.get(k) is not None else None)
    ws_bytes = lib.stca_forward_full_workspace(B, C, kv_total, D, heads, d_h, dt)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    cd = _dev_i64(cand, dev, cand_offsets_dev)
    kbd = _dev_i64(kb, dev, kv_begin_dev)
    ked = _dev_i64(ke, dev, kv_end_dev)
    st = lib.stca_forward_full(_p(q), dt, _hp(cand), _p(cd), B, _p(kv), kv.shape[0], _hp(kb), _hp(ke),
                               _p(kbd), _p(ked), D, heads, d_h, len(layers), arr, _p(res),
                               _p(workspace), workspace.numel(), _stream(stream))
    _check("stca_forward_full", st)
    return res


def selftest_bounded_wait(budget_cycles: int = 2_000_000, stream=None) -> None:
    """Launch a kernel whose only wait cannot complete (bounded to ~budget_cycles);
    the next poll_device_status() raises SAError with SA_ERR_TIMEOUT."""
    _check("sa_selftest_bounded_wait", load().sa_selftest_bounded_wait(budget_cycles, _stream(stream)))


def measure_exp2_rate(mode: int = 1, stream=None) -> float:
    """Exponentials per second on the current GPU: mode 0 all on the MUFU, mode 1 the
    SA forward kernels' mix (one pair in four on the FMA pipe)."""
    out = ctypes.c_double(0.0)
    _check("sa_measure_exp2_rate", load().sa_measure_exp2_rate(mode, ctypes.byref(out), _stream(stream)))
    return out.value


def sa_gather_events(item_table: torch.Tensor, action_table: torch.Tensor, item_ids: torch.Tensor,
                     action_ids: torch.Tensor, *, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """X[i] = item_table[item_ids[i]] + action_table[action_ids[i]] (bf16 tables and
    output, int32 / uint8 ids, CUDA tensors).  Returns X [n, d] bf16."""
    lib = load()
    _need_cuda(item_table, action_table, item_ids, action_ids)
    if item_table.dtype != torch.bfloat16 or action_table.dtype != torch.bfloat16:
        raise TypeError("the tables must be bf16")
    if item_ids.dtype != torch.int32 or action_ids.dtype != torch.uint8:
        raise TypeError("item_ids must be int32 and action_ids uint8")
    n, d = item_ids.numel(), item_table.shape[1]
    X = out if out is not None else torch.empty(n, d, dtype=torch.bfloat16, device=item_table.device)
    st = lib.sa_gather_events(_p(item_table), item_table.shape[0], _p(action_table), action_table.shape[0],
                              _p(item_ids), _p(action_ids), n, d, _p(X), _stream(stream))
    _check("sa_gather_events", st)
    return X


def sa_gather_events_fused_workspace(n_actions: int, d: int = 128, d_ff: int = 256) -> int:
    return int(load().sa_gather_events_fused_workspace(n_actions, d, d_ff))


def sa_gather_events_fused(item_table: torch.Tensor, action_table: torch.Tensor, item_ids: torch.Tensor,
                           action_ids: torch.Tensor, W1: torch.Tensor, W3: torch.Tensor, W2: torch.Tensor, *,
                           out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    """X[i] = e + (SiLU(z W1) * (z W3)) W2 with e = item_table[item_ids[i]],
    z = [e ; action_table[action_ids[i]]] (eq. (20)); bf16 tables and output,
    int32 / uint8 ids, fp32 weights W1, W3 [2d, d_ff], W2 [d_ff, d].  Returns X [n, d]."""
    lib = load()
    _need_cuda(item_table, action_table, item_ids, action_ids, W1, W3, W2)
    if item_table.dtype != torch.bfloat16 or action_table.dtype != torch.bfloat16:
        raise TypeError("the tables must be bf16")
    if item_ids.dtype != torch.int32 or action_ids.dtype != torch.uint8:
        raise TypeError("item_ids must be int32 and action_ids uint8")
    n, d = item_ids.numel(), item_table.shape[1]
    d_ff = W2.shape[0]
    na = action_table.shape[0]
    X = out if out is not None else torch.empty(n, d, dtype=torch.bfloat16, device=item_table.device)
    if workspace is None:
        workspace = torch.empty(max(sa_gather_events_fused_workspace(na, d, d_ff), 16), dtype=torch.uint8,
                                device=item_table.device)
    st = lib.sa_gather_events_fused(_p(item_table), item_table.shape[0], _p(action_table), na, _p(item_ids),
                                    _p(action_ids), n, d, _p(W1), _p(W3), _p(W2), d_ff, _p(X), _p(workspace),
                                    workspace.numel(), _stream(stream))
    _check("sa_gather_events_fused", st)
    return X


def _full_layers_c(layers):
    arr = (StcaFullLayerC * len(layers))()
    for i, L in enumerate(layers):
        _need_cuda(L["W_Q"], L["W_K"], L["W_V"], L.get("W_O"), *(L.get(k) for k in STCA_FFN_KEYS))
        arr[i].attn.W_Q = L["W_Q"].data_ptr()
        arr[i].attn.W_K = L["W_K"].data_ptr()
        arr[i].attn.W_V = L["W_V"].data_ptr()
        arr[i].attn.W_O = L["W_O"].data_ptr() if L.get("W_O") is not None else None
        for k in STCA_FFN_KEYS:
            setattr(arr[i], k, L[k].data_ptr() if L.get(k) is not None else None)
    return arr


def stca_backward_full_workspace(cand_offsets, kv_begin, kv_end, D: int, heads: int, d_h: int,
                                 n_layers: int, dtype: int) -> int:
    cand, kb, ke = _host_i64(cand_offsets), _host_i64(kv_begin), _host_i64(kv_end)
    return int(load().stca_backward_full_workspace(len(cand) - 1, _hp(cand), _hp(kb), _hp(ke), D, heads, d_h,
                                                   n_layers, dtype))


def stca_backward_full(q: torch.Tensor, cand_offsets, kv: torch.Tensor, kv_begin, kv_end,
                       layers: Sequence[dict], heads: int, d_h: int, dout: torch.Tensor, *,
                       cand_offsets_dev=None, kv_begin_dev=None, kv_end_dev=None,
                       out: Optional[dict] = None, workspace: Optional[torch.Tensor] = None,
                       stream=None) -> dict:
    """Backward of stca_forward_full.  ``dout`` [C_total, D] fp32.  Returns {"dq": [C, D],
    "dkv": [kv_rows, D], "layers": [dict of weight gradients per layer]} (fp32; the
    gradient keys are dW_Q, dW_K, dW_V, dW_O and hist_dW1.. / q_dW1.. for the FFNs that
    the layer has).  ``out`` may supply any of these buffers."""
    lib = load()
    _need_cuda(q, kv, dout)
    dt = _dtype_code(q)
    if kv.dtype != q.dtype:
        raise TypeError("q and kv must have the same dtype")
    cand = _host_i64(cand_offsets)
    kb, ke = _host_i64(kv_begin), _host_i64(kv_end)
    B = len(cand) - 1
    D = q.shape[1]
    dev = q.device
    C = int(cand[-1])
    out = dict(out or {})
    dq = out.get("dq") if out.get("dq") is not None else torch.empty(C, D, device=dev)
    dkv = out.get("dkv") if out.get("dkv") is not None else torch.empty(kv.shape[0], D, device=dev)
    lg_out = out.get("layers") or [{} for _ in layers]
    grads = []
    garr = (StcaFullLayerGradC * len(layers))()
    for i, L in enumerate(layers):
        g = {}
        have = {"dW_Q": "W_Q", "dW_K": "W_K", "dW_V": "W_V", "dW_O": "W_O", "hist_dW1": "hist_W1",
                "hist_dW3": "hist_W3", "hist_dW2": "hist_W2", "q_dW1": "q_W1", "q_dW3": "q_W3", "q_dW2": "q_W2"}
        for gk, wk in have.items():
            if L.get(wk) is None:
                continue
            buf = lg_out[i].get(gk) if lg_out[i].get(gk) is not None else torch.empty_like(L[wk])
            _need_cuda(buf)
            g[gk] = buf
            setattr(garr[i], gk, buf.data_ptr())
        grads.append(g)
    arr = _full_layers_c(layers)
    ws_bytes = lib.stca_backward_full_workspace(B, _hp(cand), _hp(kb), _hp(ke), D, heads, d_h, len(layers), dt)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    cd = _dev_i64(cand, dev, cand_offsets_dev)
    kbd = _dev_i64(kb, dev, kv_begin_dev)
    ked = _dev_i64(ke, dev, kv_end_dev)
    st = lib.stca_backward_full(_p(q), dt, _hp(cand), _p(cd), B, _p(kv), kv.shape[0], _hp(kb), _hp(ke),
                                _p(kbd), _p(ked), D, heads, d_h, len(layers), arr, _p(dout), _p(dq), _p(dkv),
                                garr, _p(workspace), workspace.numel(), _stream(stream))
    _check("stca_backward_full", st)
    return {"dq": dq, "dkv": dkv, "layers": grads}


REFINE_KEYS = ("W_Q", "W_K", "ln1_g", "ln1_b", "W1", "W3", "W2", "ln2_g", "ln2_b")


def sa_refine_workspace(B: int, n_total: int, k: int, d: int, x_dtype: int) -> int:
    return int(load().sa_refine_workspace(B, n_total, k, d, x_dtype))


def sa_refine_forward(X: torch.Tensor, offsets, P0: torch.Tensor, layers: Sequence[dict],
                      ln_eps: float = 1e-5, *, offsets_dev=None, out: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Stacked SA refinement, len(layers) iterations from the shared prototypes P0
    [k, d].  ``layers``: dicts with W_Q, W_K [d, d], W1, W3 [d, 2d], W2 [2d, d] and
    optional ln1_g, ln1_b, ln2_g, ln2_b [d] (fp32 CUDA tensors).  Returns the
    sketch [B, k, d] fp32."""
    lib = load()
    _need_cuda(X, P0)
    dt = _dtype_code(X)
    off = _host_i64(offsets)
    B = len(off) - 1
    k, d = P0.shape
    dev = X.device
    res = out if out is not None else torch.empty(B, k, d, device=dev)
    arr = (RefineLayerC * len(layers))()
    for i, L in enumerate(layers):
        for key in REFINE_KEYS:
            t = L.get(key)
            _need_cuda(t)
            setattr(arr[i], key, t.data_ptr() if t is not None else None)
    ws_bytes = lib.sa_refine_workspace(B, int(off[-1]), k, d, dt)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    od = _dev_i64(off, dev, offsets_dev)
    st = lib.sa_refine_forward(_p(X), dt, _hp(off), _p(od), B, k, d, _p(P0), len(layers), arr,
                               ln_eps, _p(res), _p(workspace), workspace.numel(), _stream(stream))
    _check("sa_refine_forward", st)
    return res


def sa_refine_backward_workspace(B: int, n_total: int, k: int, d: int, n_iter: int, dtype: int) -> int:
    return int(load().sa_refine_backward_workspace(B, n_total, k, d, n_iter, dtype))


def sa_refine_backward(X: torch.Tensor, offsets, P0: torch.Tensor, layers: Sequence[dict], dsketch: torch.Tensor,
                       ln_eps: float = 1e-5, *, offsets_dev=None, out: Optional[dict] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """Gradients of <dsketch, sa_refine_forward(X, offsets, P0, layers)>: returns
    {"dX": [n, d] fp32, "dP0": [k, d] fp32, "layers": [{"dW_Q", "dW_K", "dW1", "dW3", "dW2",
    and "dln1_g", ... for the LayerNorm parameters the layer has}]}."""
    lib = load()
    _need_cuda(X, P0, dsketch)
    dt = _dtype_code(X)
    off = _host_i64(offsets)
    B = len(off) - 1
    k, d = P0.shape
    n = int(off[-1])
    dev = X.device
    o = dict(out or {})
    dX = o.get("dX") if o.get("dX") is not None else torch.empty(max(n, 1), d, device=dev)
    dP0 = o.get("dP0") if o.get("dP0") is not None else torch.empty(k, d, device=dev)
    arr = (RefineLayerC * len(layers))()
    garr = (RefineLayerGradC * len(layers))()
    gl = []
    for i, L in enumerate(layers):
        g = {}
        for key in REFINE_KEYS:
            t = L.get(key)
            _need_cuda(t)
            setattr(arr[i], key, t.data_ptr() if t is not None else None)
            if t is not None:
                g["d" + key] = torch.empty_like(t)
                setattr(garr[i], "d" + key, g["d" + key].data_ptr())
        gl.append(g)
    ws_bytes = lib.sa_refine_backward_workspace(B, n, k, d, len(layers), dt)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    od = _dev_i64(off, dev, offsets_dev)
    st = lib.sa_refine_backward(_p(X), dt, _hp(off), _p(od), B, k, d, _p(P0), len(layers), arr, ln_eps,
                                _p(dsketch), _p(dX), _p(dP0), garr, _p(workspace), workspace.numel(),
                                _stream(stream))
    _check("sa_refine_backward", st)
    return {"dX": dX[:n], "dP0": dP0, "layers": gl}


def stca_fuse(z_r: torch.Tensor, z_u: torch.Tensor, W_F: torch.Tensor, b_F=None, *,
              out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """[z_r ; z_u] W_F + b_F."""
    lib = load()
    _need_cuda(z_r, z_u, W_F, b_F)
    C, D = z_r.shape
    res = out if out is not None else torch.empty(C, D, device=z_r.device)
    st = lib.stca_fuse(_p(z_r), _p(z_u), _p(W_F), _p(b_F), C, D, _p(res), _stream(stream))
    _check("stca_fuse", st)
    return res


def poll_device_status(stream=None) -> None:
    _check("sa_poll_device_status", load().sa_poll_device_status(_stream(stream)))


# --------------------------------------------------------------------------
# measurement support
def launch_count() -> int:
    """Kernels the library has launched in this process."""
    return int(load().sa_launch_count())


def profile(enable: bool) -> None:
    """Start (clearing) or stop the library's per-kernel event timers."""
    load().sa_profile(1 if enable else 0)


def profile_read() -> dict:
    """{kernel name: (total device ms, launches)} since profile(True)."""
    lib = load()
    out = {}
    buf = ctypes.create_string_buffer(128)
    ms, cnt = ctypes.c_double(), ctypes.c_longlong()
    i = 0
    while lib.sa_profile_read(i, buf, 128, ctypes.byref(ms), ctypes.byref(cnt)):
        out[buf.value.decode()] = (ms.value, cnt.value)
        i += 1
    return out
