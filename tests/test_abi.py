"""The C-ABI library: it loads, exports every entry point the header declares,
answers workspace queries and rejects bad arguments with status codes before
touching the GPU (no compute calls here: these run without a GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

import sketch_attention_b200 as sab

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(inc, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M):
            name = m.group(1)
            if name not in ("defined",):
                names.add(name)
    return names


@pytest.fixture(scope="module")
def lib():
    from sketch_attention_b200 import build
    build.build()
    return sab.load()


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert {"sa_forward", "sa_backward", "stca_forward", "stca_fuse"} <= declared
    for name in declared:
        assert hasattr(lib, name), f"library does not export {name}"
    assert set(sab.EXPORTS) == declared


def test_version_and_workspace_queries(lib):
    assert lib.sa_version() >= 100
    w = sab.sa_forward_workspace(4, 10_000, 1024, 128, sab.SA_BF16)
    assert w >= 4 * 1024 * 128 * 4          # at least the H/(m+eps) scratch
    assert sab.sa_forward_workspace(0, 10, 4, 64, sab.SA_F32) == 0
    assert sab.sa_backward_workspace(2, 300, 64, 64, sab.SA_F32) > 300 * 4
    assert sab.stca_forward_workspace(2, 10, 128, 4, 32, sab.SA_BF16) > 0


def _fake(addr):
    return ctypes.c_void_p(addr)


def _fwd(lib, offsets, k=64, d=64, x=0x1000, ws_bytes=1 << 40, eps=1e-6):
    off = np.asarray(offsets, np.int64)
    B = len(off) - 1
    p = _fake(0x2000)
    return lib.sa_forward(_fake(x), sab.SA_F32, off.ctypes.data_as(ctypes.c_void_p), p, B, k, d,
                          p, p, p, p, eps, p, p, None, None, None, _fake(0x100000), ws_bytes, None)


def test_rejects_bad_arguments_without_touching_the_gpu(lib):
    assert _fwd(lib, [0, 5, 3]) == 1                   # offsets not monotone
    assert _fwd(lib, [1, 5]) == 1                      # offsets[0] != 0
    assert _fwd(lib, [0, 5], k=0) == 2                 # k out of range
    assert _fwd(lib, [0, 5], k=5000) == 2
    assert _fwd(lib, [0, 5], d=96) == 2                # d unsupported
    assert _fwd(lib, [0, 5], x=0x1004) == 1            # misaligned X
    assert _fwd(lib, [0, 5], x=0) == 1                 # NULL X with rows
    assert _fwd(lib, [0, 5], ws_bytes=16) == 5         # workspace too small
    assert _fwd(lib, [0, 5], eps=-1.0) == 1
    assert "workspace" in lib.sa_last_error().decode() or "eps" in lib.sa_last_error().decode()


def test_stca_rejects_bad_ranges(lib):
    cand = np.array([0, 2], np.int64)
    kb, ke = np.array([5], np.int64), np.array([3], np.int64)
    p = _fake(0x2000)
    lay = (sab.StcaLayerC * 1)()
    lay[0].W_Q = lay[0].W_K = lay[0].W_V = 0x3000
    st = lib.stca_forward(p, sab.SA_BF16, cand.ctypes.data_as(ctypes.c_void_p), p, 1, p, 10,
                          kb.ctypes.data_as(ctypes.c_void_p), ke.ctypes.data_as(ctypes.c_void_p),
                          p, p, 128, 4, 32, 1, lay, p, p, 1 << 40, None)
    assert st == 1 and "range" in lib.sa_last_error().decode()
    st = lib.stca_forward(p, sab.SA_BF16, cand.ctypes.data_as(ctypes.c_void_p), p, 1, p, 10,
                          kb.ctypes.data_as(ctypes.c_void_p), ke.ctypes.data_as(ctypes.c_void_p),
                          p, p, 96, 4, 32, 1, lay, p, p, 1 << 40, None)
    assert st == 2


def test_stca_backward_workspace_query(lib):
    """Host-only sizing of stca_backward_full's workspace: the bf16 path adds the operand
    splits of its tensor-core products; the score scratch is one user's (the largest),
    so a second, small user adds only its rows; an inverted range answers 0."""
    def ws(cands, kb, ke, dtype, n_layers=2):
        cand = np.concatenate([[0], np.cumsum(cands)]).astype(np.int64)
        return sab.stca_backward_full_workspace(cand, np.asarray(kb, np.int64), np.asarray(ke, np.int64),
                                                128, 4, 32, n_layers, dtype)
    one_f32 = ws([512], [0], [10_000], sab.SA_F32)
    one_bf16 = ws([512], [0], [10_000], sab.SA_BF16)
    score_f32 = 512 * 4 * 10_000 * 4                    # one user's S, fp32
    assert one_f32 >= 2 * score_f32                      # S and dS
    assert one_bf16 >= one_f32 + 2 * score_f32          # + P and dS as bf16 hi + lo pairs (4 B a score each)
    two_f32 = ws([512, 4], [0, 10_000], [10_000, 10_010], sab.SA_F32)
    assert one_f32 < two_f32 < one_f32 + score_f32 // 8
    assert ws([512], [0], [10_000], sab.SA_F32, n_layers=3) > one_f32
    assert ws([4], [10], [5], sab.SA_F32) == 0           # kv_end < kv_begin


def test_fused_event_rows_host_checks(lib):
    """Host-only checks of sa_gather_events_fused: its workspace holds the fp16 weights
    (3 x 256 x 128 x 2 bytes) and the per-action bias; sizes outside d = 128, d_ff = 2d
    and 1..16 action types answer 0 / SA_ERR_UNSUPPORTED, a short workspace
    SA_ERR_WORKSPACE, all before any GPU work."""
    w8 = sab.sa_gather_events_fused_workspace(8, 128, 256)
    assert w8 >= 3 * 256 * 128 * 2 + 8 * 512 * 4
    assert sab.sa_gather_events_fused_workspace(9, 128, 256) > w8
    assert sab.sa_gather_events_fused_workspace(8, 64, 128) == 0
    assert sab.sa_gather_events_fused_workspace(17, 128, 256) == 0
    p = _fake(0x10000)
    ids = _fake(0x20000)
    st = lib.sa_gather_events_fused(p, 1000, p, 8, ids, p, 10, 64, p, p, p, 128, p, p, 1 << 30, None)
    assert st == 2
    st = lib.sa_gather_events_fused(p, 1000, p, 17, ids, p, 10, 128, p, p, p, 256, p, p, 1 << 30, None)
    assert st == 2
    st = lib.sa_gather_events_fused(p, 1000, p, 8, ids, p, 10, 128, p, p, p, 256, p, p, w8 - 16, None)
    assert st == 5
    st = lib.sa_gather_events_fused(p, 1000, p, 8, _fake(0x20002), p, 10, 128, p, p, p, 256, p, p, w8, None)
    assert st == 1
