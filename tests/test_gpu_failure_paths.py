"""Failure paths that fault no GPU (through the C ABI): a device-side wait that runs
out reports SA_ERR_TIMEOUT and leaves the context usable, and no entry point writes
outside its workspace or its outputs (canary bytes around each)."""
import numpy as np
import pytest
import torch

from helpers import dev_f32, dev_x
from sa_inputs import (add_stca_ffns, event_ffn_weights, event_problem, make_sa_problem, make_stca_problem,
                       refine_layers, rng_for)

pytestmark = pytest.mark.gpu

PAD = 1 << 20          # canary bytes before and after (a multiple of 256: alignment kept)
CANARY = 0xA5


def test_bounded_wait_expires_and_reports(lib):
    lib.selftest_bounded_wait(2_000_000)          # about a millisecond of SM clocks
    torch.cuda.synchronize()
    with pytest.raises(lib.SAError) as e:
        lib.poll_device_status()
    assert e.value.status == 4                    # SA_ERR_TIMEOUT
    lib.poll_device_status()                      # the word was cleared
    # the context is still usable: a forward runs and is checked by the other tests
    p = make_sa_problem((300, 5), 128, 128, "bf16", seed=801)
    lib.sa_forward(dev_x(p.X, p.dtype), p.offsets, dev_f32(p.P), dev_f32(p.W_Q), dev_f32(p.W_K),
                   dev_f32(p.W_V), p.eps)
    torch.cuda.synchronize()
    lib.poll_device_status()


def _padded(nbytes):
    big = torch.full((nbytes + 2 * PAD,), CANARY, dtype=torch.uint8, device="cuda")
    return big, big[PAD:PAD + nbytes]


def _padded_like(shape, dtype):
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    big, mid = _padded(n)
    return big, mid.view(dtype).view(*shape)


def _intact(big, nbytes):
    head = big[:PAD]
    tail = big[PAD + nbytes:]
    return bool((head == CANARY).all()) and bool((tail == CANARY).all())


def test_sa_forward_and_backward_stay_inside_their_buffers(lib):
    p = make_sa_problem((700, 0, 1300), 256, 128, "bf16", seed=802, x_kind="events")
    X = dev_x(p.X, p.dtype)
    W = [dev_f32(a) for a in (p.P, p.W_Q, p.W_K, p.W_V)]
    B, n = p.B, p.n_total
    ws_b = lib.sa_forward_workspace(B, n, p.k, p.d, lib.SA_BF16)
    wbig, ws = _padded(ws_b)
    outs = {"S": _padded_like((B, p.k, p.d), torch.float32), "mass": _padded_like((B, p.k), torch.float32),
            "H": _padded_like((B, p.k, p.d), torch.float32), "lse": _padded_like((n,), torch.float32)}
    f = lib.sa_forward(X, p.offsets, *W, p.eps, out={k: v[1] for k, v in outs.items()}, workspace=ws)
    torch.cuda.synchronize()
    lib.poll_device_status()
    assert _intact(wbig, ws_b)
    for k, (big, t) in outs.items():
        assert _intact(big, t.numel() * t.element_size()), k
    gbytes = lib.sa_backward_workspace(B, n, p.k, p.d, lib.SA_BF16)
    gbig, gws = _padded(gbytes)
    dS = dev_f32(np.random.default_rng(3).standard_normal((B, p.k, p.d)).astype(np.float32))
    gout = {"dX": _padded_like((n, p.d), torch.bfloat16), "dP": _padded_like((p.k, p.d), torch.float32),
            "dW_Q": _padded_like((p.d, p.d), torch.float32), "dW_K": _padded_like((p.d, p.d), torch.float32),
            "dW_V": _padded_like((p.d, p.d), torch.float32)}
    lib.sa_backward(X, p.offsets, *W, p.eps, f["H"], f["mass"], dS, None, f["lse"],
                    out={k: v[1] for k, v in gout.items()}, workspace=gws)
    torch.cuda.synchronize()
    lib.poll_device_status()
    assert _intact(gbig, gbytes)
    for k, (big, t) in gout.items():
        assert _intact(big, t.numel() * t.element_size()), k


def test_stca_entry_points_stay_inside_their_workspaces(lib):
    prob = make_stca_problem(3, (5, 0, 37), (1, 200, 130), 64, 128, 4, 32, 2, "bf16", seed=803)
    add_stca_ffns(rng_for(804), prob.layers_r, 128)
    br = prob.recent
    q, kv = dev_x(br.q, "bf16"), dev_x(br.kv, "bf16")
    keys = ("W_Q", "W_K", "W_V", "W_O", "hist_W1", "hist_W3", "hist_W2", "q_W1", "q_W3", "q_W2")
    layers = [{k: (None if getattr(L, k) is None else dev_f32(getattr(L, k))) for k in keys} for L in prob.layers_r]
    B, C = 3, int(br.cand_offsets[-1])
    kv_total = int((br.kv_end - br.kv_begin).sum())
    ws_b = lib.stca_forward_workspace(B, C, 128, 4, 32, lib.SA_BF16)
    big, ws = _padded(ws_b)
    lib.stca_forward(q, br.cand_offsets, kv, br.kv_begin, br.kv_end, layers, 4, 32, workspace=ws)
    torch.cuda.synchronize()
    assert _intact(big, ws_b)
    ws_b = lib.stca_forward_full_workspace(B, C, kv_total, 128, 4, 32, lib.SA_BF16)
    big, ws = _padded(ws_b)
    lib.stca_forward_full(q, br.cand_offsets, kv, br.kv_begin, br.kv_end, layers, 4, 32, workspace=ws)
    torch.cuda.synchronize()
    assert _intact(big, ws_b)
    ws_b = lib.stca_backward_full_workspace(br.cand_offsets, br.kv_begin, br.kv_end, 128, 4, 32, 2, lib.SA_BF16)
    big, ws = _padded(ws_b)
    dout = dev_f32(np.random.default_rng(5).standard_normal((C, 128)).astype(np.float32))
    lib.stca_backward_full(q, br.cand_offsets, kv, br.kv_begin, br.kv_end, layers, 4, 32, dout, workspace=ws)
    torch.cuda.synchronize()
    lib.poll_device_status()
    assert _intact(big, ws_b)


def test_refine_and_tokenwise_stay_inside_their_workspaces(lib):
    p = make_sa_problem((900, 0, 300), 256, 128, "bf16", seed=805, x_kind="events")
    X = dev_x(p.X, p.dtype)
    layers = [{k: (dev_f32(v) if v is not None else None) for k, v in L.items()} for L in refine_layers(rng_for(806), 2, 128)]
    ws_b = lib.sa_refine_workspace(p.B, p.n_total, p.k, p.d, lib.SA_BF16)
    big, ws = _padded(ws_b)
    lib.sa_refine_forward(X, p.offsets, dev_f32(p.P), layers, workspace=ws)
    torch.cuda.synchronize()
    assert _intact(big, ws_b)
    ws_b = lib.sa_forward_tokenwise_workspace(p.B, p.n_total, p.k, p.d, lib.SA_BF16)
    big, ws = _padded(ws_b)
    lib.sa_forward_tokenwise(X, p.offsets, dev_f32(p.P), dev_f32(p.W_Q), dev_f32(p.W_K), dev_f32(p.W_V), p.eps,
                             workspace=ws)
    torch.cuda.synchronize()
    lib.poll_device_status()
    assert _intact(big, ws_b)


def test_refine_backward_stays_inside_its_buffers(lib):
    """The batched refinement backward (per-user prototypes in both SA backward kernels, E
    drained per user piece into user rows or chunk slots) writes only its workspace and its
    outputs."""
    p = make_sa_problem((900, 0, 300, 2500), 256, 128, "bf16", seed=807, x_kind="events")
    X = dev_x(p.X, p.dtype)
    layers = [{k: (dev_f32(v) if v is not None else None) for k, v in L.items()}
              for L in refine_layers(rng_for(808), 2, 128)]
    ws_b = lib.sa_refine_backward_workspace(p.B, p.n_total, p.k, p.d, 2, lib.SA_BF16)
    big, ws = _padded(ws_b)
    outs = {"dX": _padded_like((p.n_total, p.d), torch.float32), "dP0": _padded_like((p.k, p.d), torch.float32)}
    dsk = dev_f32(np.random.default_rng(9).standard_normal((p.B, p.k, p.d)).astype(np.float32))
    lib.sa_refine_backward(X, p.offsets, dev_f32(p.P), layers, dsk, out={k: v[1] for k, v in outs.items()},
                           workspace=ws)
    torch.cuda.synchronize()
    lib.poll_device_status()
    assert _intact(big, ws_b)
    for k, (b, t) in outs.items():
        assert _intact(b, t.numel() * t.element_size()), k


def test_event_rows_stay_inside_their_buffers(lib):
    """Both event-row entry points (the plain sum and eq. (20)'s fused FFN) write only their
    output rows and, for the fused form, its workspace; a ragged last tile (n not a multiple
    of 128) included."""
    item, action, ids, acts = event_problem(1000, 4096, 128, seed=809)
    t = lambda b: torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16)
    dev = (t(item), t(action), torch.from_numpy(ids).cuda(), torch.from_numpy(acts).cuda())
    xbig, X = _padded_like((len(ids), 128), torch.bfloat16)
    lib.sa_gather_events(*dev, out=X)
    torch.cuda.synchronize()
    lib.poll_device_status()
    assert _intact(xbig, X.numel() * 2)
    W1, W3, W2 = (dev_f32(w) for w in event_ffn_weights(rng_for(810), 128))
    ws_b = lib.sa_gather_events_fused_workspace(action.shape[0], 128, 256)
    wbig, ws = _padded(ws_b)
    xbig, X = _padded_like((len(ids), 128), torch.bfloat16)
    lib.sa_gather_events_fused(*dev, W1, W3, W2, out=X, workspace=ws)
    torch.cuda.synchronize()
    lib.poll_device_status()
    assert _intact(wbig, ws_b)
    assert _intact(xbig, X.numel() * 2)
