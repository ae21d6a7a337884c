"""The N>1 host path on CPU: two gloo ranks each take a contiguous shard of
users, compute the weight gradients of their shard with the oracle and sum
them with the same all-reduce the GPU step uses.  The result must equal the
gradients of the whole batch (weights are shared, users are independent)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sa_inputs import make_sa_problem
from sketch_attention_b200.dist import WEIGHT_GRADS, allreduce_weight_grads, shard_offsets, shard_users

LENGTHS = [37, 0, 80, 5, 61]
K, D = 8, 16
NAMES = ("dX",) + WEIGHT_GRADS


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    return make_sa_problem(LENGTHS, K, D, "f32", seed=11, with_grad=True)


def _rank(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        pr = _problem()
        u0, u1 = shard_users(pr.B, rank, world)
        off = shard_offsets(pr.offsets, u0, u1)
        X = pr.X[pr.offsets[u0]:pr.offsets[u1]]
        g = dict(zip(NAMES, oracle.sa_backward(X, off, pr.P, pr.W_Q, pr.W_K, pr.W_V, pr.eps,
                                               pr.dS[u0:u1])))
        t = {n: torch.from_numpy(np.ascontiguousarray(g[n])) for n in WEIGHT_GRADS}
        allreduce_weight_grads(t)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), **{n: t[n].numpy() for n in WEIGHT_GRADS},
                 dX=np.asarray(g["dX"]), u0=u0, u1=u1)
    finally:
        dist.destroy_process_group()


def test_shard_users_covers_batch():
    for B in (0, 1, 5, 8, 33):
        for world in (1, 2, 3, 8):
            parts = [shard_users(B, r, world) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == B
            assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_users(4, 2, 2)


def test_two_gloo_ranks_match_whole_batch(tmp_path):
    world = 2
    mp.start_processes(_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    pr = _problem()
    ref = dict(zip(NAMES, oracle.sa_backward(pr.X, pr.offsets, pr.P, pr.W_Q, pr.W_K, pr.W_V,
                                             pr.eps, pr.dS)))
    dX = []
    for r in range(world):
        got = np.load(tmp_path / f"r{r}.npz")
        for n in WEIGHT_GRADS:
            np.testing.assert_allclose(got[n], ref[n], rtol=1e-10, atol=1e-12)
        dX.append(got["dX"])
    # the token gradients need no exchange: the shards' dX concatenate to the batch's
    np.testing.assert_allclose(np.concatenate(dX), ref["dX"], rtol=1e-10, atol=1e-12)
