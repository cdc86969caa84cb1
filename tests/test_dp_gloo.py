"""Data-parallel exchange of the adapter gradients, on CPU with two gloo ranks.

Each rank holds the same frozen weight and adapters and its own token shard; the
only exchange is the sum of dL1 and dL2 across ranks (what bench.py does with
NCCL for N > 1 GPUs). The summed gradients must equal the gradients of the
concatenated batch; Y, T, U and dX stay local.
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import lora

WORLD = 2


def _worker(rank, port, result_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        rng = np.random.default_rng(0)
        M, h, o, r, s = 64, 32, 48, 4, 2.0
        X = rng.standard_normal((M, h)); W = rng.standard_normal((o, h)) * 0.1
        L1 = rng.standard_normal((h, r)) * 0.1; L2 = rng.standard_normal((r, o)) * 0.1
        dY = rng.standard_normal((M, o))
        sl = slice(rank * M // WORLD, (rank + 1) * M // WORLD)
        g = lora.backward(X[sl], W, L1, L2, dY[sl], s)
        dL1 = torch.from_numpy(g["dL1"]).clone()
        dL2 = torch.from_numpy(g["dL2"]).clone()
        dist.all_reduce(dL1)
        dist.all_reduce(dL2)
        full = lora.backward(X, W, L1, L2, dY, s)
        ok = (np.allclose(dL1.numpy(), full["dL1"], rtol=1e-12, atol=1e-12)
              and np.allclose(dL2.numpy(), full["dL2"], rtol=1e-12, atol=1e-12)
              and np.allclose(g["dX"], full["dX"][sl], rtol=1e-12, atol=1e-12))
        result_q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


def test_gradient_allreduce_equals_full_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    res = dict(q.get(timeout=5) for _ in range(WORLD))
    assert all(p.exitcode == 0 for p in procs)
    assert res == {0: True, 1: True}
