"""The allocation pass over several ranks (CPU, gloo): matrices sharded by element
count, each rank scores its own (here with the oracle standing in for a GPU's error
pass), one all-reduce of the zero-padded fp64 error vector, and the same ranking on
every rank. The result must equal the unsharded oracle's errors, order and keep mask
on every rank."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import layer_error
from quantized_lora_fine_b200 import dist as qdist
from quantized_lora_fine_b200 import synth

LINEARS = (("a", 256, 512), ("b", 512, 256), ("c", 128, 384), ("d", 64, 1024))


def _oracle_errors(Ws):
    return torch.tensor([layer_error.layer_error(synth.bf16_bits(W), True) for W in Ws], dtype=torch.float64)


def _oracle_rank(err, K):
    order = layer_error.rank_layers(err.numpy())
    return torch.from_numpy(order), torch.from_numpy(layer_error.keep_mask(order, K))


def test_shard_by_numel_balances_and_covers():
    rng = np.random.default_rng(0)
    for world in (1, 2, 3, 4, 8):
        numel = [int(x) for x in rng.integers(1, 10 ** 6, 57)]
        own = qdist.shard_by_numel(numel, world)
        assert len(own) == len(numel) and set(own) <= set(range(world))
        load = [sum(n for n, o in zip(numel, own) if o == r) for r in range(world)]
        assert max(load) - min(load) <= max(numel)
        assert own == qdist.shard_by_numel(numel, world)          # deterministic
    # the 7 linear shapes of a Llama-7B layer over 2 ranks: q,k,v,o on one side do not
    # outweigh gate/up/down on the other by more than one matrix
    numel = [4096 * 4096] * 4 + [11008 * 4096] * 3
    own = qdist.shard_by_numel(numel, 2)
    load = [sum(n for n, o in zip(numel, own) if o == r) for r in range(2)]
    assert abs(load[0] - load[1]) <= 11008 * 4096


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mats = synth.stack_matrices(n_layers=3, linears=LINEARS, seed=5)
        Ws = [synth.stack_weight(m) for m in mats]
        numel = [W.numel() for W in Ws]
        owners = qdist.shard_by_numel(numel, world)
        mine = {i: Ws[i] for i, o in enumerate(owners) if o == rank}
        err, order, keep = qdist.sharded_layer_error_rank(mine, numel, 4, double_quant=True,
                                                          errors_fn=_oracle_errors, rank_fn=_oracle_rank)
        ref = _oracle_errors(Ws)
        ref_order, ref_keep = _oracle_rank(ref, 4)
        ok = (torch.equal(err, ref) and torch.equal(order, ref_order) and torch.equal(keep, ref_keep)
              and len(mine) > 0)
        q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_error_pass_equals_unsharded(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    res = dict(q.get(timeout=5) for _ in range(world))
    assert all(p.exitcode == 0 for p in procs)
    assert res == {r: True for r in range(world)}
