"""The allocation-free entry point nf4_layer_error_rank_noalloc.

It exists for callers that cannot allocate device memory where they call it
(fixed device-memory pools sized at start-up, allocator hooks or host callbacks
where cudaMalloc is off-limits, pipelines that cannot take the device-wide
synchronization of cudaMalloc/cudaFree). Its scratch is a fixed array inside the
library, shared by every call, and it has no status word: a layer holding NaN or
+-Inf reports err = NaN and ranks ahead of the finite layers.

The GPU test makes two calls in a row. The first runs on a stack where every
16384-weight chunk of the big layers holds a non-finite weight, so it leaves NaN
partial sums across the array; the second runs on a clean stack that reads the
same part of the array. A partial the second call failed to write would show as
NaN. Both calls are checked against the oracle (errors within 1e-6 relative,
order and keep bit-exact) and the second also against the workspace entry point.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import layer_error
from quantized_lora_fine_b200 import _lib, api, build, synth

ERR_RTOL = 1e-6  # the layer-error tolerance used by the other GPU tests
CHUNK = 16384    # weights per partial sum


def _noalloc(Ws, K, dq):
    lib = _lib.load()
    L = len(Ws)
    dev = Ws[0].device
    ptrs = (ctypes.c_void_p * L)(*[W.data_ptr() for W in Ws])
    numel = (ctypes.c_int64 * L)(*[W.numel() for W in Ws])
    err = torch.full((L,), -1.0, dtype=torch.float64, device=dev)
    order = torch.full((L,), -1, dtype=torch.int32, device=dev)
    keep = torch.full((L,), 7, dtype=torch.uint8, device=dev)
    st = lib.nf4_layer_error_rank_noalloc(L, ptrs, numel, _lib.DTYPE_BF16, _lib.NF4QConfig(64, 1 if dq else 0, 256), K,
                                          err.data_ptr(), order.data_ptr(), keep.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)
    assert st == 0, _lib.STATUS.get(st, st)
    torch.cuda.synchronize()
    return err.cpu().numpy(), order.cpu().numpy(), keep.cpu().numpy()


def _expected(Ws_cpu, bad, K, dq):
    """Oracle errors of the finite layers (NaN for the others), the order with NaN
    layers first by index and then (error desc, index asc), and the keep mask."""
    ref = np.array([np.nan if i in bad else layer_error.layer_error(synth.bf16_bits(W), dq)
                    for i, W in enumerate(Ws_cpu)])
    finite = [i for i in range(len(Ws_cpu)) if i not in bad]
    fin_order = [finite[j] for j in layer_error.rank_layers(ref[finite])]
    order = np.array(sorted(bad) + fin_order, dtype=np.int32)
    return ref, order, layer_error.keep_mask(order, K)


def _check(got, want):
    e, o, k = got
    ref, order, keep = want
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(e), nan), (e, ref)
    nz = ~nan & (ref > 0)
    assert np.all(np.abs(e[nz] - ref[nz]) <= ERR_RTOL * ref[nz])
    assert np.all(e[~nan & (ref == 0)] == 0)
    assert np.array_equal(o, order)
    assert np.array_equal(k, keep)


def _poisoned(W, value, every):
    """A copy of W with `value` at one position in every `every` weights."""
    flat = W.clone().reshape(-1)
    flat[7::every] = value
    return flat.reshape(W.shape)


@pytest.mark.gpu
def test_noalloc_two_calls_against_oracle(cuda_device):
    build.build()
    dq = True
    # call 1: two big layers with a non-finite weight in every chunk, and finite
    # layers between them (75 chunks in all)
    mats = synth.stack_matrices(n_layers=1, linears=(("a", 1024, 512), ("b", 256, 512), ("c", 512, 1024),
                                                     ("d", 128, 384)), seed=3)
    W1 = [synth.stack_weight(m, seed=3) for m in mats]
    W1[0] = _poisoned(W1[0], float("nan"), CHUNK)
    W1[2] = _poisoned(W1[2], float("-inf"), CHUNK)
    bad1 = {0, 2}
    assert sum(-(-W.numel() // CHUNK) for W in W1) == 75
    got1 = _noalloc([W.to(cuda_device) for W in W1], 3, dq)
    _check(got1, _expected(W1, bad1, 3, dq))

    # call 2: a clean stack over part of the same chunk range (64 chunks): every partial it
    # reads held NaN or a finite sum from call 1, so a missed write fails the test
    mats2 = synth.stack_matrices(n_layers=2, linears=(("a", 512, 512), ("b", 64, 1024), ("c", 256, 768)), seed=4)
    W2 = [synth.stack_weight(m, seed=4) for m in mats2]
    assert sum(-(-W.numel() // CHUNK) for W in W2) == 64
    g2 = [W.to(cuda_device) for W in W2]
    got2 = _noalloc(g2, 2, dq)
    _check(got2, _expected(W2, set(), 2, dq))
    e_ws, o_ws, k_ws = api.layer_error_rank(g2, 2, double_quant=dq)
    torch.cuda.synchronize()
    assert np.all(np.abs(got2[0] - e_ws.cpu().numpy()) <= ERR_RTOL * np.abs(e_ws.cpu().numpy()))
    assert np.array_equal(got2[1], o_ws.cpu().numpy())
    assert np.array_equal(got2[2], k_ws.cpu().numpy())


def test_noalloc_refuses_oversize_on_host():
    build.build()
    lib = _lib.load()
    ptrs = (ctypes.c_void_p * 1)(0x100000)
    numel = (ctypes.c_int64 * 1)((1 << 20) * 16384 + 64)  # one chunk past the fixed array
    st = lib.nf4_layer_error_rank_noalloc(1, ptrs, numel, _lib.DTYPE_BF16, _lib.NF4QConfig(64, 0, 256), 0,
                                          0x1000, 0x1000, 0x1000, None)
    assert st == 2  # QLORA_ERR_SHAPE, before any device work
