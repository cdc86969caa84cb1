"""The allocation-free entry point nf4_layer_error_rank_noalloc.

It exists for callers that cannot allocate device memory where they call it
(fixed device-memory pools sized at start-up, allocator hooks or host callbacks
where cudaMalloc is off-limits, pipelines that cannot take the device-wide
synchronization of cudaMalloc/cudaFree). Its scratch is a fixed array inside the
library, so these tests check that it gives the same results as the workspace
entry point, twice in a row (the second call must not see the first call's
leftovers), and that oversize requests are refused on the host.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from quantized_lora_fine_b200 import _lib, api, build, synth

ERR_RTOL = 1e-6  # the layer-error tolerance used by the other GPU tests


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
    return err, order, keep


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice(cuda_device):
    build.build()
    stacks = [
        ([synth.stack_weight(m) for m in synth.stack_matrices(
            n_layers=3, linears=(("a", 256, 512), ("b", 512, 256), ("c", 128, 384)), seed=0)], 4, False),
        ([synth.stack_weight(m, seed=1) for m in synth.stack_matrices(
            n_layers=2, linears=(("a", 1024, 256), ("b", 64, 1024)), seed=1)], 1, True),
    ]
    for Ws_cpu, K, dq in stacks:  # two calls in a row, different sizes
        Ws = [W.to(cuda_device) for W in Ws_cpu]
        e_ref, o_ref, k_ref = api.layer_error_rank(Ws, K, double_quant=dq)
        e, o, k = _noalloc(Ws, K, dq)
        torch.cuda.synchronize()
        e_ref, e = e_ref.cpu().numpy(), e.cpu().numpy()
        assert np.all(np.abs(e - e_ref) <= ERR_RTOL * np.abs(e_ref))
        assert np.array_equal(o.cpu().numpy(), o_ref.cpu().numpy())
        assert np.array_equal(k.cpu().numpy(), k_ref.cpu().numpy())


def test_noalloc_refuses_oversize_on_host():
    build.build()
    lib = _lib.load()
    ptrs = (ctypes.c_void_p * 1)(0x100000)
    numel = (ctypes.c_int64 * 1)((1 << 20) * 16384 + 64)  # one chunk past the fixed array
    st = lib.nf4_layer_error_rank_noalloc(1, ptrs, numel, _lib.DTYPE_BF16, _lib.NF4QConfig(64, 0, 256), 0,
                                          0x1000, 0x1000, 0x1000, None)
    assert st == 2  # QLORA_ERR_SHAPE, before any device work
