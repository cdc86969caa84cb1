"""Torch-facing binding of the C ABI: tensors in, tensors out.

PyTorch supplies device memory and the current stream; the arithmetic of every
step runs in libqlora_b200.so. Functions mirror the C entry points:

    quantize(W, double_quant)              -> NF4Weight        (nf4_quantize)
    dequantize(w)                          -> bf16 tensor      (nf4_dequantize)
    linear_fwd(w, X, L1, L2, scale)        -> (Y, T)           (qlora_linear_fwd)
    linear_bwd(w, X, dY, L1, L2, scale, T) -> (dX, dL1, dL2)   (qlora_linear_bwd)
    layer_error_rank(Ws, K, double_quant)  -> (err, order, keep) (nf4_layer_error_rank)
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import List, Optional, Sequence, Tuple

import torch

from . import _lib
from ._lib import DTYPE_BF16, DTYPE_F32, NF4QConfig, QLoraWeight, check


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _need(t: torch.Tensor, dtype, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


class Workspace:
    """A grow-only device scratch buffer per (device, stream), zeroed at allocation
    (its first 4 bytes are the library's sticky device status word). Calls on
    different streams get different buffers, so they may run at the same time."""

    _bufs = {}

    @classmethod
    def get(cls, nbytes: int, device: torch.device) -> torch.Tensor:
        dev = torch.device(device)
        idx = dev.index if dev.index is not None else torch.cuda.current_device()
        key = (idx, torch.cuda.current_stream(idx).cuda_stream)
        buf = cls._bufs.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=dev)
            cls._bufs[key] = buf
        return buf

    @classmethod
    def all(cls, index: int):
        return [b for (i, _), b in cls._bufs.items() if i == index]


def read_status(ws: torch.Tensor) -> int:
    return _lib.load().qlora_read_status(ctypes.c_void_p(ws.data_ptr()), ctypes.c_void_p(_stream()))


def reset_status(ws: torch.Tensor) -> None:
    """Clears the status word and the tile counters / block flags after it (an
    interrupted GEMM can leave those set)."""
    check(_lib.load().qlora_reset_workspace(ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size(),
                                            ctypes.c_void_p(_stream())), "reset_status")


@dataclasses.dataclass
class NF4Weight:
    """An NF4 (or protected bf16) frozen weight stored out x in."""
    out: int
    inp: int
    double_quant: bool
    codes: Optional[torch.Tensor] = None
    absmax: Optional[torch.Tensor] = None
    absmax_q: Optional[torch.Tensor] = None
    absmax2: Optional[torch.Tensor] = None
    w_bf16: Optional[torch.Tensor] = None

    @property
    def is_bf16(self) -> bool:
        return self.w_bf16 is not None

    @staticmethod
    def protected(W: torch.Tensor) -> "NF4Weight":
        _need(W, torch.bfloat16, "W")
        return NF4Weight(W.shape[0], W.shape[1], False, w_bf16=W)

    def c_struct(self) -> QLoraWeight:
        s = QLoraWeight()
        s.out, s.in_ = self.out, self.inp
        s.q = NF4QConfig(64, 1 if self.double_quant else 0, 256)
        s.is_bf16 = 1 if self.is_bf16 else 0
        s.codes = _ptr(self.codes)
        s.absmax = _ptr(self.absmax)
        s.absmax_q = _ptr(self.absmax_q)
        s.absmax2 = _ptr(self.absmax2)
        s.w_bf16 = _ptr(self.w_bf16)
        return s


def quantize(W: torch.Tensor, double_quant: bool = False, keep_absmax: bool = False,
             codes: Optional[torch.Tensor] = None, absmax: Optional[torch.Tensor] = None) -> NF4Weight:
    """NF4-quantize a 2-D bf16 or fp32 CUDA tensor stored out x in. `codes` and
    `absmax` may be given as preallocated outputs (no double quant)."""
    if W.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("W must be bf16 or fp32")
    _need(W, W.dtype, "W")
    lib = _lib.load()
    out, inp = W.shape
    n = W.numel()
    nb = (n + 63) // 64
    dev = W.device
    if codes is None:
        codes = torch.empty((n + 1) // 2, dtype=torch.uint8, device=dev)
    elif codes.numel() < (n + 1) // 2 or codes.dtype != torch.uint8 or not codes.is_contiguous():
        raise ValueError("codes: need a contiguous uint8 tensor of (numel + 1) // 2 bytes")
    if absmax is None:
        absmax = torch.empty(nb, dtype=torch.float32, device=dev) if (not double_quant or keep_absmax) else None
    elif absmax.numel() < nb or absmax.dtype != torch.float32 or not absmax.is_contiguous():
        raise ValueError("absmax: need a contiguous fp32 tensor of one value per 64 weights")
    absmax_q = torch.empty(nb, dtype=torch.uint8, device=dev) if double_quant else None
    absmax2 = torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev) if double_quant else None
    ws = Workspace.get(lib.nf4_quantize_workspace_size(n), dev)
    check(lib.nf4_quantize(_ptr(W), DTYPE_BF16 if W.dtype == torch.bfloat16 else DTYPE_F32, out, inp,
                           NF4QConfig(64, 1 if double_quant else 0, 256), _ptr(codes), _ptr(absmax),
                           _ptr(absmax_q), _ptr(absmax2), _ptr(ws), ws.numel(), _stream()), "nf4_quantize")
    return NF4Weight(out, inp, double_quant, codes=codes, absmax=absmax, absmax_q=absmax_q, absmax2=absmax2)


def quantize_batch(Ws: Sequence[torch.Tensor], double_quant: bool = False, keep_absmax: bool = False,
                   outs: Optional[Sequence[NF4Weight]] = None) -> list:
    """quantize() for up to 512 bf16 matrices in one launch (same bits per matrix).
    `outs` may supply preallocated weights (same shapes and settings)."""
    lib = _lib.load()
    L = len(Ws)
    for i, W in enumerate(Ws):
        _need(W, torch.bfloat16, f"W[{i}]")
    dev = Ws[0].device
    if outs is None:
        outs = []
        for W in Ws:
            n = W.numel()
            nb = (n + 63) // 64
            outs.append(NF4Weight(
                W.shape[0], W.shape[1], double_quant,
                codes=torch.empty((n + 1) // 2, dtype=torch.uint8, device=dev),
                absmax=torch.empty(nb, dtype=torch.float32, device=dev) if (not double_quant or keep_absmax) else None,
                absmax_q=torch.empty(nb, dtype=torch.uint8, device=dev) if double_quant else None,
                absmax2=torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev) if double_quant else None))
    ptrs = (ctypes.c_void_p * L)(*[W.data_ptr() for W in Ws])
    numel = (ctypes.c_int64 * L)(*[W.numel() for W in Ws])

    def arr(name):
        return (ctypes.c_void_p * L)(*[(_ptr(getattr(o, name)) or 0) for o in outs])

    ws = Workspace.get(lib.nf4_quantize_workspace_size(0), dev)
    check(lib.nf4_quantize_batch(L, ptrs, numel, DTYPE_BF16, NF4QConfig(64, 1 if double_quant else 0, 256),
                                 arr("codes"), arr("absmax"), arr("absmax_q"), arr("absmax2"), _ptr(ws), ws.numel(),
                                 _stream()), "nf4_quantize_batch")
    return list(outs)


def dequantize(w: NF4Weight) -> torch.Tensor:
    lib = _lib.load()
    out = torch.empty((w.out, w.inp), dtype=torch.bfloat16, device=w.codes.device)
    cs = w.c_struct()
    check(lib.nf4_dequantize(ctypes.byref(cs), _ptr(out), _stream()), "nf4_dequantize")
    return out


def quantize_residual(W: torch.Tensor, w1: NF4Weight, double_quant: bool = False,
                      keep_absmax: bool = False) -> NF4Weight:
    """Second NF4 stage of W over the first stage w1: quantizes
    R = fp32_rn(W - fp32_rn(c1 a1)) as quantize() would quantize an fp32 tensor."""
    _need(W, torch.bfloat16, "W")
    if tuple(W.shape) != (w1.out, w1.inp):
        raise ValueError("W must have the first stage's shape")
    lib = _lib.load()
    dev = W.device
    n = W.numel()
    nb = (n + 63) // 64
    o = NF4Weight(w1.out, w1.inp, double_quant,
                  codes=torch.empty((n + 1) // 2, dtype=torch.uint8, device=dev),
                  absmax=torch.empty(nb, dtype=torch.float32, device=dev) if (not double_quant or keep_absmax) else None,
                  absmax_q=torch.empty(nb, dtype=torch.uint8, device=dev) if double_quant else None,
                  absmax2=torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev) if double_quant else None)
    ws = Workspace.get(lib.nf4_quantize_residual_workspace_size(n), dev)
    cs = w1.c_struct()
    check(lib.nf4_quantize_residual(_ptr(W), ctypes.byref(cs), NF4QConfig(64, 1 if double_quant else 0, 256),
                                    _ptr(o.codes), _ptr(o.absmax), _ptr(o.absmax_q), _ptr(o.absmax2), _ptr(ws),
                                    ws.numel(), _stream()), "nf4_quantize_residual")
    return o


def dequantize_two_stage(w1: NF4Weight, w2: NF4Weight) -> torch.Tensor:
    """bf16_rn(fp32_rn(v1 + v2)) of two NF4 stages, stored out x in."""
    lib = _lib.load()
    out = torch.empty((w1.out, w1.inp), dtype=torch.bfloat16, device=w1.codes.device)
    c1, c2 = w1.c_struct(), w2.c_struct()
    check(lib.nf4_dequantize_two_stage(ctypes.byref(c1), ctypes.byref(c2), _ptr(out), _stream()),
          "nf4_dequantize_two_stage")
    return out


def lora_merge(w: NF4Weight, L1: torch.Tensor, L2: torch.Tensor, scale: float) -> torch.Tensor:
    """bf16 [out x in] = W_hat + scale (L1 L2)^T (a negative scale unmerges)."""
    _need(L1, torch.bfloat16, "L1")
    _need(L2, torch.bfloat16, "L2")
    lib = _lib.load()
    dev = L1.device
    out = torch.empty((w.out, w.inp), dtype=torch.bfloat16, device=dev)
    cs = w.c_struct()
    check(lib.qlora_lora_merge(ctypes.byref(cs), _ptr(L1), _ptr(L2), L1.shape[1], float(scale), _ptr(out), _stream()),
          "qlora_lora_merge")
    return out


def lora_merge_requantize(w: NF4Weight, L1: torch.Tensor, L2: torch.Tensor, scale: float,
                          double_quant: bool = False, keep_absmax: bool = False) -> NF4Weight:
    """The merged weight W_hat + scale (L1 L2)^T, NF4-quantized as quantize() would."""
    _need(L1, torch.bfloat16, "L1")
    _need(L2, torch.bfloat16, "L2")
    lib = _lib.load()
    dev = L1.device
    n = w.out * w.inp
    nb = (n + 63) // 64
    o = NF4Weight(w.out, w.inp, double_quant,
                  codes=torch.empty((n + 1) // 2, dtype=torch.uint8, device=dev),
                  absmax=torch.empty(nb, dtype=torch.float32, device=dev) if (not double_quant or keep_absmax) else None,
                  absmax_q=torch.empty(nb, dtype=torch.uint8, device=dev) if double_quant else None,
                  absmax2=torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev) if double_quant else None)
    ws = Workspace.get(lib.qlora_lora_merge_requantize_workspace_size(w.out, w.inp), dev)
    cs = w.c_struct()
    check(lib.qlora_lora_merge_requantize(ctypes.byref(cs), _ptr(L1), _ptr(L2), L1.shape[1], float(scale),
                                          NF4QConfig(64, 1 if double_quant else 0, 256), _ptr(o.codes),
                                          _ptr(o.absmax), _ptr(o.absmax_q), _ptr(o.absmax2), _ptr(ws), ws.numel(),
                                          _stream()), "qlora_lora_merge_requantize")
    return o


def linear_fwd(w: NF4Weight, X: torch.Tensor, L1: torch.Tensor, L2: torch.Tensor, scale: float,
               save_T: bool = True, Y: Optional[torch.Tensor] = None,
               T: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Y = X W^T + s (X L1) L2. With T given (from lora_down), X L1 is not
    recomputed and T is returned as is."""
    for t, nm in ((X, "X"), (L1, "L1"), (L2, "L2")):
        _need(t, torch.bfloat16, nm)
    lib = _lib.load()
    M, r = X.shape[0], L1.shape[1]
    dev = X.device
    if Y is None:
        Y = torch.empty((M, w.out), dtype=torch.bfloat16, device=dev)
    ws = Workspace.get(lib.qlora_fwd_workspace_size(M, w.out, w.inp, r), dev)
    cs = w.c_struct()
    if T is not None:
        _need(T, torch.bfloat16, "T")
        check(lib.qlora_linear_fwd_t(ctypes.byref(cs), _ptr(X), M, _ptr(T), _ptr(L2), r, float(scale), _ptr(Y),
                                     _ptr(ws), ws.numel(), _stream()), "qlora_linear_fwd_t")
        return Y, T
    T = torch.empty((M, r), dtype=torch.bfloat16, device=dev) if save_T else None
    check(lib.qlora_linear_fwd(ctypes.byref(cs), _ptr(X), M, _ptr(L1), _ptr(L2), r, float(scale), _ptr(Y), _ptr(T),
                               _ptr(ws), ws.numel(), _stream()), "qlora_linear_fwd")
    return Y, T


def lora_down(X: torch.Tensor, L1: torch.Tensor, T: Optional[torch.Tensor] = None) -> torch.Tensor:
    """T = X L1 (bf16 [M x r]): the LoRA down-projection alone, for overlapping it
    with other work; pass the result to linear_fwd(..., T=T)."""
    _need(X, torch.bfloat16, "X")
    _need(L1, torch.bfloat16, "L1")
    lib = _lib.load()
    M, r = X.shape[0], L1.shape[1]
    dev = X.device
    if T is None:
        T = torch.empty((M, r), dtype=torch.bfloat16, device=dev)
    ws = Workspace.get(lib.qlora_lora_down_workspace_size(M, X.shape[1], r), dev)
    check(lib.qlora_lora_down(_ptr(X), M, X.shape[1], _ptr(L1), r, _ptr(T), _ptr(ws), ws.numel(), _stream()),
          "qlora_lora_down")
    return T


def linear_bwd(w: NF4Weight, X: torch.Tensor, dY: torch.Tensor, L1: torch.Tensor, L2: torch.Tensor, scale: float,
               T: Optional[torch.Tensor] = None, need_dX: bool = True):
    for t, nm in ((X, "X"), (dY, "dY"), (L1, "L1"), (L2, "L2")):
        _need(t, torch.bfloat16, nm)
    lib = _lib.load()
    M, r = X.shape[0], L1.shape[1]
    dev = X.device
    dX = torch.empty((M, w.inp), dtype=torch.bfloat16, device=dev) if need_dX else None
    dL1 = torch.empty((w.inp, r), dtype=torch.float32, device=dev)
    dL2 = torch.empty((r, w.out), dtype=torch.float32, device=dev)
    ws = Workspace.get(lib.qlora_bwd_workspace_size(M, w.out, w.inp, r), dev)
    cs = w.c_struct()
    check(lib.qlora_linear_bwd(ctypes.byref(cs), _ptr(X), _ptr(dY), M, _ptr(L1), _ptr(L2), r, float(scale), _ptr(T),
                               _ptr(dX), _ptr(dL1), _ptr(dL2), _ptr(ws), ws.numel(), _stream()), "qlora_linear_bwd")
    return dX, dL1, dL2


def layer_error_rank(Ws: Sequence[torch.Tensor], K: int, double_quant: bool = False):
    lib = _lib.load()
    L = len(Ws)
    for i, W in enumerate(Ws):
        _need(W, torch.bfloat16, f"W[{i}]")
    dev = Ws[0].device
    ptrs = (ctypes.c_void_p * L)(*[W.data_ptr() for W in Ws])
    numel = (ctypes.c_int64 * L)(*[W.numel() for W in Ws])
    err = torch.empty(L, dtype=torch.float64, device=dev)
    order = torch.empty(L, dtype=torch.int32, device=dev)
    keep = torch.empty(L, dtype=torch.uint8, device=dev)
    ws = Workspace.get(lib.nf4_layer_error_rank_workspace_size(L, numel), dev)
    check(lib.nf4_layer_error_rank(L, ptrs, numel, DTYPE_BF16, NF4QConfig(64, 1 if double_quant else 0, 256), K,
                                   _ptr(err), _ptr(order), _ptr(keep), _ptr(ws), ws.numel(), _stream()),
          "nf4_layer_error_rank")
    return err, order, keep


def layer_error_rank_budget(Ws: Sequence[torch.Tensor], budget_bytes: int, double_quant: bool = False):
    """layer_error_rank with K from a memory budget: the longest prefix of the
    ranking whose bf16 copies add at most budget_bytes to the NF4 storage.
    Returns (err, order, keep, K) with K a one-element device int32 tensor."""
    lib = _lib.load()
    L = len(Ws)
    for i, W in enumerate(Ws):
        _need(W, torch.bfloat16, f"W[{i}]")
    dev = Ws[0].device
    ptrs = (ctypes.c_void_p * L)(*[W.data_ptr() for W in Ws])
    numel = (ctypes.c_int64 * L)(*[W.numel() for W in Ws])
    err = torch.empty(L, dtype=torch.float64, device=dev)
    order = torch.empty(L, dtype=torch.int32, device=dev)
    keep = torch.empty(L, dtype=torch.uint8, device=dev)
    K = torch.empty(1, dtype=torch.int32, device=dev)
    ws = Workspace.get(lib.nf4_layer_error_rank_workspace_size(L, numel), dev)
    check(lib.nf4_layer_error_rank_budget(L, ptrs, numel, DTYPE_BF16, NF4QConfig(64, 1 if double_quant else 0, 256),
                                          int(budget_bytes), _ptr(err), _ptr(order), _ptr(keep), _ptr(K), _ptr(ws),
                                          ws.numel(), _stream()), "nf4_layer_error_rank_budget")
    return err, order, keep, K


def k_from_fraction(num: int, den: int, n_layers: int) -> int:
    """K = round half up of (num / den) * n_layers (host only)."""
    k = ctypes.c_int32(0)
    check(_lib.load().nf4_k_from_fraction(int(num), int(den), int(n_layers), ctypes.byref(k)), "nf4_k_from_fraction")
    return int(k.value)


def quantize_error_rank(Ws: Sequence[torch.Tensor], K: int, double_quant: bool = False, keep_absmax: bool = False,
                        outs: Optional[Sequence[NF4Weight]] = None):
    """The allocation pass fused with the quantization: one read of every matrix
    gives (err, order, keep) as layer_error_rank and every layer's NF4Weight as
    quantize. `outs` may supply preallocated weights (same shapes and settings)."""
    lib = _lib.load()
    L = len(Ws)
    for i, W in enumerate(Ws):
        _need(W, torch.bfloat16, f"W[{i}]")
    dev = Ws[0].device
    if outs is None:
        outs = []
        for W in Ws:
            n = W.numel()
            nb = n // 64
            outs.append(NF4Weight(
                W.shape[0], W.shape[1], double_quant,
                codes=torch.empty(n // 2, dtype=torch.uint8, device=dev),
                absmax=torch.empty(nb, dtype=torch.float32, device=dev) if (not double_quant or keep_absmax) else None,
                absmax_q=torch.empty(nb, dtype=torch.uint8, device=dev) if double_quant else None,
                absmax2=torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev) if double_quant else None))
    ptrs = (ctypes.c_void_p * L)(*[W.data_ptr() for W in Ws])
    numel = (ctypes.c_int64 * L)(*[W.numel() for W in Ws])
    arr = lambda name: (ctypes.c_void_p * L)(*[_ptr(getattr(w, name)) for w in outs])
    err = torch.empty(L, dtype=torch.float64, device=dev)
    order = torch.empty(L, dtype=torch.int32, device=dev)
    keep = torch.empty(L, dtype=torch.uint8, device=dev)
    ws = Workspace.get(lib.nf4_layer_error_rank_workspace_size(L, numel), dev)
    check(lib.nf4_quantize_error_rank(L, ptrs, numel, DTYPE_BF16, NF4QConfig(64, 1 if double_quant else 0, 256), K,
                                      arr("codes"), arr("absmax"), arr("absmax_q"), arr("absmax2"),
                                      _ptr(err), _ptr(order), _ptr(keep), _ptr(ws), ws.numel(), _stream()),
          "nf4_quantize_error_rank")
    return err, order, keep, list(outs)


def rank_errors(err: torch.Tensor, K: int):
    """(order, keep) of per-layer errors already on the device (fp64): the ranking
    step alone, (error desc, index asc), NaN first."""
    _need(err, torch.float64, "err")
    lib = _lib.load()
    L = err.numel()
    order = torch.empty(L, dtype=torch.int32, device=err.device)
    keep = torch.empty(L, dtype=torch.uint8, device=err.device)
    check(lib.nf4_rank_errors(L, _ptr(err), int(K), _ptr(order), _ptr(keep), _stream()), "nf4_rank_errors")
    return order, keep


def status() -> int:
    """First nonzero device status word among this device's workspaces (one per
    stream the library was called on); synchronizes."""
    idx = torch.cuda.current_device()
    dev = torch.device("cuda", idx)
    for ws in Workspace.all(idx) or [Workspace.get(256, dev)]:
        st = read_status(ws)
        if st:
            return st
    return 0
