"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module only draws random numbers and rounds them to bf16 with torch's own
cast. It holds none of the method's arithmetic (no NF4 code table, no absmax,
no GEMM), so the CPU oracle and the CUDA path can both consume its tensors
without sharing any implementation of the method.

Stream convention (one independent generator per tensor role, offset by a
matrix index so that stacked layers get their own draws):

    W = 1, X = 2, L1 = 3, L2 = 4, dY = 5, per-layer (nu, scale) draws = 6

Value distributions follow the workload descriptions: activations and output
gradients ~ N(0, 1); Gaussian weights ~ N(0, 0.02^2); Student-t weights
``scale * t_nu``; LoRA factors ~ N(0, 0.01^2). The pages fine-tune real
checkpoints on public datasets; none of those are used here, only tensors of
the same shapes.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

STREAM_W, STREAM_X, STREAM_L1, STREAM_L2, STREAM_DY, STREAM_LAYER = 1, 2, 3, 4, 5, 6


def _torch_generator(seed: int, stream: int, index: int, device: str) -> torch.Generator:
    state = np.random.SeedSequence([int(seed), int(stream), int(index)]).generate_state(1, np.uint64)[0]
    g = torch.Generator(device=device)
    g.manual_seed(int(state) & ((1 << 63) - 1))
    return g


def normal_bf16(shape: Sequence[int], std: float, seed: int, stream: int, index: int = 0,
                device: str = "cpu") -> torch.Tensor:
    """bf16 tensor ~ N(0, std^2); draws in fp32, rounded by torch's bf16 cast."""
    g = _torch_generator(seed, stream, index, device)
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def student_t_bf16(shape: Sequence[int], nu: float, scale: float, seed: int, stream: int,
                   index: int = 0, device: str = "cpu") -> torch.Tensor:
    """bf16 tensor ``scale * t_nu`` (Student-t with nu degrees of freedom).

    t = z / sqrt(v / nu) with z ~ N(0,1) and v ~ chi2(nu) = 2 * Gamma(nu/2, 1).
    Drawn in fp32 and rounded by torch's bf16 cast.
    """
    g = _torch_generator(seed, stream, index, device)
    z = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    conc = torch.full(tuple(shape), nu / 2.0, device=device, dtype=torch.float32)
    # torch._standard_gamma takes no generator; reseed the default one from our stream.
    gseed = int(torch.randint(0, 2**62, (1,), generator=g, device=device).item())
    with torch.random.fork_rng(devices=[torch.device(device)] if device != "cpu" else []):
        torch.manual_seed(gseed)
        v = torch._standard_gamma(conc).mul_(2.0)
    del conc
    t = z.div_(v.div_(nu).sqrt_())
    del v
    return t.mul_(scale).to(torch.bfloat16)


def layer_draws(n_matrices: int, seed: int, nu_range=(3.0, 30.0),
                scale_range=(0.005, 0.05)) -> List[Tuple[float, float]]:
    """One (nu, scale) pair per matrix, uniform on the given ranges, from stream 6."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), STREAM_LAYER])))
    out = []
    for _ in range(n_matrices):
        nu = float(rng.uniform(*nu_range))
        sc = float(rng.uniform(*scale_range))
        out.append((nu, sc))
    return out


# --------------------------------------------------------------------------- workloads

@dataclasses.dataclass(frozen=True)
class LinearCase:
    """One NF4-LoRA linear: W is stored out x in (nn.Linear layout)."""
    name: str
    M: int
    out: int
    inp: int
    r: int
    alpha: float
    double_quant: bool
    w_dist: str = "normal"      # "normal" (std w_std) or "t" (nu, w_std as scale)
    w_std: float = 0.02
    nu: float = 5.0
    seed: int = 0
    index: int = 0              # matrix index for stream offsets

    @property
    def scale(self) -> float:
        return self.alpha / self.r

    def make(self, device: str = "cpu", with_dy: bool = True):
        W = (normal_bf16((self.out, self.inp), self.w_std, self.seed, STREAM_W, self.index, device)
             if self.w_dist == "normal" else
             student_t_bf16((self.out, self.inp), self.nu, self.w_std, self.seed, STREAM_W, self.index, device))
        X = normal_bf16((self.M, self.inp), 1.0, self.seed, STREAM_X, self.index, device)
        L1 = normal_bf16((self.inp, self.r), 0.01, self.seed, STREAM_L1, self.index, device)
        L2 = normal_bf16((self.r, self.out), 0.01, self.seed, STREAM_L2, self.index, device)
        dY = normal_bf16((self.M, self.out), 1.0, self.seed, STREAM_DY, self.index, device) if with_dy else None
        return dict(W=W, X=X, L1=L1, L2=L2, dY=dY)


def case_small(seed: int = 0) -> LinearCase:
    """Single linear, h = o = 512, M = 256, rank 8, alpha 16, fp32 absmax, N(0, 0.02^2) weights."""
    return LinearCase("single-512", M=256, out=512, inp=512, r=8, alpha=16.0, double_quant=False, seed=seed)


def case_q_proj(seed: int = 0, M: int = 8192) -> LinearCase:
    """Llama-7B q_proj shape: W 4096 x 4096 with double-quant, X 8192 x 4096, rank 16, alpha 32."""
    return LinearCase("llama7b-q_proj", M=M, out=4096, inp=4096, r=16, alpha=32.0, double_quant=True, seed=seed)


def cases_mlp(seed: int = 0, M: int = 8192) -> List[LinearCase]:
    """Llama-7B MLP: gate/up 4096 -> 11008, down 11008 -> 4096; Student-t(5) * 0.02; rank 64, alpha 128."""
    return [
        LinearCase("llama7b-gate", M=M, out=11008, inp=4096, r=64, alpha=128.0, double_quant=False,
                   w_dist="t", nu=5.0, seed=seed, index=0),
        LinearCase("llama7b-up", M=M, out=11008, inp=4096, r=64, alpha=128.0, double_quant=False,
                   w_dist="t", nu=5.0, seed=seed, index=1),
        LinearCase("llama7b-down", M=M, out=4096, inp=11008, r=64, alpha=128.0, double_quant=False,
                   w_dist="t", nu=5.0, seed=seed, index=2),
    ]


def cases_14b(r: int, M: int = 16384, seed: int = 0, kinds=("q", "gate", "down"), layer: int = 0) -> List[LinearCase]:
    """14B-shaped decoder linears (hidden 5120, intermediate 13824) with double
    quant, rank r, alpha = 2r, X of M tokens; weights are the stack's per-matrix
    scale * Student-t(nu) draws of the given layer."""
    mats = {m.name: m for m in stack_matrices_14b(n_layers=layer + 1) if m.layer == layer}
    out = []
    for k in kinds:
        m = mats[k]
        out.append(LinearCase(f"14b-{k}-r{r}", M=M, out=m.out, inp=m.inp, r=r, alpha=2.0 * r, double_quant=True,
                              w_dist="t", nu=m.nu, w_std=m.scale, seed=m.seed + seed, index=m.index))
    return out


LLAMA7B_LINEARS = (("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                   ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008))
QWEN14B_LINEARS = (("q", 5120, 5120), ("k", 5120, 5120), ("v", 5120, 5120), ("o", 5120, 5120),
                   ("gate", 13824, 5120), ("up", 13824, 5120), ("down", 5120, 13824))


@dataclasses.dataclass(frozen=True)
class StackMatrix:
    layer: int
    name: str
    out: int
    inp: int
    nu: float
    scale: float
    index: int
    seed: int = 0               # seed of the stack's draws and of its weights


# The 14B-shaped stack draws from its own seed (the Llama-7B-shaped stack uses 0).
STACK_14B_SEED = 1


def stack_matrices(n_layers: int = 32, linears=LLAMA7B_LINEARS, seed: int = 0) -> List[StackMatrix]:
    """Matrix list of a decoder stack in layer-major, then q,k,v,o,gate,up,down order."""
    draws = layer_draws(n_layers * len(linears), seed)
    mats = []
    for l in range(n_layers):
        for j, (nm, o, i) in enumerate(linears):
            idx = l * len(linears) + j
            nu, sc = draws[idx]
            mats.append(StackMatrix(l, nm, o, i, nu, sc, idx, seed))
    return mats


def stack_matrices_14b(n_layers: int = 40) -> List[StackMatrix]:
    """The 14B-shaped stack: hidden 5120, intermediate 13824, MHA, its own seed."""
    return stack_matrices(n_layers=n_layers, linears=QWEN14B_LINEARS, seed=STACK_14B_SEED)


def stack_weight(m: StackMatrix, seed: Optional[int] = None, device: str = "cpu") -> torch.Tensor:
    """``scale * t_nu`` weights of one stack matrix (seed defaults to the stack's)."""
    sd = m.seed if seed is None else seed
    return student_t_bf16((m.out, m.inp), m.nu, m.scale, sd, STREAM_W, m.index, device)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (CPU copy)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bf16_bits(a: np.ndarray, device: str = "cpu") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
