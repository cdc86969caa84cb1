"""Full decoder stacks of seeded weights generated on the host, one matrix per
spawned worker process.

Each worker runs torch single-threaded and draws its matrix exactly as
``synth.stack_weight`` does on the CPU (the draws do not depend on the thread
count), so the golden script and the GPU tests see the same bits. Workers are
spawned, never forked, so a caller that has already touched the GPU is safe.
Nothing here computes any part of the method; the optional oracle sums are the
oracle's own function, run in the worker next to the draw.
"""
from __future__ import annotations

import concurrent.futures as cf
import multiprocessing as mp
import os
from typing import Iterator, Optional, Sequence, Tuple

import numpy as np


def _init() -> None:
    import torch
    torch.set_num_threads(1)


def _bits(m) -> Tuple[int, np.ndarray]:
    from quantized_lora_fine_b200 import synth
    return m.index, synth.bf16_bits(synth.stack_weight(m))


def _oracle_sums(job) -> Tuple[int, float, float]:
    m, dq = job
    from oracle import layer_error
    from quantized_lora_fine_b200 import synth
    sd, sw = layer_error.layer_sums(synth.bf16_bits(synth.stack_weight(m)), dq)
    return m.index, sd, sw


def _pool(n: int, workers: Optional[int]) -> cf.ProcessPoolExecutor:
    w = workers or min(n, os.cpu_count() or 1)
    return cf.ProcessPoolExecutor(max_workers=max(1, w), mp_context=mp.get_context("spawn"), initializer=_init)


def stack_bits(mats: Sequence, workers: Optional[int] = None) -> Iterator[Tuple[int, np.ndarray]]:
    """(matrix index, uint16 bf16 bits [out, in]) for every matrix, in order."""
    with _pool(len(mats), workers) as ex:
        yield from ex.map(_bits, mats)


def oracle_stack_sums(mats: Sequence, double_quant: bool, workers: Optional[int] = None):
    """The oracle's (sum (w - w_hat)^2, sum w^2) of every matrix, in order."""
    with _pool(len(mats), workers) as ex:
        return list(ex.map(_oracle_sums, [(m, double_quant) for m in mats]))
