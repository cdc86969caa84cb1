"""Writes the oracle's per-layer NF4 errors, ranking and keep mask for the two full
synthetic decoder stacks:

  stack_rank_llama7b.json  32 layers x {q, k, v, o 4096^2, gate/up 11008x4096,
                           down 4096x11008} = 224 matrices, NF4 blocks of 64 with
                           fp32 absmax, K = 16
  stack_rank_14b.json      40 layers x {q, k, v, o 5120^2, gate/up 13824x5120,
                           down 5120x13824} = 280 matrices, NF4 with double
                           quantization, K = 8

What is computed ("AQLoRA: A Zero-Search Recipe for Fast Quantized LoRA
Fine-Tuning", section 3.1: one data-free pass scores every linear layer by its
NF4 reconstruction error; section 3.2: layers are ranked by that error and the
top K are kept in 16-bit): per matrix the relative Frobenius error
e = sqrt(sum (w - w_hat)^2 / sum w^2) with w_hat the bf16 dequantized weight, the
order by (error descending, index ascending) and keep = the first K.

Inputs: the seeded stack generators (per matrix nu ~ U(3, 30), scale ~
U(0.005, 0.05), W = scale * t_nu rounded to bf16), drawn on the host. Only the
oracle computes; this script imports nothing from the CUDA path.

    python tests/golden/make_stack_rank_goldens.py [--workers N] [--only llama7b|14b]

About 3 minutes (Llama-7B-shaped stack) and 6 minutes (14B-shaped) on 8 cores,
at most about 4.5 GB of memory per worker.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from oracle import layer_error  # noqa: E402
from quantized_lora_fine_b200 import synth  # noqa: E402
from tests import stack_pool  # noqa: E402

STACKS = {
    "llama7b": dict(file="stack_rank_llama7b.json", mats=lambda: synth.stack_matrices(), dq=False, K=16,
                    workload="32-layer Llama-2-7B-shaped stack (q,k,v,o 4096x4096; gate,up 11008x4096; "
                             "down 4096x11008), 224 matrices, NF4 blocksize 64, fp32 absmax, keep top 16"),
    "14b": dict(file="stack_rank_14b.json", mats=lambda: synth.stack_matrices_14b(), dq=True, K=8,
                workload="40-layer 14B-shaped stack (hidden 5120, intermediate 13824, MHA), 280 matrices, "
                         "NF4 blocksize 64 + double quantization (E4M3 scales, group 256), keep top 8"),
}

CITATION = ("AQLoRA: A Zero-Search Recipe for Fast Quantized LoRA Fine-Tuning, section 3.1 (per-layer NF4 "
            "reconstruction error over 64-element blocks, one data-free pass) and section 3.2 (rank by error, "
            "keep the top K in 16-bit); QLoRA: How to fine-tune large language models with less memory, "
            "'1. NormalFloat' and '2. Double quantization' (the NF4 format the error is measured in)")


def make(name: str, workers: int) -> str:
    spec = STACKS[name]
    mats = spec["mats"]()
    t0 = time.time()
    sums = stack_pool.oracle_stack_sums(mats, spec["dq"], workers)
    err = [math.sqrt(sd / sw) if sw > 0 else 0.0 for _, sd, sw in sums]
    order = [int(i) for i in layer_error.rank_layers(err)]
    keep = [int(k) for k in layer_error.keep_mask(order, spec["K"])]
    out = {
        "citation": CITATION,
        "workload": spec["workload"],
        "generator": "quantized_lora_fine_b200.synth stack generators drawn on the host (stack seed "
                     f"{mats[0].seed}); error, order and keep from oracle.layer_error",
        "double_quant": spec["dq"],
        "K": spec["K"],
        "matrices": [{"layer": m.layer, "name": m.name, "out": m.out, "in": m.inp} for m in mats],
        "err": err,
        "sum_d2": [sd for _, sd, _ in sums],
        "sum_w2": [sw for _, _, sw in sums],
        "order": order,
        "keep": keep,
        "seconds": round(time.time() - t0, 1),
    }
    path = os.path.join(HERE, spec["file"])
    with open(path, "w") as f:
        json.dump(out, f, indent=0)
    return path


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--workers", type=int, default=None)
    ap.add_argument("--only", choices=sorted(STACKS), default=None)
    a = ap.parse_args()
    for nm in ([a.only] if a.only else sorted(STACKS)):
        print(make(nm, a.workers), flush=True)
