"""Benchmark of the NF4-LoRA hot path on B200.

Workload (one GPU): the Llama-7B q_proj shape -- W 4096 x 4096 stored NF4 with
double quantization (E4M3 absmax, groups of 256), X 8192 x 4096 bf16 (batch 4 x
seq 2048), rank 16, alpha 32, forward + backward (dX, dL1, dL2).

One timed step runs every step of the path once on that batch:
  nf4_quantize_error_rank([W], K=0)    the allocation pass with the quantization it
                                       measures: codes, double-quantized scales,
                                       per-layer NF4 error and ranking from one read
                                       of W (on a second stream, beside T)
  qlora_lora_down                      T = X L1
  qlora_linear_fwd_t                   Y = X W^T + s T L2 (fused dequant GEMM)
  qlora_linear_bwd                     U, dL2, dL1, dX = dY W + s U L1^T (fused dequant GEMM)
`value` counts only the algorithmic fwd+bwd flops (4 M h o + 6 M r (h + o))
over the whole step time; per-leg times are reported beside it.

With torchrun (N > 1 GPUs) every rank runs the same step on its own batch of
8192 tokens (weak scaling) and the adapter gradients dL1 / dL2 are summed
across ranks with an NCCL all-reduce, the one exchange a data-parallel step has.

`--impl reference` times the CPU oracle (the plain fp64 restatement of the
method used by the tests) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NF4-LoRA linear fwd+bwd TFLOP/s (frac of bf16 peak); NF4 quant/error GB/s"
UNIT = "TFLOP/s"
WORKLOAD = "llama7b-q_proj: W 4096x4096 NF4 blocksize 64 + double-quant (e4m3 absmax, group 256), X 8192x4096 bf16, r=16, alpha=32, fwd+bwd"


def flops_fwd_bwd(M, h, o, r):
    return 4.0 * M * h * o + 6.0 * M * r * (h + o)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def config_dict(args, world):
    return {"workload": WORKLOAD, "M_per_gpu": args.M, "in": 4096, "out": 4096, "r": 16, "alpha": 32,
            "global_tokens": args.M * world, "l2": "flushed between timed steps (256 MiB write)",
            "parallelism": f"dp{world}" if world > 1 else "single-gpu"}


# --------------------------------------------------------------------------- CPU oracle leg

def run_oracle_sample(rows: int, out_rows: int = 4096, seed: int = 0):
    """Times the oracle on a sub-problem of the q_proj workload: the first
    `out_rows` output rows of W (all 4096 inputs) quantized with double
    quantization, their NF4 error, and fwd+bwd on `rows` token rows.
    Returns (seconds, fwd+bwd flops of the sub-problem, description)."""
    import numpy as np
    from oracle import layer_error, lora, nf4
    from quantized_lora_fine_b200 import synth

    case = synth.case_q_proj(seed=seed, M=rows)
    d = case.make()
    W = d["W"][:out_rows].contiguous()
    L2 = d["L2"][:, :out_rows].contiguous()
    dYt = d["dY"][:, :out_rows].contiguous()
    Wb = synth.bf16_bits(W)
    X, L1, L2, dY = (nf4.f32_from_bf16_bits(synth.bf16_bits(t)).astype(np.float64) for t in (d["X"], d["L1"], L2, dYt))
    t0 = time.perf_counter()
    qw = nf4.quantize(nf4.f32_from_bf16_bits(Wb).reshape(W.shape), double_quant=True)
    What = nf4.f32_from_bf16_bits(nf4.dequantize_bf16_bits(qw)).astype(np.float64).reshape(W.shape)
    layer_error.layer_error(Wb, True)
    lora.forward(X, What, L1, L2, case.scale)
    lora.backward(X, What, L1, L2, dY, case.scale)
    dt = time.perf_counter() - t0
    return dt, flops_fwd_bwd(rows, 4096, out_rows, 16), (
        f"oracle (numpy fp64): {out_rows}x4096 slice of W quantized with DQ + its error pass + fwd+bwd on "
        f"{rows} of 8192 token rows; rate = fwd+bwd flops of that sub-problem / wall time")


def oracle_rate(min_seconds: float, rows: int, out_rows: int):
    run_oracle_sample(16, 64)  # NF4 table cache
    tot_t = tot_f = 0.0
    desc = ""
    while tot_t < min_seconds:
        dt, fl, desc = run_oracle_sample(rows, out_rows)
        tot_t += dt
        tot_f += fl
    return tot_f / tot_t / 1e12, tot_t, desc


def cpu_threads():
    try:
        import numpy as np  # noqa: F401
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info()]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def reference_main(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    rows, out_rows = 256, 512
    run_oracle_sample(16, 64)  # NF4 table cache
    for _ in range(args.warmup):
        run_oracle_sample(rows, out_rows)
    times, desc, fl = [], "", 0.0
    for _ in range(max(1, args.steps)):
        dt, fl, desc = run_oracle_sample(rows, out_rows)
        times.append(dt)
    dt = sum(times) / len(times)
    tf = fl / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": tf, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(args, 1),
            "cpu_baseline": {"value": tf, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle", "sample": desc},
            "e2e": {"value": tf, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- GPU leg

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"qlb_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for ln in open(self.path):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), reasons=parts[4:9]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        seen = set()
        for r in rows:
            for nm, v in zip(names, r["reasons"][1:]):
                if v.lower() in ("active", "0x1", "1", "yes"):
                    seen.add(nm)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(seen), "samples": len(rows)}


def cpus_near_gpu(torch, dev):
    """The host CPUs NVML lists as local to `dev` (its NUMA node), or None."""
    try:
        import pynvml
        props = torch.cuda.get_device_properties(dev)
        pynvml.nvmlInit()
        bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        words = (os.cpu_count() + 63) // 64
        mask = pynvml.nvmlDeviceGetCpuAffinity(h, words)
        cpus = {w * 64 + b for w, m in enumerate(mask) for b in range(64) if (int(m) >> b) & 1}
        cpus &= set(os.sched_getaffinity(0))
        return cpus or None
    except Exception:
        return None


def pair_gemm_traffic(name: str):
    """DRAM bytes per launch of a fused pair GEMM from the committed ncu capture in
    profiles/roofline_traffic.json, or None when the GEMM's sources changed since the
    capture (their hash no longer matches)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "roofline_traffic.json")
    try:
        d = json.load(open(path))
        h = hashlib.sha256()
        for f in d["sources"]:
            with open(os.path.join(ROOT, f), "rb") as fh:
                h.update(fh.read())
        if h.hexdigest() != d["sources_sha256"]:
            return None
        k = d["kernels"][name]
        return k["dram_bytes_read"] + k["dram_bytes_write"]
    except (OSError, KeyError, ValueError):
        return None


def mlp_leg(api, synth, torch, dev, peaks, reps: int = 5):
    """The Llama-7B MLP at M = 8192 (gate and up 4096 -> 11008, down 11008 -> 4096;
    NF4 blocks of 64 without double quant; r = 64, alpha = 128): fwd+bwd of the three
    linears (the one-call forward, T in the GEMM's T tiles), weights quantized once
    outside the timed region, captured in one CUDA graph and replayed (L2 flushed
    before each replay)."""
    items = []
    fl = 0.0
    for c in synth.cases_mlp():
        d = c.make(device=str(dev))
        w = api.quantize(d["W"], double_quant=False)
        items.append((c, w, d))
        fl += flops_fwd_bwd(c.M, c.inp, c.out, c.r)

    def run():
        for c, w, d in items:
            _, T = api.linear_fwd(w, d["X"], d["L1"], d["L2"], c.scale)   # one call: T in the GEMM's T tiles
            api.linear_bwd(w, d["X"], d["dY"], d["L1"], d["L2"], c.scale, T=T)

    run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = []
    for i in range(reps + 1):
        flush.zero_()
        e0.record()
        g.replay()
        e1.record()
        e1.synchronize()
        if i:
            ts.append(e0.elapsed_time(e1))
    assert api.status() == 0, "device status set in the MLP leg"
    ms = statistics.median(ts)
    tf = fl / (ms * 1e-3) / 1e12
    del g, items
    torch.cuda.empty_cache()
    return {"workload": "llama7b MLP: gate/up 4096->11008, down 11008->4096, M=8192, NF4 (no double quant), "
                        "r=64, alpha=128, fwd+bwd of the three linears",
            "ms": ms, "TFLOP/s": tf, "frac_of_burst": tf / peaks["bf16"],
            "timing": f"CUDA-graph replay, median of {reps}, L2 flushed before each"}


def hbm_legs(api, synth, torch, dev, stream, peaks, reps: int = 3, layers: int = 32):
    """Quantize-all and error/rank over the Llama-7B-shaped stack (32 layers, 224
    matrices by default; fewer layers for small profiler captures)."""
    mats = synth.stack_matrices(n_layers=layers)
    Ws = [synth.stack_weight(m, device=str(dev)) for m in mats]
    numel = sum(w.numel() for w in Ws)
    nb = numel // 64
    q_bytes = numel * 2 + numel // 2 + nb * 4              # bf16 in; codes, fp32 absmax out (no double quant)
    e_bytes = numel * 2
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    outs = []
    for w in Ws:   # outputs allocated once, outside the timed region
        outs.append((torch.empty(w.numel() // 2, dtype=torch.uint8, device=dev),
                     torch.empty(w.numel() // 64, dtype=torch.float32, device=dev)))
    fused_outs = [api.NF4Weight(w.shape[0], w.shape[1], False, codes=c, absmax=a) for w, (c, a) in zip(Ws, outs)]

    def q_each():
        for w, (c, a) in zip(Ws, outs):
            api.quantize(w, codes=c, absmax=a)

    def q_all():
        api.quantize_batch(Ws, double_quant=False, outs=fused_outs)

    def e_all():
        api.layer_error_rank(Ws, min(16, len(Ws)), double_quant=False)

    def f_all():
        api.quantize_error_rank(Ws, min(16, len(Ws)), double_quant=False, outs=fused_outs)

    # each leg is captured once into a CUDA graph (after an eager warm-up call) and
    # replayed, so host launch work for the 224 matrices is not in the timed region
    times = {}
    for name, fn in (("qe", q_each), ("q", q_all), ("e", e_all), ("f", f_all)):
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize()
        ts = []
        for i in range(reps + 1):
            e0.record(stream)
            g.replay()
            e1.record(stream)
            e1.synchronize()
            if i:
                ts.append(e0.elapsed_time(e1))
        times[name] = ts
        del g
    qe_ms, q_ms, e_ms, f_ms = times["qe"], times["q"], times["e"], times["f"]
    assert api.status() == 0, "device status set in the codec legs"
    qem, qm, em, fm = min(qe_ms), min(q_ms), min(e_ms), min(f_ms)
    del Ws, outs
    torch.cuda.empty_cache()
    return {"workload": f"llama7b stack: {len(mats)} matrices ({layers} x q,k,v,o 4096^2, gate/up 11008x4096, "
                        f"down 4096x11008), {numel / 1e9:.2f} G weights, per-matrix scale * Student-t(nu), "
                        "NF4 blocksize 64, no double quant",
            "quantize_all": {"ms": qm, "bytes": q_bytes, "GB/s": q_bytes / (qm * 1e-3) / 1e9,
                             "frac_hbm": q_bytes / (qm * 1e-3) / 1e9 / peaks["hbm"], "launches": 1,
                             "note": "nf4_quantize_batch over all matrices"},
            "quantize_each": {"ms": qem, "bytes": q_bytes, "GB/s": q_bytes / (qem * 1e-3) / 1e9,
                              "frac_hbm": q_bytes / (qem * 1e-3) / 1e9 / peaks["hbm"], "launches": len(mats),
                              "note": "one nf4_quantize call per matrix"},
            "error_rank_all": {"ms": em, "bytes": e_bytes, "GB/s": e_bytes / (em * 1e-3) / 1e9,
                               "frac_hbm": e_bytes / (em * 1e-3) / 1e9 / peaks["hbm"], "launches": 3},
            "quantize_error_rank_all": {"ms": fm, "bytes": q_bytes, "GB/s": q_bytes / (fm * 1e-3) / 1e9,
                                        "frac_hbm": q_bytes / (fm * 1e-3) / 1e9 / peaks["hbm"], "launches": 3,
                                        "note": "one pass over the weights: codes, absmax, error partials; then per-layer finish and rank"},
            "timing": f"CUDA-graph replay, best of {reps} (inputs {numel * 2 / 1e9:.2f} GB, above L2)"}


def protect_leg(api, synth, torch, dev, peaks, reps: int = 3, K: int = 8):
    """What keeping layers in bf16 does to the step time on this part (the speed
    effect the AQLoRA page attributes to protected layers). The fwd+bwd of one
    linear (T, forward, backward; M = 16384, r = 16) is timed for the three
    14B-stack shapes with the NF4 weight (double quant) and with the same weight
    kept in bf16; the 280-matrix stack (40 layers of q, k, v, o, gate, up, down) is
    ranked by the error pass, and the step over all its linears is composed from
    the per-shape times with no layer kept and with the top K kept."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    shapes = {}
    for c in synth.cases_14b(16, M=16384):
        d = c.make(device=str(dev))
        kind = c.name.split("-")[1]
        row = {"out": c.out, "in": c.inp}
        for mode in ("nf4", "bf16", "two_stage"):
            if mode == "two_stage":   # two NF4 stages, reconstructed to bf16 once per step
                w1 = api.quantize(d["W"], double_quant=True)
                w2 = api.quantize_residual(d["W"], w1, double_quant=True)
            w = api.quantize(d["W"], double_quant=True) if mode == "nf4" else api.NF4Weight.protected(d["W"])

            def run():
                ww = api.NF4Weight.protected(api.dequantize_two_stage(w1, w2)) if mode == "two_stage" else w
                _, T = api.linear_fwd(ww, d["X"], d["L1"], d["L2"], c.scale)
                api.linear_bwd(ww, d["X"], d["dY"], d["L1"], d["L2"], c.scale, T=T)

            run()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                run()
            ts = []
            for i in range(reps + 1):
                flush.zero_()
                e0.record()
                g.replay()
                e1.record()
                e1.synchronize()
                if i:
                    ts.append(e0.elapsed_time(e1))
            ms = statistics.median(ts)
            row[f"{mode}_ms"] = ms
            row[f"{mode}_TFLOP/s"] = flops_fwd_bwd(c.M, c.inp, c.out, c.r) / (ms * 1e-3) / 1e12
            del g, w
        shapes[kind] = row
        row["two_stage_vs_bf16"] = row["two_stage_ms"] / row["bf16_ms"] - 1.0
        del d
        torch.cuda.empty_cache()
    assert api.status() == 0, "device status set in the protection leg"
    # rank the whole stack (12.7 G weights) once with the error pass
    mats = synth.stack_matrices_14b()
    Ws = [synth.stack_weight(m, device=str(dev)) for m in mats]
    _, order, _ = api.layer_error_rank(Ws, K, double_quant=True)
    order = order.cpu().tolist()
    del Ws
    torch.cuda.empty_cache()
    kind_of = {"q": "q", "k": "q", "v": "q", "o": "q", "gate": "gate", "up": "gate", "down": "down"}
    all_nf4 = sum(shapes[kind_of[m.name]]["nf4_ms"] for m in mats)
    kept = [mats[l] for l in order[:K]]
    with_k = all_nf4 + sum(shapes[kind_of[m.name]]["bf16_ms"] - shapes[kind_of[m.name]]["nf4_ms"] for m in kept)
    with_k2 = all_nf4 + sum(shapes[kind_of[m.name]]["two_stage_ms"] - shapes[kind_of[m.name]]["nf4_ms"] for m in kept)
    return {"workload": "14B-stack linears (hidden 5120, intermediate 13824), M = 16384, r = 16, alpha = 32, "
                        "NF4 with double quant vs the same weight kept in bf16 vs two NF4 stages (reconstructed "
                        "to bf16 once per step); fwd+bwd = the one-call forward (T in the NF4 GEMM's T tiles; "
                        "a bf16 layer computes T as its own pass) and the backward",
            "per_shape": shapes,
            "stack": {"matrices": len(mats), "K": K,
                      "kept": [f"layer {m.layer} {m.name}" for m in kept],
                      "step_ms_no_layer_kept": all_nf4, "step_ms_top_K_kept": with_k,
                      "change": with_k / all_nf4 - 1.0,
                      "step_ms_top_K_two_stage": with_k2, "change_two_stage": with_k2 / all_nf4 - 1.0,
                      "note": "composed from the per-shape times (each linear timed alone, L2 flushed)"},
            "timing": f"CUDA-graph replay, median of {reps}, L2 flushed before each"}


def linear_set_leg(api, synth, torch, dev, peaks, ranks=(16, 32, 64, 128), K: int = 8, alpha_frac: float = 0.85,
                   M: int = 16384):
    """The 14B-shaped decoder's whole linear set, run for real: 40 layers x {q, k, v, o
    5120^2, gate/up 13824x5120, down 5120x13824} = 280 NF4 linears (double quant),
    X of M = 16384 tokens per linear, r in `ranks` with alpha = 2r. The allocation
    pass ranks all 280 matrices and the top K = 8 are kept in bf16. Three settings
    (AQLoRA summary page, section 3.3: adapters on every block, or only on the top
    blocks with the backward stopped below the cut; AQLoRA-s uses alpha = .85):
      qlora        every linear NF4, adapters everywhere, full backward (dX everywhere)
      protect      the top K in bf16, adapters everywhere, full backward
      protect_top  the top K in bf16, adapters on the top alpha_frac of the blocks: the
                   blocks below run the forward only, the lowest adapted block runs
                   its backward without dX (early stop)
    Inputs are shared per shape (one X and dY per input / output width); every
    linear has its own weight. Each setting runs once untimed, then once timed with
    CUDA events around the 280 linears (eager calls; every linear lasts milliseconds).
    The forward of a block without adapters still adds its rank-r term, as every
    call of the library does."""
    mats = synth.stack_matrices_14b()
    Ws = [synth.stack_weight(m, device=str(dev)) for m in mats]
    _, order, keep, nf4 = api.quantize_error_rank(Ws, K, double_quant=True)
    keep = keep.cpu().tolist()
    weights = [api.NF4Weight.protected(W) if keep[i] else None for i, W in enumerate(Ws)]
    del Ws
    torch.cuda.empty_cache()
    shapes = sorted({(m.inp, m.out) for m in mats})
    n_layers = 1 + max(m.layer for m in mats)
    cut = n_layers - int(round(alpha_frac * n_layers))   # blocks [cut, n_layers) carry adapters
    X = {h: synth.normal_bf16((M, h), 1.0, 0, synth.STREAM_X, h, device=str(dev)) for h in {h for h, _ in shapes}}
    dY = {o: synth.normal_bf16((M, o), 1.0, 0, synth.STREAM_DY, o, device=str(dev)) for o in {o for _, o in shapes}}
    Y = {o: torch.empty((M, o), dtype=torch.bfloat16, device=dev) for o in dY}
    out = {"workload": f"14B-shaped stack: {len(mats)} linears (hidden 5120, intermediate 13824), NF4 + double "
                       f"quant, M = {M} tokens per linear, alpha = 2r; top {K} of the error ranking kept in bf16; "
                       f"adapters on blocks {cut}..{n_layers - 1} in the protect_top setting",
           "kept": [f"layer {mats[l].layer} {mats[l].name}" for l in order[:K].tolist()],
           "timing": "CUDA events around the 280 linears (eager calls), after one untimed pass", "per_rank": {}}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for r in ranks:
        s = 2.0
        L1 = {h: synth.normal_bf16((h, r), 0.01, 0, synth.STREAM_L1, h, device=str(dev)) for h in X}
        L2 = {o: synth.normal_bf16((r, o), 0.01, 0, synth.STREAM_L2, o, device=str(dev)) for o in dY}
        fl_full = sum(flops_fwd_bwd(M, m.inp, m.out, r) for m in mats)

        def run(setting):
            for i, m in enumerate(mats):
                w = weights[i] if (setting != "qlora" and keep[i]) else nf4[i]
                _, T = api.linear_fwd(w, X[m.inp], L1[m.inp], L2[m.out], s, Y=Y[m.out])
                if setting == "protect_top" and m.layer < cut:
                    continue                        # no adapter below the cut: no backward
                early = setting == "protect_top" and m.layer == cut
                api.linear_bwd(w, X[m.inp], dY[m.out], L1[m.inp], L2[m.out], s, T=T, need_dX=not early)

        row = {}
        for setting in ("qlora", "protect", "protect_top"):
            run(setting)
            torch.cuda.synchronize()
            e0.record()
            run(setting)
            e1.record()
            e1.synchronize()
            row[f"{setting}_ms"] = e0.elapsed_time(e1)
        row["qlora_TFLOP/s"] = fl_full / (row["qlora_ms"] * 1e-3) / 1e12
        row["qlora_frac_of_burst"] = row["qlora_TFLOP/s"] / peaks["bf16"]
        row["protect_TFLOP/s"] = fl_full / (row["protect_ms"] * 1e-3) / 1e12
        row["protect_vs_qlora"] = row["protect_ms"] / row["qlora_ms"] - 1.0
        row["protect_top_vs_qlora"] = row["protect_top_ms"] / row["qlora_ms"] - 1.0
        out["per_rank"][str(r)] = row
    assert api.status() == 0, "device status set in the linear-set leg"
    del nf4, weights, X, dY, Y
    torch.cuda.empty_cache()
    return out


def merge_leg(api, synth, torch, dev, stream, peaks, reps: int = 3, layers: int = 4, r: int = 16):
    """LoRA merge (W_hat + s (L1 L2)^T, bf16 out) and merge + NF4 re-quantization over
    the first `layers` decoder layers of the Llama-7B-shaped stack (7 matrices per
    layer), weights NF4 with double quant, r = 16, alpha = 32."""
    mats = synth.stack_matrices(n_layers=layers)
    Ws = [synth.stack_weight(m, device=str(dev)) for m in mats]
    ws = api.quantize_batch(Ws, double_quant=True)
    numel = sum(w.numel() for w in Ws)
    del Ws
    torch.cuda.empty_cache()
    ads = [(synth.normal_bf16((m.inp, r), 0.01, 0, synth.STREAM_L1, m.index, str(dev)),
            synth.normal_bf16((r, m.out), 0.01, 0, synth.STREAM_L2, m.index, str(dev))) for m in mats]
    nb = numel // 64
    l_bytes = sum(2 * r * (m.inp + m.out) for m in mats)
    in_bytes = numel // 2 + nb + 4 * ((nb + 255) // 256) + l_bytes  # codes, e4m3 scales, group scales, adapters
    m_bytes = in_bytes + 2 * numel                                    # + bf16 merged weight out
    rq_bytes = in_bytes + numel // 2 + nb + 4 * ((nb + 255) // 256)   # + re-quantized codes and scales out
    flops = 2.0 * r * numel                                           # fp64 rank sums
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def merge():
        for w, (L1, L2) in zip(ws, ads):
            api.lora_merge(w, L1, L2, 2.0)

    def merge_rq():
        for w, (L1, L2) in zip(ws, ads):
            api.lora_merge_requantize(w, L1, L2, 2.0, double_quant=True)

    # warm-up and capture on one stream, so the re-quantize workspace (the bf16 merged
    # weight, keyed by stream) is allocated before the capture and not inside the graph
    cap = torch.cuda.Stream(device=dev)
    times = {}
    for name, fn in (("m", merge), ("rq", merge_rq)):
        with torch.cuda.stream(cap):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            fn()
        torch.cuda.synchronize()
        ts = []
        for i in range(reps + 1):
            e0.record(stream)
            g.replay()
            e1.record(stream)
            e1.synchronize()
            if i:
                ts.append(e0.elapsed_time(e1))
        times[name] = min(ts)
        del g
    assert api.status() == 0, "device status set in the merge legs"
    del ws, ads
    torch.cuda.empty_cache()
    mm, rm = times["m"], times["rq"]
    return {"workload": f"llama7b stack, first {layers} layers: {len(mats)} matrices, {numel / 1e9:.2f} G weights, "
                        f"NF4 with double quant, r={r}, s=2",
            "merge": {"ms": mm, "bytes": m_bytes, "GB/s": m_bytes / (mm * 1e-3) / 1e9,
                      "frac_hbm": m_bytes / (mm * 1e-3) / 1e9 / peaks["hbm"],
                      "fp64_TFLOP/s": flops / (mm * 1e-3) / 1e12, "launches": len(mats)},
            "merge_requantize": {"ms": rm, "bytes": rq_bytes, "GB/s": rq_bytes / (rm * 1e-3) / 1e9,
                                 "frac_hbm": rq_bytes / (rm * 1e-3) / 1e9 / peaks["hbm"],
                                 "fp64_TFLOP/s": flops / (rm * 1e-3) / 1e12, "launches": 2 * len(mats),
                                 "note": "NF4 in, NF4 out: each block is quantized where it is merged (exact "
                                         "fp32 scales to a scratch array), then one double-quant pass over the scales"},
            "timing": f"CUDA-graph replay, best of {reps} (outputs {2 * numel / 1e9:.2f} GB, above L2)"}


def summary_of(line):
    """Short form of the legs' headline rates (the end of the line)."""
    def g(*path):
        v = line
        for k in path:
            if not isinstance(v, dict) or k not in v:
                return None
            v = v[k]
        return round(v, 4) if isinstance(v, float) else v
    out = {"step_TFLOP/s": g("value"), "e2e_TFLOP/s": g("e2e", "value"),
           "fwd_bwd_TFLOP/s": g("legs", "fwd_bwd", "TFLOP/s"),
           "fwd_bwd_frac_of_burst": g("legs", "fwd_bwd", "frac_of_burst"),
           "fwd_gemm_TFLOP/s": g("legs", "fwd_gemm", "TFLOP/s"), "dx_gemm_TFLOP/s": g("legs", "dx_gemm", "TFLOP/s"),
           "mlp_TFLOP/s": g("mlp", "TFLOP/s"), "mlp_frac_of_burst": g("mlp", "frac_of_burst")}
    for leg in ("quantize_all", "quantize_each", "error_rank_all", "quantize_error_rank_all"):
        out[f"{leg}_GB/s"] = g("hbm_legs", leg, "GB/s")
        out[f"{leg}_frac_hbm"] = g("hbm_legs", leg, "frac_hbm")
    for r in ("16", "32", "64", "128"):
        out[f"linear_set_r{r}_TFLOP/s"] = g("linear_set", "per_rank", r, "qlora_TFLOP/s")
        out[f"linear_set_r{r}_protect_top_vs_qlora"] = g("linear_set", "per_rank", r, "protect_top_vs_qlora")
    out["merge_fp64_TFLOP/s"] = g("merge", "merge", "fp64_TFLOP/s")
    return {k: v for k, v in out.items() if v is not None}


def gpu_main(args):
    import ctypes

    import torch
    import torch.distributed as dist

    from quantized_lora_fine_b200 import _lib, api, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    lib = _lib.load()
    peaks = load_peaks()
    if args.gemm_only:   # the step's linear calls twice, as the step runs them (profiler captures; not a bench line)
        c = synth.case_q_proj()
        dd = {k: v.to(dev) for k, v in c.make().items()}
        w = api.quantize(dd["W"], double_quant=True)
        for _ in range(2):
            T = api.lora_down(dd["X"], dd["L1"])
            api.linear_fwd(w, dd["X"], dd["L1"], dd["L2"], c.scale, T=T)
            api.linear_bwd(w, dd["X"], dd["dY"], dd["L1"], dd["L2"], c.scale, T=T)
        api.linear_fwd(w, dd["X"], dd["L1"], dd["L2"], c.scale)   # then the one-call forward (T tiles)
        torch.cuda.synchronize()
        assert api.status() == 0, "device status set"
        print(json.dumps({"gemm_only": "ok", "pairs": int(lib.qlora_pair_clusters())}), flush=True)
        return
    if args.linear_set_only:   # the linear-set leg alone (not a bench line)
        print(json.dumps({"linear_set": linear_set_leg(api, synth, torch, dev, peaks)}), flush=True)
        return
    if args.protect_only:   # the protected-layer leg alone (not a bench line)
        print(json.dumps({"protect": protect_leg(api, synth, torch, dev, peaks)}), flush=True)
        return
    if args.merge_only:   # the merge legs alone (profiling aid; not a bench line)
        print(json.dumps({"merge": merge_leg(api, synth, torch, dev, torch.cuda.current_stream(), peaks,
                                             layers=args.merge_layers)}), flush=True)
        return
    if args.hbm_only:   # the codec legs alone (profiling aid; not a bench line)
        print(json.dumps({"hbm_legs": hbm_legs(api, synth, torch, dev, torch.cuda.current_stream(), peaks,
                                                layers=args.hbm_layers)}), flush=True)
        return

    M, h, o, r, alpha = args.M, 4096, 4096, 16, 32.0
    s = alpha / r
    case = synth.case_q_proj(seed=0, M=M)
    # weak scaling: each rank draws its own batch (matrix index offset) over the same weights
    d = case.make(device="cpu")
    if world > 1 and rank > 0:
        import dataclasses
        d2 = dataclasses.replace(case, index=rank).make(device="cpu")
        d["X"], d["dY"] = d2["X"], d2["dY"]
    g = {k: v.to(dev) for k, v in d.items()}
    stream = torch.cuda.current_stream()

    side = torch.cuda.Stream(device=dev)

    def alloc_and_down(W, X, L1):
        """T = X L1 on this stream and, launched after it on a second stream, the
        independent allocation pass (quantize W with double quant, error, rank: one
        read of W), whose small CTAs fill the SMs beside T's. (Launched in the other
        order the allocation pass took every SM first and the step ran 29 us longer.)"""
        main = torch.cuda.current_stream()
        side.wait_stream(main)
        T = api.lora_down(X, L1)
        with torch.cuda.stream(side):
            err, order, keep, (w,) = api.quantize_error_rank([W], 0, double_quant=True)
        main.wait_stream(side)
        for t in (w.codes, w.absmax_q, w.absmax2, err, order, keep):
            t.record_stream(main)
        return w, T

    def run_step(W, X, dY, L1, L2):
        w, T = alloc_and_down(W, X, L1)
        Y, T = api.linear_fwd(w, X, L1, L2, s, T=T)
        dX, dL1, dL2 = api.linear_bwd(w, X, dY, L1, L2, s, T=T)
        if world > 1:
            dist.all_reduce(dL1)
            dist.all_reduce(dL2)
        return Y, dX, dL1, dL2

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    prof = [torch.cuda.Event(enable_timing=True) for _ in range(4)]

    # Warm up eagerly (sizes the workspace, sets kernel attributes), then capture
    # one whole step -- and each leg on its own -- into CUDA graphs; timing
    # replays removes host launch gaps from the device time.
    for _ in range(max(3, args.warmup)):
        run_step(g["W"], g["X"], g["dY"], g["L1"], g["L2"])
    torch.cuda.synchronize()
    assert api.status() == 0, "device status set during warm-up"
    for e in prof:  # torch creates the CUDA event on first record
        e.record(stream)
    torch.cuda.synchronize()
    lib.qlora_profile_events(ctypes.c_void_p(prof[0].cuda_event), ctypes.c_void_p(prof[1].cuda_event),
                             ctypes.c_void_p(prof[2].cuda_event), ctypes.c_void_p(prof[3].cuda_event))
    state = {}

    def leg_quant():   # the allocation pass alone (on this stream)
        _, _, _, (state["w"],) = api.quantize_error_rank([g["W"]], 0, double_quant=True)

    def leg_down():    # T = X L1 alone
        state["T"] = api.lora_down(g["X"], g["L1"])

    def leg_fwd():
        state["Y"], state["T"] = api.linear_fwd(state["w"], g["X"], g["L1"], g["L2"], s, T=state["T"])

    def leg_fwd_fused_t():   # the one-call forward: T = X L1 in the GEMM's own tiles
        state["Y"], state["T"] = api.linear_fwd(state["w"], g["X"], g["L1"], g["L2"], s)

    def leg_bwd():
        state["dX"], state["dL1"], state["dL2"] = api.linear_bwd(state["w"], g["X"], g["dY"], g["L1"], g["L2"], s,
                                                                  T=state["T"])
        if world > 1:
            dist.all_reduce(state["dL1"])
            dist.all_reduce(state["dL2"])

    def whole_step():
        state["w"], state["T"] = alloc_and_down(g["W"], g["X"], g["L1"])
        leg_fwd(); leg_bwd()

    def fwd_bwd():     # the linear's fwd+bwd alone (weights already quantized)
        leg_down(); leg_fwd(); leg_bwd()

    use_graphs = not args.eager and world == 1
    graphs = {}
    if use_graphs:
        try:
            for name, fn in (("step", whole_step), ("quantize_error_rank", leg_quant), ("lora_down", leg_down),
                             ("fwd", leg_fwd), ("fwd_fused_t", leg_fwd_fused_t), ("bwd", leg_bwd),
                             ("fwd_bwd", fwd_bwd)):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr):
                    fn()
                graphs[name] = gr
            torch.cuda.synchronize()
        except Exception as exc:  # fall back to eager timing
            print(f"graph capture failed ({exc}); timing eagerly", file=sys.stderr)
            graphs, use_graphs = {}, False

    def run(name, fn):
        if use_graphs:
            graphs[name].replay()
        else:
            fn()

    step_ms, legs = [], {"quantize_error_rank": [], "lora_down": [], "fwd": [], "fwd_fused_t": [], "bwd": [],
                         "fwd_bwd": [], "fwd_gemm": [], "dx_gemm": [], "fwd_fused_t_gemm": []}
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    for i in range(args.steps):
        flush.zero_()
        ev[0].record(stream)
        run("step", whole_step)
        ev[1].record(stream)
        ev[1].synchronize()
        step_ms.append(ev[0].elapsed_time(ev[1]))
        legs["fwd_gemm"].append(prof[0].elapsed_time(prof[1]))
        legs["dx_gemm"].append(prof[2].elapsed_time(prof[3]))
    clk = clocks.stop()
    for name, fn in (("quantize_error_rank", leg_quant), ("lora_down", leg_down), ("fwd", leg_fwd),
                     ("fwd_fused_t", leg_fwd_fused_t), ("bwd", leg_bwd), ("fwd_bwd", fwd_bwd)):
        for i in range(max(5, min(args.steps, 50))):
            flush.zero_()
            ev[2].record(stream)
            run(name, fn)
            ev[3].record(stream)
            ev[3].synchronize()
            legs[name].append(ev[2].elapsed_time(ev[3]))
            if name == "fwd_fused_t":
                legs["fwd_fused_t_gemm"].append(prof[0].elapsed_time(prof[1]))
    lib.qlora_profile_events(None, None, None, None)
    torch.cuda.synchronize()
    assert api.status() == 0, "device status set during timing"
    graphs.clear()

    total_ms = sum(step_ms)
    if world > 1:
        t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms = total_ms / args.steps
    fl = flops_fwd_bwd(M, h, o, r)
    value = fl * world / (ms * 1e-3) / 1e12

    med = {k: statistics.median(v) for k, v in legs.items()}
    fl_fwd_gemm = 2.0 * M * h * o + 2.0 * M * r * o
    fl_dx_gemm = 2.0 * M * o * h + 2.0 * M * r * h
    fwd_tf = fl_fwd_gemm / (med["fwd_gemm"] * 1e-3) / 1e12
    dx_tf = fl_dx_gemm / (med["dx_gemm"] * 1e-3) / 1e12
    # dominant kernel = the longer of the two fused GEMMs
    engine = {"1cta": "tc_gemm_kernel", "pair256": "tc_gemm_nf4_pair_kernel"}.get(
        os.environ.get("QLORA_B200_GEMM", ""), "tc_gemm_nf4_pair2_kernel")
    dom = (f"qlora_fwd_gemm ({engine} fwd)", fwd_tf, med["fwd_gemm"]) if med["fwd_gemm"] >= med["dx_gemm"] \
        else (f"qlora_bwd_dx_gemm ({engine} dX)", dx_tf, med["dx_gemm"])
    numel = h * o
    qer_bytes = numel * 2 + numel // 2 + numel // 64 + 4 * (numel // 64 // 256)   # bf16 in; codes, E4M3, fp32 out
    # the burst GEMM rate is the denominator unless the clocks sampled during the timed region show the
    # power cap engaged, in which case the seconds-long (power-capped) rate is the comparable one
    capped = "sw_power_cap" in (clk or {}).get("reasons", [])
    peak_key, peak_kind = ("bf16_sus", "bf16 sustained") if capped else ("bf16", "bf16 burst")
    roofline = {"kernel": dom[0], "bound": "tensor", "achieved": dom[1], "peak": peaks[peak_key],
                "unit": "TFLOP/s", "frac": dom[1] / peaks[peak_key],
                "peak_kind": f"{peak_kind} ({peaks['source']}; power cap {'seen' if capped else 'not seen'})",
                "frac_of_burst": dom[1] / peaks["bf16"], "frac_of_sustained": dom[1] / peaks["bf16_sus"],
                "traffic": pair_gemm_traffic("qlora_fwd_gemm" if dom[0].startswith("qlora_fwd") else "qlora_bwd_dx_gemm"),
                "traffic_unit": "bytes per launch (ncu dram read + write)",
                "per_launch_flops": fl_fwd_gemm if dom[0].startswith("qlora_fwd") else fl_dx_gemm}
    legs_out = {
        "quantize_error_rank": {"ms": med["quantize_error_rank"],
                                "GB/s": qer_bytes / (med["quantize_error_rank"] * 1e-3) / 1e9,
                                "frac_hbm": qer_bytes / (med["quantize_error_rank"] * 1e-3) / 1e9 / peaks["hbm"]},
        "lora_down": {"ms": med["lora_down"], "note": "T = X L1; in the step the allocation pass runs beside it"},
        "fwd": {"ms": med["fwd"], "note": "with T given"},
        "fwd_fused_t": {"ms": med["fwd_fused_t"], "gemm_ms": med["fwd_fused_t_gemm"],
                        "note": "the one-call forward: T = X L1 in the GEMM's own tiles (the step instead runs "
                                "T beside the allocation pass, which measured faster)"},
        "bwd": {"ms": med["bwd"]},
        "fwd_bwd": {"ms": med["fwd_bwd"], "TFLOP/s": fl / (med["fwd_bwd"] * 1e-3) / 1e12,
                    "frac_of_burst": fl / (med["fwd_bwd"] * 1e-3) / 1e12 / peaks["bf16"],
                    "note": "T, forward and backward of the linear without the allocation pass"},
        "fwd_gemm": {"ms": med["fwd_gemm"], "TFLOP/s": fwd_tf}, "dx_gemm": {"ms": med["dx_gemm"], "TFLOP/s": dx_tf},
    }

    # ------------------------------------------------ end to end with host buffers
    # Every step copies its inputs (W, X, dY, L1, L2) from pinned host memory and its
    # result, the adapter gradients dL1 and dL2, back to pinned host memory (Y and dX
    # are what the neighbouring layers consume on the device; a second run also
    # copies them back and is reported beside). The steps are pipelined on three
    # streams: the host-to-device copies of step k + 1 (into the second of two device
    # input sets) and the device-to-host copies of step k - 1 run while step k
    # computes; the timed region spans all steps, from the first input copy to the
    # last result copy.
    e2e = None
    if args.e2e_steps > 0:
        # the pinned buffers are placed while this thread runs on the GPU's own NUMA
        # node, so the copy engines read local memory
        near, before = cpus_near_gpu(torch, dev), os.sched_getaffinity(0)
        if near:
            os.sched_setaffinity(0, near)
        pin = {k: v.cpu().pin_memory() for k, v in d.items()}
        outs = [{"Y": torch.empty((M, o), dtype=torch.bfloat16).pin_memory(),
                 "dX": torch.empty((M, h), dtype=torch.bfloat16).pin_memory(),
                 "dL1": torch.empty((h, r), dtype=torch.float32).pin_memory(),
                 "dL2": torch.empty((r, o), dtype=torch.float32).pin_memory()} for _ in range(2)]
        if near:
            os.sched_setaffinity(0, before)
        h2d = sum(t.numel() * t.element_size() for t in pin.values())
        result_names = ("dL1", "dL2")
        d2h = sum(outs[0][k].numel() * outs[0][k].element_size() for k in result_names)
        d2h_all = sum(t.numel() * t.element_size() for t in outs[0].values())
        dev_in = [{k: torch.empty_like(v, device=dev) for k, v in pin.items()} for _ in range(2)]
        s_in = torch.cuda.Stream(device=dev)
        s_out = torch.cuda.Stream(device=dev)

        def pipeline(n_steps, names):
            ready = [torch.cuda.Event() for _ in range(n_steps)]
            done = [torch.cuda.Event() for _ in range(n_steps)]
            copied = [torch.cuda.Event() for _ in range(n_steps)]

            def load(k):
                with torch.cuda.stream(s_in):
                    if k >= 2:
                        s_in.wait_event(done[k - 2])   # step k - 2 has finished reading this input set
                    for key in pin:
                        dev_in[k % 2][key].copy_(pin[key], non_blocking=True)
                    ready[k].record(s_in)

            load(0)
            for k in range(n_steps):
                if k + 1 < n_steps:
                    load(k + 1)
                stream.wait_event(ready[k])
                b = dev_in[k % 2]
                res = run_step(b["W"], b["X"], b["dY"], b["L1"], b["L2"])
                done[k].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(done[k])
                    for name, t in zip(("Y", "dX", "dL1", "dL2"), res):
                        if name not in names:
                            continue
                        t.record_stream(s_out)
                        outs[k % 2][name].copy_(t, non_blocking=True)
                    copied[k].record(s_out)
            stream.wait_event(copied[n_steps - 1])

        def timed(names):
            pipeline(3, names)   # warm-up
            torch.cuda.synchronize()
            flush.zero_()
            s_in.wait_stream(stream)
            ev[0].record(stream)
            s_in.wait_event(ev[0])
            pipeline(args.e2e_steps, names)
            ev[1].record(stream)
            ev[1].synchronize()
            em = ev[0].elapsed_time(ev[1]) / args.e2e_steps
            assert api.status() == 0, "device status set in the end-to-end run"
            if world > 1:
                t = torch.tensor([em], dtype=torch.float64, device=dev)
                dist.all_reduce(t, op=dist.ReduceOp.MAX)
                em = float(t.item())
            return em

        em = timed(result_names)
        em_all = timed(("Y", "dX", "dL1", "dL2"))
        e2e = {"value": fl * world / (em * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": em,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "result": "dL1, dL2 (the adapter gradients)",
               "host_buffers": "pinned on the GPU's NUMA node" if near else "pinned (NUMA node not known)",
               "with_Y_dX_back": {"ms_per_step": em_all, "TFLOP/s": fl * world / (em_all * 1e-3) / 1e12,
                                  "d2h_bytes_per_step": d2h_all},
               "timing": f"{args.e2e_steps} steps pipelined over three streams (input copies of the next step and "
                         "result copies of the previous one beside each step), one event pair around all of them"}

    # ------------------------------------------------ codec kernels at full model scale
    # The q_proj weight (33.5 MB) fits in L2 and its kernels last tens of
    # microseconds; the HBM roofline of the quantizer and the error pass is taken
    # on the Llama-7B-shaped stack instead: 224 matrices, 6.48 G weights (12.95 GB
    # of bf16), quantize every matrix (one call each) and one error/rank call over
    # all of them, as the allocation pass does.
    # The side legs run after the step's own numbers are taken; one that fails is
    # reported in its own entry and does not cost the line.
    def side_leg(fn, *a, **k):
        try:
            return fn(*a, **k)
        except Exception as e:   # noqa: BLE001 -- reported, not hidden
            return {"error": f"{type(e).__name__}: {e}"}

    hbm = None
    if rank == 0 and world == 1 and not args.no_hbm_legs:
        hbm = side_leg(hbm_legs, api, synth, torch, dev, stream, peaks, layers=args.hbm_layers)
    mlp = None
    if rank == 0 and world == 1 and not args.no_mlp_leg:
        mlp = side_leg(mlp_leg, api, synth, torch, dev, peaks)
    protect = None
    if rank == 0 and world == 1 and not args.no_protect_leg:
        protect = side_leg(protect_leg, api, synth, torch, dev, peaks)
    merge = None
    if rank == 0 and world == 1 and not args.no_merge_leg:
        merge = side_leg(merge_leg, api, synth, torch, dev, stream, peaks, layers=args.merge_layers)
    linear_set = None
    if rank == 0 and world == 1 and not args.no_linear_set_leg:
        linear_set = side_leg(linear_set_leg, api, synth, torch, dev, peaks)

    # ------------------------------------------------ CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, secs, desc = oracle_rate(args.cpu_seconds, args.cpu_rows, 4096)
        cpu = {"value": rate, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": desc + f"; repeated for {secs:.1f} s", "seconds": secs}

    launches_per_step = 2 + 1 + 3 + 5  # quantize+error, finish+rank; T; fwd (scales, s.L2^T, GEMM); bwd (U + s.U, dL2, dL1, scales, dX GEMM)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_dict(args, world),
            "roofline": roofline, "gemm_pairs": int(lib.qlora_pair_clusters()), "legs": legs_out, "mlp": mlp,
            "hbm_legs": hbm, "merge": merge, "protect": protect, "linear_set": linear_set, "cpu_baseline": cpu,
            "e2e": e2e, "gpu_launches": launches_per_step * args.steps, "clocks": clk,
            "timing": "cuda-graph replay of the step" if use_graphs else "eager API calls",
            "peaks": {"bf16_tflops": peaks["bf16"], "bf16_tflops_sustained": peaks["bf16_sus"],
                      "hbm_gbs": peaks["hbm"], "source": peaks["source"]}}
    # the headline figures of every leg again, last, in a short form
    line["summary"] = summary_of(line)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--M", type=int, default=8192)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-rows", type=int, default=512)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-hbm-legs", action="store_true", help="skip the full-stack quantizer / error-pass legs")
    ap.add_argument("--no-mlp-leg", action="store_true", help="skip the Llama-7B MLP (gate, up, down) fwd+bwd leg")
    ap.add_argument("--no-merge-leg", action="store_true", help="skip the LoRA merge / merge + re-quantize leg")
    ap.add_argument("--no-protect-leg", action="store_true",
                    help="skip the protected-layer (bf16 vs NF4) step-time leg on the 14B-stack shapes")
    ap.add_argument("--gemm-only", action="store_true",
                    help="two forward + backward calls of the q_proj linear, nothing timed (profiler captures)")
    ap.add_argument("--no-linear-set-leg", action="store_true",
                    help="skip the 280-linear 14B-shaped linear set (all NF4 / top 8 in bf16 / top-block adapters)")
    ap.add_argument("--linear-set-only", action="store_true",
                    help="run only the linear-set leg and print it (not a bench line)")
    ap.add_argument("--protect-only", action="store_true",
                    help="run only the protected-layer leg and print it (not a bench line)")
    ap.add_argument("--merge-layers", type=int, default=4, help="decoder layers of the stack for the merge leg")
    ap.add_argument("--merge-only", action="store_true",
                    help="run only the merge legs and print them (profiling aid; not a bench line)")
    ap.add_argument("--hbm-layers", type=int, default=32, help="decoder layers of the stack for those legs")
    ap.add_argument("--hbm-only", action="store_true",
                    help="run only the full-stack codec legs and print them (for profiler captures)")
    ap.add_argument("--eager", action="store_true", help="time eager API calls instead of CUDA-graph replays")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return reference_main(args)
    return gpu_main(args)


if __name__ == "__main__":
    sys.exit(main())
