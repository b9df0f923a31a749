"""Benchmark of the routed-MoE FFN layer (Hy3 shapes) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--config decode|prefill|skewed|fp8|fp4_decode]
                    [--impl ours|reference] [--path auto|stream|gemm]

One step = one pass of the whole layer (route, group, gate_up, down, combine)
over one batch of T synthetic tokens, inputs resident in HBM. Rank 0 prints one
JSON line. With N > 1 (torchrun) every rank runs an independent replica on its
own batch (tokens are independent: no collective on the data path) and the
value is the tokens of all ranks over the slowest rank's time.

The step is timed through the public entry points one stage at a time
(moe_route3, moe_permute_index or moe_permute, moe_expert_gate_up_gather or
moe_expert_gate_up, moe_expert_down, moe_combine -- the same sequence
moe_forward3 runs), with CUDA events on the launching stream; ``e2e`` times
moe_forward3 with the input copied in from and the output copied back to
pinned host memory every step. bf16 expert weights for the tensor-core kernels are
packed once at load (moe_pack_weights), outside every timed region.

The metric has two halves, % of the HBM roofline at decode and % of the dense
bf16 tensor peak at prefill: the default line (``--config decode``) carries the
prefill workload, measured in the same run the same way, as its ``prefill``
object (``--no-prefill`` leaves it out). Tensor fractions divide by the burst
bf16 peak (steps last milliseconds); the sustained peak is given beside it.

``--impl reference`` times the fp64 CPU oracle on the host cores instead (each
step a bounded sample of the same workload), rank 0 only.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synthetic import CONFIGS, make_layer  # noqa: E402
from sparse_moe_transformer_gemm_b200 import work  # noqa: E402

WORKLOADS = {
    "decode": "Hy3 MoE layer decode: T=64 tokens, d=4096, E=192, top-8, d_ff=1536 SwiGLU, "
              "scale 2.826, fp32 combine; x bf16 N(0,1), W_gate/experts bf16 N(0,0.02)",
    "prefill": "Hy3 MoE layer prefill: T=4096 tokens, same shapes/dtypes/init as decode",
    "skewed": "Hy3 MoE layer, skewed routing: T=16384, logit bias 0.5*ln(Zipf(1.1) rank weight)",
    "fp8": "Hy3 MoE layer FP8 weights: T=8192, experts e4m3 + fp32 per-output-row scales",
    "tiny": "Tiny MoE layer: T=64, d=256, E=16, top-4, d_ff=128",
    "fp4_decode": "Second routing/precision variant at the Hy3 decode shape: T=64, d=4096, "
                  "E=192, top-6 sqrt-softplus scores (scale 1.5), d_ff=1536, experts E2M1 + "
                  "E8M0 block-32 scales",
}

# ncu dram__bytes_read.sum + dram__bytes_write.sum of the dominant kernel, from
# one capture of a smaller case of the same workload, as bytes per unit of work
# so that it scales to the benchmarked launch (traffic grows with the touched
# experts at decode, with the routed rows at prefill). An entry is removed when
# its kernel changes.
NCU_TRAFFIC = {
    # bf16 pair gate_up, decode case E=96, T=32: 2.2438 GB for 89 touched experts
    ("decode", "gate_up_gemm"): {"per": "touched_expert", "bytes": 2.2438e9 / 89},
    # bf16 pair gate_up, prefill case E=96, T=2048: 2.5879 GB for 16384 routed rows
    ("prefill", "gate_up_gemm"): {"per": "row", "bytes": 2.5879e9 / 16384},
    # FP8 pair gate_up, case E=48, T=2048 (341 rows per expert, as at T=8192):
    # 0.9362 GB for 16384 routed rows
    ("fp8", "gate_up_gemm"): {"per": "row", "bytes": 0.9362e9 / 16384},
    # FP4 pair gate_up, decode case E=96, T=32: 0.5638 GB for 83 touched experts
    ("fp4_decode", "gate_up_gemm"): {"per": "touched_expert", "bytes": 0.5638e9 / 83},
}


def ncu_traffic(config, kernel, touched, rows, full_shape):
    t = NCU_TRAFFIC.get((config, kernel)) if full_shape else None
    if t is None:
        return None
    return t["bytes"] * (touched if t["per"] == "touched_expert" else rows)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def slowest_rank_ms(ms: float, dist=None, device=None) -> float:
    """Max over ranks of a per-rank device time (identity without a process group)."""
    if dist is None:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(tokens_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput of independent replicas: all ranks' tokens over the slowest rank's time."""
    return world * tokens_per_rank / (ms / 1e3)


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def run_reference(args, world, rank):
    """The fp64 CPU oracle, as it stands, on the host cores (rank 0 only)."""
    if rank != 0:
        return
    import numpy as np
    import oracle

    shape = CONFIGS[args.config]
    layer = make_layer(shape, seed=0, device="cuda" if torch.cuda.is_available() else "cpu")
    O = oracle.OracleLayer(layer)
    del layer
    # size each step's token sample so that one step is ~args.ref_step_seconds of CPU work
    t0 = time.perf_counter()
    oracle.forward_tokens(O, np.array([0], np.int32))
    one = max(time.perf_counter() - t0, 1e-6)
    per_step = int(max(1, min(shape.T, round(args.ref_step_seconds * oracle.num_threads() / one))))
    rng = np.random.default_rng(0)
    samples = [rng.choice(shape.T, size=per_step, replace=False).astype(np.int32)
               for _ in range(args.warmup + args.steps)]
    for i in range(args.warmup):
        oracle.forward_tokens(O, samples[i])
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle.forward_tokens(O, samples[args.warmup + i])
    dt = time.perf_counter() - t0
    tok_s = per_step * args.steps / dt
    line = {
        "impl": "reference", "metric": "MoE-layer tokens/s", "value": tok_s, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, seed 0)",
        "config": {"workload": WORKLOADS[args.config], "T": shape.T},
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{per_step} random tokens of the {shape.T}-token batch per step"},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(layer, shape, seconds: float):
    """The oracle timed on the host cores on a bounded sample of the workload."""
    import numpy as np
    import oracle

    O = oracle.OracleLayer(layer)
    t0 = time.perf_counter()
    oracle.forward_tokens(O, np.array([0], np.int32))
    one = max(time.perf_counter() - t0, 1e-6)
    n = int(max(1, min(shape.T, round(seconds * oracle.num_threads() / one))))
    toks = np.arange(n, dtype=np.int32)
    t0 = time.perf_counter()
    oracle.forward_tokens(O, toks)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {n} of the {shape.T} tokens of the same batch ({dt:.1f} s)"}


def measure(args, name, dev, local, rank, world, pg, moe, block=False, cpu_seconds=None):
    """Time one workload: the staged step (device time, CUDA events on the
    launching stream) and the end-to-end moe_forward3 with host copies. Returns
    the fields of one bench line (without the cpu baseline unless asked)."""
    import dataclasses

    shape = CONFIGS[name]
    if args.experts or args.tokens:
        shape = dataclasses.replace(shape, E=args.experts or shape.E, T=args.tokens or shape.T)
    if block:
        shape = dataclasses.replace(shape, shared=True, score_bias_std=0.05)
    layer = make_layer(shape, seed=rank, device=dev)
    T, d, E, k, F = shape.T, shape.d, shape.E, shape.k, shape.F
    # bf16 weights on the tensor-core pair kernels are packed once, at load time
    # (moe_pack_weights), outside every timed region
    packed = (not shape.fp8 and not shape.fp4 and args.path != "stream" and d % 256 == 0 and
              F % 256 == 0)
    cfg = moe.config_of(shape, None if args.path == "auto" else args.path, packed=packed)
    # grouped slots per token (the shared expert, when present, is slot k of
    # every token and expert E)
    ks = k + (1 if shape.shared else 0)
    Eg = E + (1 if shape.shared else 0)
    R = T * ks
    ws = moe.workspace(cfg, device=dev)
    stream = torch.cuda.Stream(device=dev)
    wgu, sgu, wd, sd = moe.layer_args(layer)
    if packed:
        wgu, wd = moe.pack_layer_weights(cfg, wgu, wd)
        torch.cuda.synchronize(dev)
    x, wg, gb, sb = layer["x"], layer["w_gate"], layer["gate_bias"], layer["score_bias"]
    # router options: the score bias (complete Hy3 block) and the score function
    ropt = moe.route_options(sb, None, 1e-6, shape.score_fn)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    counts = torch.empty(Eg, dtype=torch.int32, device=dev)
    offsets = torch.empty(Eg + 1, dtype=torch.int32, device=dev)
    row_of = torch.empty(R, dtype=torch.int32, device=dev)
    gather = R <= moe.MOE_GATHER_MAX_SLOTS  # moe_forward's grouping rule
    tok = torch.empty(R, dtype=torch.int32, device=dev)
    xp = None if gather else torch.empty((R, d), dtype=torch.bfloat16, device=dev)
    h = torch.empty((R, F), dtype=torch.bfloat16, device=dev)
    y = torch.empty((R, d), dtype=torch.bfloat16, device=dev)
    out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)

    stages = ["route", "permute", "gate_up", "down", "combine"]
    # small batches: one grouping launch, and gate_up gathers its token rows inside
    # the GEMM on the bf16 SM-pair path (a row-gather kernel first on the others);
    # large batches: rank/scan/scatter with the permuted copy, then gate_up
    fused_gather = (not shape.fp8 and not shape.fp4 and args.path != "stream" and
                    d % 256 == 0 and F % 256 == 0)
    n_launch = {"route": 1, "permute": 1 if gather else 3,
                "gate_up": 2 if gather and not fused_gather else 1, "down": 1, "combine": 1}

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        moe.moe_route3(cfg, x, wg, gb, ropt, idx, w, ws, stream)
        if ev is not None:
            ev[1].record(stream)
        if gather:
            moe.moe_permute_index(cfg, idx, counts, offsets, row_of, tok, ws, stream)
        else:
            moe.moe_permute(cfg, idx, x, counts, offsets, row_of, xp, ws, stream)
        if ev is not None:
            ev[2].record(stream)
        if gather:
            moe.moe_expert_gate_up_gather(cfg, x, tok, offsets, wgu, sgu, h, ws, stream)
        else:
            moe.moe_expert_gate_up(cfg, xp, offsets, wgu, sgu, h, ws, stream)
        if ev is not None:
            ev[3].record(stream)
        moe.moe_expert_down(cfg, h, offsets, wd, sd, y, ws, stream)
        if ev is not None:
            ev[4].record(stream)
        moe.moe_combine(cfg, y, row_of, w, out, ws, stream)
        if ev is not None:
            ev[5].record(stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    assert moe.moe_read_status(ws, stream) == moe.MOE_OK

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        # the timed steps run as a user runs them: the layer's launches back to
        # back (an event between two kernels would stop the next one from
        # launching while the previous one finishes)
        t_begin.record(stream)
        for i in range(args.steps):
            step()
        t_end.record(stream)
        stream.synchronize()
        # the stage breakdown: the same steps again, an event between stages
        for i in range(args.steps):
            step(evs[i])
        stream.synchronize()
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    status = moe.moe_read_status(ws, stream)
    ms = t_begin.elapsed_time(t_end) / args.steps
    stage_ms = {s: sum(e[j].elapsed_time(e[j + 1]) for e in evs) / args.steps
                for j, s in enumerate(stages)}
    ms = slowest_rank_ms(ms, pg, dev)

    # touched experts of this batch (for the algorithmic bytes)
    touched = int((counts > 0).sum().item())
    rows = int(offsets[-1].item())
    peaks, peak_src = load_peaks()
    fp8, fp4 = shape.fp8, shape.fp4
    # the shared expert counts as one more touched expert with T more rows
    lw = work.layer_work(T, d, E, ks, F, touched, fp8, fp4)
    gw = work.gate_up_work(T, rows, touched, d, F, fp8, fp4)
    dw = work.down_work(rows, touched, d, F, fp8, fp4)
    dominant = max(("gate_up", "down"), key=lambda s: stage_ms[s])
    dom_work = gw if dominant == "gate_up" else dw
    dom_s = stage_ms[dominant] / 1e3
    # quantised weights on shapes the SM-pair kernels do not take, and FP4 at up
    # to one mean row per expert, run on the streaming kernels (the library's
    # automatic choice, include/moe.h)
    use_stream = (args.path == "stream" or ((fp8 or fp4) and (d % 256 or F % 256)) or
                  (fp4 and args.path == "auto" and T * k <= E))
    kernel_name = f"{dominant}_{'stream' if use_stream else 'gemm'}"
    # The metric's roofline: HBM for the decode workloads (weights streamed once),
    # dense bf16 tensor peak for the larger batches. A step lasts milliseconds,
    # so the tensor peak is the burst figure; the sustained one (a seconds-long
    # loop under the power cap) is given beside it.
    if name in ("decode", "tiny", "fp4_decode"):
        achieved = dom_work["bytes"] / dom_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
    else:
        achieved = dom_work["flops"] / dom_s / 1e12
        pk = peaks["bf16_tflops"]
        sus = peaks.get("bf16_tflops_sustained")
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk, "unit": "TFLOP/s",
                "frac": achieved / pk,
                "frac_of_sustained_peak": achieved / sus if sus else None}
    roof["traffic"] = ncu_traffic(name, kernel_name, touched, rows, shape == CONFIGS[name])
    roof["traffic_source"] = "ncu capture of a smaller case of the same kernel, scaled" \
        if roof["traffic"] is not None else None
    roof["kernel"] = kernel_name
    roof["peak_source"] = (f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'}"
                           f"{', burst' if roof['bound'] == 'tensor' else ''})")
    roof["algorithmic_bytes_per_launch"] = dom_work["bytes"]
    roof["algorithmic_flops_per_launch"] = dom_work["flops"]
    roof["implementation_bytes_per_launch"] = dom_work["implementation_bytes"]

    # End to end through moe_forward: every step copies its input from pinned host
    # memory and its output back to pinned host memory. The copies run on two
    # more streams (one per direction, so both copy engines work at once),
    # double-buffered, so that step i+1's input and step i-1's output cross PCIe
    # while step i computes (a serving loop's pipelining); the timed region spans
    # all copies and launches of the e2e_steps steps.
    x_host = x.cpu().pin_memory()
    out_host = [torch.empty((T, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    out_dev = [torch.empty((T, d), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    h2d_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)
    e2e_steps = max(3, args.steps // 2)

    def e2e_run(n):
        fwd = [None, None]
        d2h = [None, None]
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(h2d_stream):
                if fwd[b] is not None:
                    h2d_stream.wait_event(fwd[b])  # step i-2 has consumed x_dev[b]
                x_dev[b].copy_(x_host, non_blocking=True)
                h2d = torch.cuda.Event()
                h2d.record(h2d_stream)
            stream.wait_event(h2d)
            if d2h[b] is not None:
                stream.wait_event(d2h[b])  # step i-2's output has been read back
            moe.moe_forward3(cfg, x_dev[b], wg, gb, ropt, wgu, sgu, wd, sd, out_dev[b], ws,
                             stream)
            fwd[b] = torch.cuda.Event()
            fwd[b].record(stream)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(fwd[b])
                out_host[b].copy_(out_dev[b], non_blocking=True)
                d2h[b] = torch.cuda.Event()
                d2h[b].record(d2h_stream)
        for st in (h2d_stream, d2h_stream):
            done = torch.cuda.Event()
            done.record(st)
            stream.wait_event(done)

    e2e_run(args.warmup)
    stream.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    h2d_stream.wait_event(e0)
    d2h_stream.wait_event(e0)
    e2e_run(e2e_steps)
    e1.record(stream)
    stream.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = slowest_rank_ms(e2e_ms, pg, dev)
    status2 = moe.moe_read_status(ws, stream)
    e2e_same = bool(torch.equal(out_host[(e2e_steps - 1) % 2], out.cpu()))

    cpu = None
    if cpu_seconds is not None and rank == 0 and world == 1:
        cpu = cpu_baseline(layer, shape, cpu_seconds)

    full = shape == CONFIGS[name]
    res = {
        "value": replica_value(T, world, ms), "ms_per_step": ms,
        "dtype": "e4m3 weights, bf16 activations, fp32 accumulate" if fp8 else
                 "e2m1 weights, bf16 activations, fp32 accumulate" if fp4 else
                 "bf16 (fp32 accumulate, fp32 combine)",
        "config": {"workload": (WORKLOADS[name] if full else
                                f"{name} with the complete Hy3 block (+ a shared expert "
                                "and an e_score_correction_bias)" if block and
                                (T, E) == (CONFIGS[name].T, CONFIGS[name].E) else
                                f"smaller case of {name}: T={T}, E={E}"),
                   "T": T, "d": d, "E": E, "k": k,
                   "d_ff": F, "path": args.path, "parallelism": f"replicas x{world}",
                   "weights": ("e4m3 + fp32 row scales" if fp8 else
                               "e2m1 + e8m0 block-32 scales" if fp4 else
                               "bf16, packed in 128x64 blocks once at load (moe_pack_weights)"
                               if packed else "bf16, row-major"),
                   "l2": "no flush: each step streams the touched experts' weights "
                         f"({touched} experts, "
                         f"{touched * work.expert_bytes(d, F, fp8, fp4) / 1e9:.2f} GB) "
                         "through the 126 MB L2"},
        "roofline": roof,
        "layer_roofline": {
            "hbm_frac": lw["bytes"] / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "tensor_frac": lw["flops"] / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
            "algorithmic_bytes": lw["bytes"], "algorithmic_flops": lw["flops"],
            "touched_experts": touched},
        "stage_ms": stage_ms,
        "stage_timing": "a second pass of the same steps with an event between stages "
                        "(value and ms_per_step come from the pass without them)",
        "clocks": clocks.summary(),
        "e2e": {"value": replica_value(T, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 2,
                "ms_per_step": e2e_ms, "api": "moe_forward3",
                "copies": "one stream per direction, double-buffered, overlapping the compute",
                "output_equals_staged": e2e_same},
        "gpu_launches": sum(n_launch.values()) * args.steps,
        "status": [moe.moe_status_string(status), moe.moe_status_string(status2)],
        "cpu_baseline": cpu,
    }
    del layer, wgu, wd, ws, xp, h, y
    torch.cuda.empty_cache()
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="decode", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", default="auto", choices=["auto", "stream", "gemm"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-seconds", type=float, default=4.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="with --config decode, skip the prefill object of the line")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E (a smaller case of the same workload, e.g. for ncu)")
    ap.add_argument("--tokens", type=int, default=None, help="override T")
    ap.add_argument("--block", action="store_true",
                    help="the complete Hy3 block: + a shared expert and an "
                         "e_score_correction_bias (N(0, 0.05^2))")
    args = ap.parse_args()
    world, rank, local = dist_setup()
    if args.steps is None:
        args.steps = 10 if args.impl == "reference" else {"decode": 2000, "tiny": 2000}.get(
            args.config, 200)
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    from sparse_moe_transformer_gemm_b200 import moe

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    head = measure(args, args.config, dev, local, rank, world, pg, moe, block=args.block,
                   cpu_seconds=None if args.no_cpu_baseline else args.cpu_seconds)
    # The metric has two halves: % of the HBM roofline at decode and % of the
    # dense bf16 tensor peak at prefill. The decode line (the headline) carries
    # the prefill workload measured in the same run, every rank taking part.
    pre = None
    if args.config == "decode" and not args.no_prefill and not (args.experts or args.tokens):
        pre = measure(args, "prefill", dev, local, rank, world, pg, moe, block=args.block)
        pre = {"metric": "MoE-layer tokens/s", "unit": "tokens/s", "steps": args.steps,
               "warmup": args.warmup, **pre}
        del pre["cpu_baseline"]

    if rank == 0:
        line = {
            "metric": "MoE-layer tokens/s", "value": head["value"], "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": head["dtype"],
            "data": "synthetic (seeded; random-init weights of the Hy3 MoE layer shapes)",
        }
        line.update({k: v for k, v in head.items() if k not in line})
        if pre is not None:
            line["prefill"] = pre
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
