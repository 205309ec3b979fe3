"""Benchmark of the fused FP8 block-scaled MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill|decode|skewed|tiny|profile]
                    [--impl ours|reference]

One step = one forward of the whole layer on the device: biased grouped top-k
routing -> align/sort -> 1x128 activation quantisation -> fused g1u1 MoE
(gate/up GEMM + SiLU*up + FP8 requant, down GEMM, deterministic combine), from
fp32 router logits and bf16 hidden states resident in HBM to the bf16 output.
The default workload is the DeepSeek-V3-shaped prefill layer (T=4096, H=7168,
E=256 in 8 groups, topk_group 4, topk 8, I=2048) with seeded synthetic inputs
and random-init weights quantised to FP8 in 128x128 blocks.

Timing: W untimed warm-up steps, then K steps, each bracketed by its own CUDA
events on the launching stream with a 256 MB L2 flush between steps (outside
the events); barrier + synchronize around the whole timed loop; max over
ranks. Under torchrun every rank runs its own batch of T tokens on its own
full copy of the layer (weak scaling, no collective on the data path).

--impl reference times the CPU oracle (the plain reference of the same
computation) on the host cores on a bounded token sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp8_block_scaled_biased_b200 import inputs as I  # noqa: E402

WORKLOADS = {"tiny": I.TINY, "decode": I.DECODE, "prefill": I.PREFILL, "skewed": I.SKEWED, "profile": I.PROFILE}
L2_FLUSH_BYTES = 256 << 20
EXPERT_W1_BYTES = lambda c: 2 * c.I * c.H + (2 * c.I // 128) * (c.H // 128) * 4   # noqa: E731
EXPERT_W2_BYTES = lambda c: c.H * c.I + (c.H // 128) * (c.I // 128) * 4            # noqa: E731


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def layer_work(cfg, ids):
    """Algorithmic FLOPs and HBM bytes of one layer forward (padding excluded)."""
    n_e = int(torch.unique(ids).numel())
    P = cfg.T * cfg.K
    flops = 2 * P * cfg.H * 2 * cfg.I + 2 * P * cfg.I * cfg.H
    act_bytes = cfg.T * cfg.E * 4 + cfg.E * 4 + cfg.T * cfg.H * 2 + cfg.T * cfg.H * 2
    layer_bytes = n_e * (EXPERT_W1_BYTES(cfg) + EXPERT_W2_BYTES(cfg)) + act_bytes
    # the gate/up GEMM alone: its weights, the FP8 activations and scales it reads,
    # the FP8 intermediate and scales it writes
    gemm1_bytes = (n_e * EXPERT_W1_BYTES(cfg) + cfg.T * cfg.H + cfg.T * (cfg.H // 128) * 4
                   + P * cfg.I + P * (cfg.I // 128) * 4)
    gemm1_flops = 2 * P * cfg.H * 2 * cfg.I
    return dict(n_experts=n_e, flops=flops, layer_bytes=layer_bytes, gemm1_bytes=gemm1_bytes,
                gemm1_flops=gemm1_flops)


def run_ours(args, world, rank, local):
    from fp8_block_scaled_biased_b200 import binding as B
    from fp8_block_scaled_biased_b200.layer import MoELayer

    cfg = WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    layer = MoELayer(cfg, dev).load_synthetic_weights()
    act = I.moe_activations(cfg)
    logits, bias, x = act.logits.to(dev), act.bias.to(dev), act.x.to(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    # warm-up (also the first, eager pass through every entry point)
    for _ in range(args.warmup):
        layer.forward(logits, bias, x)
    torch.cuda.synchronize()
    assert B.device_status() == 0, "device error word set during warm-up"
    work = layer_work(cfg, layer.topk_ids)

    B.timing_enable(True)          # before capture, so the graph holds the per-kernel event records
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layer.forward(logits, bias, x)
        graph.replay()
        torch.cuda.synchronize()

    def step():
        if graph is not None:
            graph.replay()
        else:
            layer.forward(logits, bias, x)

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    kernel_ms = []
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    wall0 = time.perf_counter()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)                       # evict L2 between steps (outside the events)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
        kernel_ms.append(B.timing_last())
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    barrier(world)
    clocks = sampler.stop()
    B.timing_enable(False)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), world)
    ms_per_step = total_ms / args.steps
    status = B.device_status()
    if status:
        raise RuntimeError(f"device error word {status} after the timed steps")

    # end to end through the public API with host buffers: pinned H2D inputs, forward, D2H output
    h_logits = act.logits.pin_memory()
    h_x = act.x.pin_memory()
    h_out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory()
    e_start = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_end = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e_start[i].record(stream)
        logits.copy_(h_logits, non_blocking=True)
        x.copy_(h_x, non_blocking=True)
        step()
        h_out.copy_(layer.out, non_blocking=True)
        e_end[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_start, e_end)), world) / args.steps

    peaks = load_peaks()
    fp8_peak_tflops = 2.0 * peaks["bf16_tflops"]           # nominal FP8:BF16 dense ratio 2:1
    hbm = peaks["hbm_gbs"]
    g1_ms = statistics.mean(k[0] for k in kernel_ms)
    g2_ms = statistics.mean(k[1] for k in kernel_ms)
    cmb_ms = statistics.mean(k[2] for k in kernel_ms)
    g1_t_bytes = work["gemm1_bytes"] / hbm / 1e9 * 1e3      # ms at peak HBM
    g1_t_flops = work["gemm1_flops"] / (fp8_peak_tflops * 1e12) * 1e3
    if g1_t_bytes >= g1_t_flops:
        roofline = {"kernel": "moe_gate_up_gemm", "bound": "hbm", "achieved": work["gemm1_bytes"] / (g1_ms * 1e-3) / 1e9,
                    "peak": hbm, "unit": "GB/s"}
    else:
        roofline = {"kernel": "moe_gate_up_gemm", "bound": "tensor",
                    "achieved": work["gemm1_flops"] / (g1_ms * 1e-3) / 1e12, "peak": fp8_peak_tflops, "unit": "TFLOP/s"}
    roofline["frac"] = roofline["achieved"] / roofline["peak"]
    roofline["traffic"] = args.traffic
    roofline["peak_source"] = peaks["source"] + (" (fp8 = 2 x bf16)" if roofline["bound"] == "tensor" else "")
    t_layer_roof = max(work["flops"] / (fp8_peak_tflops * 1e12), work["layer_bytes"] / (hbm * 1e9)) * 1e3

    tokens = cfg.T * world
    result = {
        "metric": "fused FP8-blockscale MoE layer tokens/s at 1 B200 (TFLOPS and % of FP8/HBM roofline alongside)",
        "value": tokens / (ms_per_step * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8_e4m3fn x fp8_e4m3fn -> fp32 accumulate, bf16 out",
        "data": "synthetic (seeded; random-init weights quantised to FP8 in 128x128 blocks)",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "groups": cfg.G,
                   "topk_group": cfg.TG, "topk": cfg.K, "I": cfg.I, "block_m": layer.block_m,
                   "parallelism": f"dp{world} (replicated layer, token batches per GPU)",
                   "l2": "flushed between steps (256 MB write); touched expert weights exceed L2 anyway",
                   "cuda_graph": graph is not None},
        "tflops": work["flops"] * world / (ms_per_step * 1e-3) / 1e12,
        "layer_roofline": {"ms": t_layer_roof, "frac": t_layer_roof / ms_per_step,
                           "flops": work["flops"], "bytes": work["layer_bytes"],
                           "touched_experts": work["n_experts"], "fp8_peak_tflops": fp8_peak_tflops,
                           "hbm_gbs": hbm},
        "kernels_ms": {"moe_gate_up_gemm": g1_ms, "moe_down_gemm": g2_ms, "moe_combine": cmb_ms,
                       "route_sort_quant": ms_per_step - g1_ms - g2_ms - cmb_ms},
        "roofline": roofline,
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": act.logits.numel() * 4 + act.x.numel() * 2,
                "d2h_bytes_per_step": cfg.T * cfg.H * 2},
        "gpu_launches": args.steps * layer.LAUNCHES_PER_FORWARD,
        "clocks": clocks,
        "wall_s_timed": wall,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cfg, args.cpu_sample_tokens, device=dev)
    del graph
    return result


def cpu_baseline(cfg, n_tokens, device="cuda"):
    """The oracle, as it stands, on a seeded sample of the workload's tokens (host cores)."""
    from oracle import fp8moe_oracle as O

    act = I.moe_activations(cfg)
    g = torch.Generator().manual_seed(1234)
    tokens = torch.sort(torch.randperm(cfg.T, generator=g)[:n_tokens]).values
    # raw expert weights: the same draws the device layer used (generator on `device`), copied to the host
    w_ref, ids_ref = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    experts = torch.unique(ids_ref[tokens]).tolist()
    raw = {e: (I.expert_weight_raw(cfg, "w1", e, device).cpu(), I.expert_weight_raw(cfg, "w2", e, device).cpu())
           for e in experts}
    threads = torch.get_num_threads()
    t0 = time.perf_counter()
    w, ids = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    a8, asc = O.quant_1x128(act.x[tokens])

    def get(e):
        q1, s1 = O.quant_128x128(raw[e][0])
        q2, s2 = O.quant_128x128(raw[e][1])
        return q1, s1, q2, s2

    O.moe_layer(a8, asc, ids[tokens], w[tokens], get)
    dt = time.perf_counter() - t0
    return {"value": n_tokens / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n_tokens} seeded tokens of {cfg.name} (routing on all {cfg.T} tokens, "
                      f"{len(experts)} experts quantised and applied), {dt:.1f} s"}


def run_reference(args, world, rank):
    cfg = WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    times = []
    n = args.cpu_sample_tokens
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(cfg, n, device=dev)
        if i >= args.warmup:
            times.append(n / r["value"])
    sec = statistics.mean(times)
    value = n / sec
    return {
        "impl": "reference",
        "metric": "fused FP8-blockscale MoE layer tokens/s at 1 B200 (TFLOPS and % of FP8/HBM roofline alongside)",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp64 oracle (fp32 where a routing choice or FP8 code is decided)",
        "data": "synthetic (seeded)",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "topk": cfg.K, "I": cfg.I},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": torch.get_num_threads(), "kind": "oracle",
                         "sample": f"{n} seeded tokens of {cfg.name} per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="prefill")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of replaying a CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=2)
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch of the gate/up GEMM from an ncu capture (reported as is)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps(run_reference(args, world, rank)), flush=True)
        else:
            res = run_ours(args, world, rank, local)
            if rank == 0:
                print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
