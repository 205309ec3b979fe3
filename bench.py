"""Benchmark of the fused FP8 block-scaled MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload prefill|decode|skewed|tiny|profile|gemm|mla_decode|mla_long|prefill_tp|prefill_ep]
                    [--tokens T] [--impl ours|reference]

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

--workload mla_decode / mla_long time the section's other decode kernel, MLA
decode over a paged latent KV cache (64 sequences, 16 heads, 544 or 8192 cached
tokens); the default run reports both under "workloads".

--impl reference times the CPU oracle (the plain reference of the same
computation) on the host cores on a bounded token sample of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import re
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp8_block_scaled_biased_b200 import inputs as I  # noqa: E402

WORKLOADS = {"tiny": I.TINY, "decode": I.DECODE, "prefill": I.PREFILL, "skewed": I.SKEWED, "profile": I.PROFILE,
             "prefill_ep8": I.PREFILL_EP8, "prefill_tp8": I.PREFILL_TP8}
# The prefill layer split over the torchrun ranks: over I (tensor parallel: one batch of
# 4096 tokens per step, every rank routes all of it, partial outputs reduced over NCCL) or
# over E (expert parallel: every rank its own batch of 4096 tokens and E/N experts,
# dispatch and return all-to-alls over NCCL).
DIST_WORKLOADS = {"prefill_tp": I.PREFILL, "prefill_ep": I.PREFILL}
DIST_PREHEAT_STEPS = 100
L2_FLUSH_BYTES = 256 << 20
METRIC = "fused FP8-blockscale MoE layer tokens/s and TFLOPS at 1 B200; % of FP8/HBM roofline"
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


def _nvml_handle(local):
    """NVML handle of CUDA device `local`, matched by PCI address (CUDA and NVML orders may differ)."""
    import pynvml
    pynvml.nvmlInit()
    props = torch.cuda.get_device_properties(local)
    bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
    return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus), bus


class ClockSampler:
    """SM clock, power and clock-event reasons of the benchmarked GPU, sampled
    every 10 ms (NVML, read-only queries) while the timed region runs."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, local, period_s=0.01):
        self.local = local
        self.period = period_s
        self.samples = []
        self.err = None
        self._stop = threading.Event()
        self.thread = None

    def start(self):
        try:
            self.nv, self.h, self.bus = _nvml_handle(self.local)
            self.max_mhz = self.nv.nvmlDeviceGetMaxClockInfo(self.h, self.nv.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 - sampling is best effort; the reason is reported
            self.err = f"nvml unavailable: {type(e).__name__}: {e}"
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv, h = self.nv, self.h
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, pw, rs))
            except Exception as e:  # noqa: BLE001
                self.err = f"nvml query failed: {e}"
                return
            time.sleep(self.period)

    def stop(self):
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "not sampled"]}
        self._stop.set()
        self.thread.join(timeout=5)
        reasons = set()
        for _, _, rs in self.samples:
            for name, const in self.REASONS:
                if rs & getattr(self.nv, const, 0):
                    reasons.add(name)
        sm = [x[0] for x in self.samples]
        pw = [x[1] for x in self.samples]
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
               "sm_mhz_min": min(sm) if sm else None, "power_w_median": statistics.median(pw) if pw else None,
               "reasons": sorted(reasons), "samples": len(sm), "period_ms": self.period * 1e3,
               "source": f"nvml, device {self.bus}"}
        if self.err:
            out["error"] = self.err
        return out


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


def ep_config(cfg):
    """Config keys of an expert- or tensor-parallel workload: which part of the layer it keeps."""
    out = {}
    if cfg.ep_ranks > 0:
        kept = torch.nonzero(I.expert_mask(cfg)).flatten()
        out["expert_parallel"] = (f"rank {cfg.ep_rank} of {cfg.ep_ranks}: experts {int(kept[0])}-{int(kept[-1])} "
                                  "(expert_mask), partial output of every token")
    if cfg.tp_ranks > 0:
        Is = cfg.I // cfg.tp_ranks
        out["tensor_parallel"] = (f"rank {cfg.tp_rank} of {cfg.tp_ranks}: intermediate columns "
                                  f"{cfg.tp_rank * Is}-{(cfg.tp_rank + 1) * Is - 1} of every expert, partial output "
                                  "of every token")
    return out


PREHEAT_SECONDS = 0.4


def preheat(step, flush, seconds=PREHEAT_SECONDS):
    """Untimed steps back to back for about `seconds` before the timed ones, so the timed
    steps run at the clock the 1000 W power limit settles at under sustained load rather
    than at the boost clock of a GPU coming out of idle."""
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    step()
    torch.cuda.synchronize()
    n = max(1, int(seconds / max(time.perf_counter() - t0, 1e-5)))
    for i in range(min(n, 20000)):
        flush.fill_(i & 0xFF)
        step()


def layer_work(cfg, ids, mask=None):
    """Algorithmic FLOPs and HBM bytes of one layer forward (padding excluded). With an
    expert mask only the kept experts' pairs count."""
    flat = ids.flatten().long().cpu()
    if mask is not None:
        flat = flat[mask.cpu().bool()[flat]]
    n_e = int(torch.unique(flat).numel())
    P = int(flat.numel())
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


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one gate/up GEMM
# launch from a one-pass ncu capture of this bench's own command, keyed by
# workload, with the SHA-256 of the GEMM kernel sources the capture ran. A
# figure whose sources have changed since is not reported.
GATE_UP_TRAFFIC = {
    "prefill_t4096_h7168_e256": {
        "bytes": 6.752e9,
        "sha256": "730be5c99bff17e3b4cfc065e91115dd7e912e0198471e5d7299704ee96b3daa",
        "capture": "ncu --metrics gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum of "
                   "`python bench.py --steps 2 --warmup 3 --no-cpu-baseline --no-graph --no-workloads` "
                   "(2 launches, mean; tiled weights)",
    },
}
GEMM_SOURCES = ("fp8_block_scaled_biased_b200/csrc/gemm_sm100.cuh", "fp8_block_scaled_biased_b200/csrc/common.cuh")


def source_sha(paths):
    """SHA-256 of C++ sources with comments and all whitespace removed, so that edits to
    comments or layout keep it and any change to the code changes it."""
    import hashlib
    import re
    h = hashlib.sha256()
    for path in paths:
        with open(path, encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)       # block comments
        text = re.sub(r"//[^\n]*", " ", text)                      # line comments
        h.update("".join(text.split()).encode())
    return h.hexdigest()


def gemm_source_sha():
    return source_sha(os.path.join(ROOT, rel) for rel in GEMM_SOURCES)


def gate_up_traffic(workload, override):
    if override is not None:
        return override, "given on the command line"
    rec = GATE_UP_TRAFFIC.get(workload)
    if rec is None:
        return None, "no capture for this workload"
    if rec["sha256"] != gemm_source_sha():
        return None, "kernel sources changed since the capture"
    return rec["bytes"], rec["capture"]


def e2e_pipelined(layer, step, logits, x, h_logits, h_x, h_out, steps, world):
    """ms per step of `steps` forwards fed from and drained to pinned host memory, with the
    copies of neighbouring steps overlapping the compute (two-deep double buffering)."""
    s_comp = torch.cuda.current_stream()
    s_h2d = torch.cuda.Stream(device=logits.device)
    s_d2h = torch.cuda.Stream(device=logits.device)
    d_logits = [torch.empty_like(logits) for _ in range(2)]
    d_x = [torch.empty_like(x) for _ in range(2)]
    d_out = [torch.empty_like(layer.out) for _ in range(2)]
    ev_h2d = [torch.cuda.Event() for _ in range(2)]
    ev_in_free = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    ev_d2h = [torch.cuda.Event() for _ in range(2)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record(s_comp)
    s_h2d.wait_event(start)
    s_d2h.wait_event(start)
    for i in range(steps):
        b = i % 2
        with torch.cuda.stream(s_h2d):
            if i >= 2:
                s_h2d.wait_event(ev_in_free[b])           # step i-2 has read this input buffer
            d_logits[b].copy_(h_logits, non_blocking=True)
            d_x[b].copy_(h_x, non_blocking=True)
            ev_h2d[b].record(s_h2d)
        s_comp.wait_event(ev_h2d[b])
        logits.copy_(d_logits[b])                           # into the forward's (graph's) input buffers
        x.copy_(d_x[b])
        ev_in_free[b].record(s_comp)
        step()
        if i >= 2:
            s_comp.wait_event(ev_d2h[b])                    # step i-2's output has left this buffer
        d_out[b].copy_(layer.out)
        ev_out[b].record(s_comp)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(ev_out[b])
            h_out[b].copy_(d_out[b], non_blocking=True)
            ev_d2h[b].record(s_d2h)
    s_comp.wait_stream(s_h2d)
    s_comp.wait_stream(s_d2h)
    end.record(s_comp)
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(start.elapsed_time(end), world) / steps


NOMINAL_HBM_GBS = 8000.0      # the ~8 TB/s HBM3e figure of the B200 spec sheet (context beside the measured peak)


def measure_layer(args, world, local, cfg, layer, flush, headline=True):
    """Times `args.steps` forwards of `layer` on its workload's seeded inputs (CUDA graph,
    L2 flushed between steps, after a preheat) and returns the bench result: headline keys,
    roofline of the dominant kernel, per-kernel times averaged over an instrumented run,
    and (headline only) the boost-clock context figure and the end-to-end figures."""
    from fp8_block_scaled_biased_b200 import binding as B

    dev = torch.device("cuda", local)
    act = I.moe_activations(cfg)
    logits, bias, x = act.logits.to(dev), act.bias.to(dev), act.x.to(dev)
    mask = I.expert_mask(cfg)
    mask_dev = mask.to(dev) if mask is not None else None
    stream = torch.cuda.current_stream()

    # warm-up (also the first, eager pass through every entry point)
    for _ in range(args.warmup):
        layer.forward(logits, bias, x, expert_mask=mask_dev)
    torch.cuda.synchronize()
    assert B.device_status() == 0, "device error word set during warm-up"
    work = layer_work(layer.cfg, layer.topk_ids, mask)

    # Two graphs of the forward: a plain one for the timed steps, and one holding the
    # fused call's per-kernel event records (the records add gaps between kernels,
    # about 20 us per forward, so they stay out of the headline timing).
    def capture(timing):
        B.timing_enable(timing)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            layer.forward(logits, bias, x, expert_mask=mask_dev)
        g.replay()
        torch.cuda.synchronize()
        return g

    graph = graph_timed = None
    if not args.no_graph:
        graph_timed = capture(True)
        graph = capture(False)
    B.timing_enable(False)

    def step():
        if graph is not None:
            graph.replay()
        else:
            layer.forward(logits, bias, x, expert_mask=mask_dev)

    def step_timed():
        if graph_timed is not None:
            graph_timed.replay()
        else:
            layer.forward(logits, bias, x, expert_mask=mask_dev)

    def run_steps(fn, n):
        st = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        en = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for i in range(n):
            flush.fill_(i & 0xFF)                   # evict L2 between steps (outside the events)
            st[i].record(stream)
            fn()
            en[i].record(stream)
        return st, en

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.05)
    preheat(step, flush)
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    starts, ends = run_steps(step, args.steps)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    barrier(world)
    # The same number of steps again, straight after, with the per-kernel event records.
    # The fused call's events hold one call's kernel durations, so each step is read
    # (a host wait of a few tens of microseconds) before the next one starts.
    if graph_timed is None:
        B.timing_enable(True)
    per_kernel = []
    instrumented = []
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        step_timed()
        t1.record(stream)
        per_kernel.append(B.timing_last())
        torch.cuda.synchronize()
        instrumented.append(t0.elapsed_time(t1))
    clocks = sampler.stop()
    B.timing_enable(False)
    instrumented_ms = statistics.mean(instrumented)
    kmean = [statistics.mean(k[j] for k in per_kernel) for j in range(4)]
    kmin = [min(k[j] for k in per_kernel) for j in range(4)]
    kmax = [max(k[j] for k in per_kernel) for j in range(4)]
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), world)
    ms_per_step = total_ms / args.steps
    status = B.device_status()
    if status:
        raise RuntimeError(f"device error word {status} after the timed steps")

    peaks = load_peaks()
    # The timed steps run back to back under the power limit: the tensor peak is the
    # sustained one (the burst one for the boost-clock context figure); nominal FP8:BF16 2:1.
    fp8_peak_tflops = 2.0 * peaks["bf16_tflops_sustained"]
    fp8_peak_burst = 2.0 * peaks["bf16_tflops"]
    hbm = peaks["hbm_gbs"]
    gat_ms, g1_ms, g2_ms, cmb_ms = kmean
    g1_t_bytes = work["gemm1_bytes"] / hbm / 1e9 * 1e3      # ms at peak HBM
    g1_t_flops = work["gemm1_flops"] / (fp8_peak_tflops * 1e12) * 1e3
    if g1_t_bytes >= g1_t_flops:
        achieved = work["gemm1_bytes"] / (g1_ms * 1e-3) / 1e9
        roofline = {"kernel": "moe_gate_up_gemm", "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                    "frac": achieved / hbm, "frac_vs_nominal_8tbs": achieved / NOMINAL_HBM_GBS}
    else:
        achieved = work["gemm1_flops"] / (g1_ms * 1e-3) / 1e12
        roofline = {"kernel": "moe_gate_up_gemm", "bound": "tensor", "achieved": achieved,
                    "peak": fp8_peak_tflops, "unit": "TFLOP/s", "frac": achieved / fp8_peak_tflops}
    roofline["traffic"], roofline["traffic_source"] = gate_up_traffic(cfg.name, args.traffic if headline else None)
    roofline["algorithmic"] = work["gemm1_bytes"] if roofline["bound"] == "hbm" else work["gemm1_flops"]
    roofline["launch_ms"] = g1_ms
    roofline["peak_source"] = peaks["source"] + (" sustained (fp8 = 2 x bf16)" if roofline["bound"] == "tensor" else "")
    t_layer_roof = max(work["flops"] / (fp8_peak_tflops * 1e12), work["layer_bytes"] / (hbm * 1e9)) * 1e3
    t_layer_roof_burst = max(work["flops"] / (fp8_peak_burst * 1e12), work["layer_bytes"] / (hbm * 1e9)) * 1e3
    t_layer_roof_nominal = max(work["flops"] / (fp8_peak_tflops * 1e12), work["layer_bytes"] / (NOMINAL_HBM_GBS * 1e9)) * 1e3
    mhz = clocks.get("sm_mhz")
    cycles = (lambda ms: ms * 1e-3 * mhz * 1e6) if mhz else (lambda ms: None)

    tokens = cfg.T * world
    result = {
        "metric": METRIC,
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
                   "cuda_graph": graph is not None, **ep_config(cfg)},
        "tflops": work["flops"] * world / (ms_per_step * 1e-3) / 1e12,
        "layer_roofline": {"ms": t_layer_roof, "frac": t_layer_roof / ms_per_step,
                           "frac_vs_nominal_8tbs": t_layer_roof_nominal / ms_per_step,
                           "flops": work["flops"], "bytes": work["layer_bytes"],
                           "touched_experts": work["n_experts"], "fp8_peak_tflops": fp8_peak_tflops,
                           "fp8_peak_source": peaks["source"] + " sustained (fp8 = 2 x bf16)",
                           "hbm_gbs": hbm, "hbm_source": peaks["source"]},
        "step_ms": {"median": statistics.median(step_ms), "min": min(step_ms), "max": max(step_ms)},
        "instrumented_ms_per_step": instrumented_ms,
        "kernels_ms": {"moe_gather": gat_ms, "moe_gate_up_gemm": g1_ms, "moe_down_gemm": g2_ms, "moe_combine": cmb_ms,
                       "route_sort_quant": instrumented_ms - sum(kmean),
                       "min": dict(zip(("moe_gather", "moe_gate_up_gemm", "moe_down_gemm", "moe_combine"), kmin)),
                       "max": dict(zip(("moe_gather", "moe_gate_up_gemm", "moe_down_gemm", "moe_combine"), kmax)),
                       "source": f"mean over the {args.steps} steps of a second run of the timed steps with the "
                                 "fused call's kernel events recorded; route_sort_quant = instrumented mean step - "
                                 "the four"},
        "kernels_mcycles": {"moe_gate_up_gemm": cycles(g1_ms) and cycles(g1_ms) / 1e6,
                            "moe_down_gemm": cycles(g2_ms) and cycles(g2_ms) / 1e6,
                            "sm_mhz": mhz, "source": "kernel ms x median sampled SM clock"},
        "roofline": roofline,
        "gpu_launches": args.steps * layer.launches_per_forward,
        "clocks": clocks,
        "wall_s_timed": wall,
    }
    if not headline:
        del graph, graph_timed
        return result

    # Context only: the same steps each started from an idle GPU (5 ms of host sleep
    # before each), i.e. at the boost clock of a layer run alone, not under sustained load.
    burst_ms = []
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        torch.cuda.synchronize()
        time.sleep(0.005)
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        step()
        b1.record(stream)
        torch.cuda.synchronize()
        burst_ms.append(b0.elapsed_time(b1))
    burst_ms_per_step = max_over_ranks(statistics.median(burst_ms), world)
    result["burst"] = {"ms_per_step": burst_ms_per_step,
                       "layer_roofline_frac": t_layer_roof_burst / burst_ms_per_step,
                       "method": "median of the same steps each started after 5 ms of idle GPU (boost clock); "
                                 "context only, the headline value is the sustained back-to-back run"}

    # End to end through the public API with host buffers. Serial: per step, the pinned H2D
    # copies of the inputs, the forward and the D2H copy of the output on one stream.
    h_logits = act.logits.pin_memory()
    h_x = act.x.pin_memory()
    h_out = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
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
        h_out[0].copy_(layer.out, non_blocking=True)
        e_end[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_serial_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_start, e_end)), world) / args.steps
    # Pipelined, as a serving loop runs it: two device input and output buffers; step i+1's
    # H2D and step i-1's D2H run on their own copy streams while step i computes. Every step
    # still moves its own inputs and output across PCIe; the time is that of all steps.
    e2e_ms = e2e_pipelined(layer, step, logits, x, h_logits, h_x, h_out, args.steps, world)
    result["e2e"] = {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
                     "h2d_bytes_per_step": act.logits.numel() * 4 + act.x.numel() * 2,
                     "d2h_bytes_per_step": cfg.T * cfg.H * 2, "ms_per_step": e2e_ms,
                     "method": "pinned host buffers through layer.forward; two-deep pipeline: step i+1's H2D and "
                               "step i-1's D2H overlap step i's forward on separate copy streams; no L2 flush "
                               "between these steps (each step reads its touched experts' weights, more than L2)",
                     "serial": {"value": tokens / (e2e_serial_ms * 1e-3), "ms_per_step": e2e_serial_ms}}
    del graph, graph_timed
    return result


# The other workloads of the same layer timed by the default run, next to the prefill
# headline: the decode and skewed batches (same expert weights) and the standalone GEMM.
EXTRA_WORKLOADS = ("decode", "skewed", "gemm", "mla_decode", "mla_long")
EXTRA_KEYS = ("value", "unit", "ms_per_step", "steps", "warmup", "tflops", "step_ms", "layer_roofline", "roofline",
              "kernels_ms", "kernels_mcycles", "clocks", "config", "gpu_launches", "l2_warm")


def run_distributed(args, world, rank, local):
    """prefill_tp / prefill_ep: the layer split over the ranks (eager steps: the step holds
    NCCL collectives and, for expert parallelism, a host read of the all-to-all counts)."""
    from fp8_block_scaled_biased_b200 import binding as B
    from fp8_block_scaled_biased_b200 import distributed as D
    from fp8_block_scaled_biased_b200.layer import MoELayer

    cfg = DIST_WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    act = I.moe_activations(cfg)
    logits, bias, x = act.logits.to(dev), act.bias.to(dev), act.x.to(dev)
    if args.workload == "prefill_tp":
        full = MoELayer(cfg, dev).load_synthetic_weights()
        model = D.TensorParallelMoE(full, reduce=args.tp_reduce)
        del full
        torch.cuda.empty_cache()
    else:
        e0, e1 = D.ep_expert_range(cfg.E, rank, world)
        shard = D.ExpertShard(cfg, e0, e1, dev).load_synthetic_weights()
        if args.ep_exchange == "peer":
            model = D.ExpertParallelPeerMoE(cfg, shard, cfg.T)
        else:
            model = D.ExpertParallelMoE(cfg, shard)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        out = model.forward(logits, bias, x)
    torch.cuda.synchronize()
    assert B.device_status() == 0, "device error word set during warm-up"
    topk_w = torch.empty(cfg.T, cfg.K, dtype=torch.float32, device=dev)      # the routing, for the work count
    topk_ids = torch.empty(cfg.T, cfg.K, dtype=torch.int32, device=dev)
    B.moe_biased_grouped_topk(logits, bias, topk_w, topk_ids, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    work = layer_work(cfg, topk_ids)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.05)
    # untimed steps before the timed ones, as preheat() does, but a fixed number of them:
    # every step holds collectives, so every rank must run the same count
    for i in range(DIST_PREHEAT_STEPS):
        flush.fill_(i & 0xFF)
        model.forward(logits, bias, x)
    barrier(world)
    torch.cuda.synchronize()
    st = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    en = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        st[i].record(stream)
        out = model.forward(logits, bias, x)
        en[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in zip(st, en)]
    ms_per_step = max_over_ranks(sum(step_ms), world) / args.steps
    if B.device_status():
        raise RuntimeError("device error word set during the timed steps")
    peaks = load_peaks()
    fp8_peak = 2.0 * peaks["bf16_tflops_sustained"]
    hbm = peaks["hbm_gbs"]
    tp = args.workload == "prefill_tp"
    batches = 1 if tp else world                   # token batches processed per step by the whole job
    flops = work["flops"] * batches
    wbytes = work["layer_bytes"] - (cfg.T * cfg.E * 4 + cfg.E * 4 + 4 * cfg.T * cfg.H)
    act_bytes = (cfg.T * cfg.E * 4 + cfg.E * 4 + 4 * cfg.T * cfg.H) * (world if tp else batches)
    t_roof = max(flops / world / (fp8_peak * 1e12), (wbytes + act_bytes) / world / (hbm * 1e9)) * 1e3
    tokens = cfg.T * batches
    del out
    return {
        "metric": METRIC, "value": tokens / (ms_per_step * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong" if tp else "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3fn x fp8_e4m3fn -> fp32 accumulate, bf16 out",
        "data": "synthetic (seeded; random-init weights quantised to FP8 in 128x128 blocks)",
        "config": {"workload": f"{cfg.name}_{'tp' if tp else 'ep'}{world}", "T": cfg.T, "H": cfg.H, "E": cfg.E,
                   "topk": cfg.K, "I": cfg.I,
                   "parallelism": (f"tp{world}: intermediate columns split over the ranks, one batch of {cfg.T} "
                                   "tokens per step, partial outputs summed " +
                                   ("by the combine fused with the all-reduce over peer memory" if args.tp_reduce ==
                                    "peer" else "by an fp32 NCCL reduce-scatter and a bf16 all-gather")) if tp else
                                  (f"ep{world}: experts split over the ranks, each rank its own batch of {cfg.T} "
                                   "tokens, " + ("dispatch and return over peer memory" if args.ep_exchange == "peer"
                                                 else "dispatch and return all-to-alls over NCCL")),
                   "l2": "flushed between steps (256 MB write)", "cuda_graph": False},
        "tflops": flops / (ms_per_step * 1e-3) / 1e12,
        "layer_roofline": {"ms": t_roof, "frac": t_roof / ms_per_step, "flops": flops,
                           "bytes": wbytes + act_bytes, "touched_experts": work["n_experts"],
                           "note": "whole-job work spread evenly over the ranks; collective time not in the bound"},
        "step_ms": {"median": statistics.median(step_ms), "min": min(step_ms), "max": max(step_ms)},
        "gpu_launches": None, "clocks": clocks,
    }


def run_tp_emulated(args, local):
    """prefill_tp with --tp-emulate N on one GPU: the N tensor-parallel ranks' forwards one
    after another, each without its combine (fused_moe_fp8_blockscale_g1u1_pairs), then their
    combine fused with the all-reduce as one cooperative launch (moe_combine_allreduce_emulated),
    every rank's CTAs running the one-rank code. A step is all N ranks' work on one GPU, so the
    line is no multi-GPU number; what it measures is the fused all-reduce kernel against the
    HBM copy rate (its stores stay in this GPU's memory)."""
    from fp8_block_scaled_biased_b200 import binding as B
    from fp8_block_scaled_biased_b200 import distributed as D
    from fp8_block_scaled_biased_b200.layer import MoELayer

    n = args.tp_emulate
    cfg = DIST_WORKLOADS["prefill_tp"]
    dev = torch.device("cuda", local)
    act = I.moe_activations(cfg)
    logits, bias, x = act.logits.to(dev), act.bias.to(dev), act.x.to(dev)
    full = MoELayer(cfg, dev).load_synthetic_weights()
    shards = [full.tp_shard(r, n) for r in range(n)]
    del full
    torch.cuda.empty_cache()
    emu = D.EmulatedTpAllReduce(cfg.T, cfg.H, n, dev)
    cap, Is = shards[0].sorted.capacity, cfg.I // n
    stream = torch.cuda.current_stream()

    def step(mid=None):
        ws = [sh.forward_pairs(logits, bias, x) for sh in shards]
        if mid is not None:
            mid.record(stream)
        return emu(ws, cap, cfg.K, Is)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert B.device_status() == 0, "device error word set during warm-up"
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.05)
    for i in range(DIST_PREHEAT_STEPS // 10):
        flush.fill_(i & 0xFF)
        step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        step(ev[i][1])
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if B.device_status():
        raise RuntimeError("device error word set during the timed steps")
    # every rank's output against bf16 of the rank-order fp32 sum of the ranks' own combines
    partials = [sh.forward(logits, bias, x).float() for sh in shards]
    want = partials[0]
    for p in partials[1:]:
        want = want + p
    outs = step()
    same = all(torch.equal(o, want.to(torch.bfloat16)) for o in outs)
    step_ms = [e[0].elapsed_time(e[2]) for e in ev]
    ar_ms = [e[1].elapsed_time(e[2]) for e in ev]
    ms_per_step = sum(step_ms) / args.steps
    ar = sum(ar_ms) / args.steps
    # per rank: its pair rows read (T*K*H bf16), its partial rows stored (T*H), its slice's n
    # partials read (~T*H) and the reduced slice stored into n outputs (~T*H)
    ar_bytes = n * cfg.T * cfg.H * 2 * (cfg.K + 3)
    hbm = load_peaks()["hbm_gbs"]
    return {
        "metric": METRIC, "value": cfg.T / (ms_per_step * 1e-3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "none (all ranks on one GPU)", "vs_baseline": None,
        "dtype": "fp8_e4m3fn x fp8_e4m3fn -> fp32 accumulate, bf16 out",
        "data": "synthetic (seeded; random-init weights quantised to FP8 in 128x128 blocks)",
        "config": {"workload": f"{cfg.name}_tp{n}_emulated_on_1_gpu", "T": cfg.T, "H": cfg.H, "E": cfg.E,
                   "topk": cfg.K, "I": cfg.I, "parallelism": f"tp{n} emulated: the {n} ranks' forwards in turn on "
                   "one GPU, then their fused combine + all-reduce as one cooperative launch",
                   "l2": "flushed between steps (256 MB write)", "cuda_graph": False},
        "allreduce": {"kernel": "tp_combine_allreduce_kernel", "bound": "hbm", "ms": ar,
                      "bytes": ar_bytes, "achieved": ar_bytes / (ar * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                      "frac": ar_bytes / (ar * 1e-3) / 1e9 / hbm, "peak_source": "measured",
                      "note": "CUDA events around the emulated launch; the ranks' stores stay in this GPU's memory"},
        "outputs_equal_rank_order_sum": same,
        "step_ms": {"median": statistics.median(step_ms), "min": min(step_ms), "max": max(step_ms)},
        "gpu_launches": None, "clocks": clocks,
    }


def run_ep_emulated(args, local):
    """prefill_ep with --ep-emulate N on one GPU: N expert-parallel ranks over peer memory
    (EmulatedExpertParallel), each with its own batch of T tokens and E/N experts, their steps
    in turn on one stream and their barriers as one launch; timed beside the one-GPU layer
    run on the same N batches. The difference is what the exchange adds (routing read across
    ranks, the owners' sorts over N*T tokens, the rows pulled in the gather and returned);
    no multi-GPU number."""
    from fp8_block_scaled_biased_b200 import binding as B
    from fp8_block_scaled_biased_b200 import distributed as D
    from fp8_block_scaled_biased_b200.layer import MoELayer

    n = args.ep_emulate
    cfg = DIST_WORKLOADS["prefill_ep"]
    dev = torch.device("cuda", local)
    layer = MoELayer(cfg, dev).load_synthetic_weights()
    shards = [D.ExpertShard(cfg, *D.ep_expert_range(cfg.E, r, n), dev).load_synthetic_weights() for r in range(n)]
    emu = D.EmulatedExpertParallel(cfg, shards, cfg.T, dev)
    inputs = []
    for r in range(n):
        act = I.moe_activations(dataclasses.replace(cfg, seed=cfg.seed + r))
        inputs.append((act.logits.to(dev), act.bias.to(dev), act.x.to(dev)))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for i, (a, b) in enumerate(ev):
            flush.fill_(i & 0xFF)
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.05)
    for _ in range(3):
        emu.forward(inputs)
    ep_ms = timed(lambda: emu.forward(inputs))
    for rk in emu.ranks:                  # the same with the rows returned by a separate kernel
        rk.return_in_gemm = False
    ep_kernel_ms = timed(lambda: emu.forward(inputs))
    for rk in emu.ranks:
        rk.return_in_gemm = True
    one_ms = timed(lambda: [layer.forward(*inp) for inp in inputs])
    clocks = sampler.stop()
    if B.device_status():
        raise RuntimeError("device error word set during the timed steps")
    outs = emu.forward(inputs)
    same = all(torch.equal(outs[r], layer.forward(*inputs[r])) for r in range(n))
    ms = sum(ep_ms) / len(ep_ms)
    base = sum(one_ms) / len(one_ms)
    return {
        "metric": METRIC, "value": n * cfg.T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "none (all ranks on one GPU)", "vs_baseline": None,
        "dtype": "fp8_e4m3fn x fp8_e4m3fn -> fp32 accumulate, bf16 out",
        "data": "synthetic (seeded; random-init weights quantised to FP8 in 128x128 blocks)",
        "config": {"workload": f"{cfg.name}_ep{n}_emulated_on_1_gpu", "T": cfg.T, "H": cfg.H, "E": cfg.E,
                   "topk": cfg.K, "I": cfg.I, "parallelism": f"ep{n} over peer memory emulated: {n} ranks' batches "
                   "and experts on one GPU, steps in turn, barriers as one launch",
                   "l2": "flushed between steps (256 MB write)", "cuda_graph": False},
        "one_gpu_layer_ms": base, "exchange_overhead": ms / base - 1.0, "outputs_equal_one_gpu_layer": same,
        "return_by_kernel_ms": sum(ep_kernel_ms) / len(ep_kernel_ms),
        "step_ms": {"median": statistics.median(ep_ms), "min": min(ep_ms), "max": max(ep_ms)},
        "gpu_launches": None, "clocks": clocks,
    }


def workload_config(args):
    """The MoE workload's configuration; with --tokens T, the same recipe (shapes, routing,
    value distributions, seed) at T tokens: one point of a batch-size sweep."""
    cfg = WORKLOADS[args.workload] if args.workload in WORKLOADS else DIST_WORKLOADS[args.workload]
    if args.tokens is None:
        return cfg
    return dataclasses.replace(cfg, name=re.sub(r"_t\d+_", f"_t{args.tokens}_", cfg.name, count=1), T=args.tokens)


def run_ours(args, world, rank, local):
    from fp8_block_scaled_biased_b200.layer import MoELayer

    if args.workload in DIST_WORKLOADS:
        if args.tp_emulate:
            return run_tp_emulated(args, local)
        if args.ep_emulate:
            return run_ep_emulated(args, local)
        return run_distributed(args, world, rank, local)
    cfg = workload_config(args)
    dev = torch.device("cuda", local)
    layer = MoELayer(cfg, dev).load_synthetic_weights()
    if cfg.tp_ranks > 0:                            # keep only this rank's shard of the weights
        layer = layer.tp_shard(cfg.tp_rank, cfg.tp_ranks)
        torch.cuda.empty_cache()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    result = measure_layer(args, world, local, cfg, layer, flush, headline=True)
    if args.workload == "prefill" and world == 1 and not args.no_workloads and args.tokens is None:
        extras = {}
        for name in EXTRA_WORKLOADS:
            if name == "gemm":
                r = run_gemm(args, world, rank, local, cpu=False)
            elif name in MLA_WORKLOADS:
                r = run_mla(args, world, rank, local, MLA_WORKLOADS[name], cpu=False)
            else:
                other = MoELayer(WORKLOADS[name], dev, weights_from=layer)
                r = measure_layer(args, world, local, WORKLOADS[name], other, flush, headline=False)
                del other
                torch.cuda.empty_cache()
            extras[name] = {k: r[k] for k in EXTRA_KEYS if k in r}
        result["workloads"] = extras
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cfg, args.cpu_sample_tokens, device=dev)
    return result


class OracleSample:
    """The oracle, as it stands, over a seeded sample of a workload's tokens.

    Setup (untimed, like the device layer's weight loading): the activations are
    drawn, the sample's experts found and their raw weights, drawn exactly as
    the device layer draws them (generator on `device`), quantised to FP8 in
    128x128 blocks. step() then times one pass of the path over the sample:
    routing, align/sort, 1x128 activation quantisation and the MoE layer with
    its combine. Every step computes the whole sample from scratch.
    """

    def __init__(self, cfg, n_tokens, device="cuda"):
        from oracle import fp8moe_oracle as O
        self.O, self.cfg = O, cfg
        act = I.moe_activations(cfg)
        g = torch.Generator().manual_seed(1234)
        tok = torch.sort(torch.randperm(cfg.T, generator=g)[:n_tokens]).values
        self.logits, self.x = act.logits[tok].contiguous(), act.x[tok].contiguous()
        self.bias = act.bias
        _, ids = O.biased_grouped_topk(self.logits, self.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
        self.mask = I.expert_mask(cfg)
        self.experts = [e for e in torch.unique(ids).tolist() if self.mask is None or self.mask[e]]
        self.weights = {}
        for e in self.experts:
            w1 = I.expert_weight_raw(cfg, "w1", e, device).cpu()
            w2 = I.expert_weight_raw(cfg, "w2", e, device).cpu()
            w1q, w1s, w2q, w2s = (*O.quant_128x128(w1), *O.quant_128x128(w2))
            if cfg.tp_ranks > 0:                    # the rank's intermediate columns only
                Is, nb, r = cfg.I // cfg.tp_ranks, cfg.I // cfg.tp_ranks // 128, cfg.tp_rank
                rows = torch.cat([torch.arange(r * Is, (r + 1) * Is), cfg.I + torch.arange(r * Is, (r + 1) * Is)])
                brows = torch.cat([torch.arange(r * nb, (r + 1) * nb),
                                   cfg.I // 128 + torch.arange(r * nb, (r + 1) * nb)])
                w1q, w1s, w2q, w2s = w1q[rows], w1s[brows], w2q[:, r * Is:(r + 1) * Is], w2s[:, r * nb:(r + 1) * nb]
            self.weights[e] = (w1q, w1s, w2q, w2s)
        self.n = n_tokens

    def step(self):
        O, cfg = self.O, self.cfg
        t0 = time.perf_counter()
        w, ids = O.biased_grouped_topk(self.logits, self.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
        O.align_sort(ids, w, cfg.E, 128, expert_mask=self.mask)
        a8, asc = O.quant_1x128(self.x)
        O.moe_layer(a8, asc, ids, w, self.weights.__getitem__, expert_mask=self.mask)
        return time.perf_counter() - t0


def cpu_baseline(cfg, n_tokens, device="cuda", min_seconds=10.0):
    """The oracle on the host cores: repeated passes over an n-token sample until min_seconds have run."""
    runner = OracleSample(cfg, n_tokens, device)
    times = []
    while sum(times) < min_seconds:
        times.append(runner.step())
    sec = sum(times) / len(times)
    return {"value": n_tokens / sec, "unit": "tokens/s", "cores": torch.get_num_threads(), "kind": "oracle",
            "sample": f"{n_tokens} seeded tokens of {cfg.name} ({len(runner.experts)} experts, weights quantised "
                      f"before timing), {len(times)} passes in {sum(times):.1f} s"}


def run_gemm(args, world, rank, local, cpu=True):
    """The standalone block-scale GEMM (C = A . B^T with 1x128 / 128x128 FP8 scales), A pre-quantised.
    cpu=False leaves out the oracle's CPU baseline."""
    from fp8_block_scaled_biased_b200 import binding as B

    cfg = I.GEMM
    dev = torch.device("cuda", local)
    a, b = I.gemm_inputs(cfg, device=dev)
    qa, sa = B.fp8_per_token_group_quant(a, 128)
    qb, sb = B.fp8_per_block_quant(b)
    c = torch.empty(cfg.M, cfg.N, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        B.fp8_blockscale_gemm(qa, qb, sa, sb, out=c)
    torch.cuda.synchronize()

    def timed(flush_l2):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        preheat(lambda: B.fp8_blockscale_gemm(qa, qb, sa, sb, out=c), flush)
        barrier(world)
        torch.cuda.synchronize()
        for i in range(args.steps):
            if flush_l2:
                flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            B.fp8_blockscale_gemm(qa, qb, sa, sb, out=c)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ms = [x.elapsed_time(y) for x, y in ev]
        return max_over_ranks(sum(ms), world) / args.steps, ms

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.05)
    ms_flushed, per_step = timed(True)
    clocks = sampler.stop()
    ms_warm, _ = timed(False)
    if B.device_status():
        raise RuntimeError("device error word set by the GEMM")

    # end to end: pinned host A (FP8 codes + scales) in, bf16 C out
    h_qa, h_sa = qa.cpu().pin_memory(), sa.cpu().pin_memory()
    h_c = torch.empty(cfg.M, cfg.N, dtype=torch.bfloat16).pin_memory()
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e0[i].record(stream)
        qa.copy_(h_qa, non_blocking=True)
        sa.copy_(h_sa, non_blocking=True)
        B.fp8_blockscale_gemm(qa, qb, sa, sb, out=c)
        h_c.copy_(c, non_blocking=True)
        e1[i].record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(x.elapsed_time(y) for x, y in zip(e0, e1)), world) / args.steps

    flops = 2.0 * cfg.M * cfg.N * cfg.K
    peaks = load_peaks()
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    tf = flops * world / (ms_flushed * 1e-3) / 1e12
    result = {
        "metric": "FP8 block-scale GEMM TFLOP/s at 1 B200 (C = A.B^T, 1x128 / 128x128 fp32 scales, bf16 out)",
        "value": tf, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_flushed, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3fn x fp8_e4m3fn -> fp32 accumulate, bf16 out", "data": "synthetic (seeded)",
        "config": {"workload": cfg.name, "M": cfg.M, "N": cfg.N, "K": cfg.K,
                   "l2": "flushed between steps (256 MB write)", "parallelism": f"dp{world} (independent GEMMs)"},
        "l2_warm": {"ms_per_step": ms_warm, "tflops": flops / (ms_warm * 1e-3) / 1e12},
        "step_ms": {"median": statistics.median(per_step), "min": min(per_step), "max": max(per_step)},
        "roofline": {"kernel": "fp8_blockscale_gemm", "bound": "tensor", "achieved": flops / (ms_flushed * 1e-3) / 1e12,
                     "peak": fp8_peak, "unit": "TFLOP/s", "frac": flops / (ms_flushed * 1e-3) / 1e12 / fp8_peak,
                     "traffic": None, "peak_source": peaks["source"] + " (fp8 = 2 x bf16)"},
        "e2e": {"value": flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": qa.numel() + sa.numel() * 4, "d2h_bytes_per_step": c.numel() * 2},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if cpu and rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import fp8moe_oracle as O
        rows = torch.arange(0, cfg.M, cfg.M // 8)
        qa_h, sa_h = O.quant_1x128(a[rows].cpu())
        qb_h, sb_h = O.quant_128x128(b.cpu())
        t0 = time.perf_counter()
        O.blockscale_gemm(qa_h, sa_h, qb_h, sb_h)
        dt = time.perf_counter() - t0
        result["cpu_baseline"] = {"value": 2.0 * len(rows) * cfg.N * cfg.K / dt / 1e12, "unit": "TFLOP/s",
                                  "cores": torch.get_num_threads(), "kind": "oracle",
                                  "sample": f"{len(rows)} of {cfg.M} rows, operands quantised before timing, {dt:.1f} s"}
    return result


MLA_WORKLOADS = {"mla_decode": I.MLA_DECODE, "mla_long": I.MLA_LONG}
MLA_METRIC = "MLA decode (paged latent KV, 576/512 head dims) sequences decoded/s at 1 B200; % of HBM roofline"


def mla_work(cfg):
    """Algorithmic bytes of one decode step: every cached KV row once, q, o, lse and the
    page table (the split partials are the kernel's own traffic, not counted), and FLOPs:
    QK^T over 576 entries and PV over 512 per head and token."""
    rows = sum(cfg.lengths())
    pages = sum((n + cfg.page_size - 1) // cfg.page_size for n in cfg.lengths())
    nbytes = (rows * cfg.Dk * 2 + cfg.B * cfg.Hq * (cfg.Dk * 2 + cfg.Dv * 2 + 4)
              + pages * 4 + (2 * cfg.B + 1) * 4)
    flops = 2 * rows * cfg.Hq * (cfg.Dk + cfg.Dv)
    return nbytes, flops


class MlaOracleSample:
    """The MLA oracle, as it stands, over the first n sequences of a workload (inputs drawn
    once, untimed); step() times one decode of the sample."""

    def __init__(self, cfg, n_seqs):
        from oracle import mla_oracle as M
        self.M = M
        sub = I.MlaConfig(cfg.name + "_sample", B=n_seqs, Hq=cfg.Hq, L=tuple(cfg.lengths()[:n_seqs]),
                          page_size=cfg.page_size, seed=cfg.seed)
        self.x = I.mla_inputs(sub)
        self.n = n_seqs

    def step(self):
        x = self.x
        t0 = time.perf_counter()
        self.M.mla_decode(x.q, x.kv_buffer, x.kv_indptr, x.kv_indices, x.kv_last_page_lens)
        return time.perf_counter() - t0


def run_mla(args, world, rank, local, cfg, cpu=True):
    """MLA decode (mla_decode_fwd) on a seeded paged batch: device-timed steps with L2
    flushed between them, the roofline of the call, end to end with q and the page
    table copied in and o copied out, and the oracle's CPU baseline."""
    from fp8_block_scaled_biased_b200 import binding as B

    dev = torch.device("cuda", local)
    x = I.mla_inputs(cfg, device=dev)
    o = torch.empty(cfg.B, cfg.Hq, cfg.Dv, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(cfg.B, cfg.Hq, dtype=torch.float32, device=dev)
    splits = B.mla_decode_num_splits(cfg.B, cfg.Hq)
    need = B.mla_decode_workspace_bytes(cfg.B, cfg.Hq, splits)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        B.mla_decode_fwd(x.q, x.kv_buffer, o, x.kv_indptr, x.kv_indices, x.kv_last_page_lens, lse=lse,
                         num_kv_splits=splits, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    def timed(flush_l2):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        preheat(step, flush)
        barrier(world)
        torch.cuda.synchronize()
        for i in range(args.steps):
            if flush_l2:
                flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ms = [a.elapsed_time(b) for a, b in ev]
        return max_over_ranks(sum(ms), world) / args.steps, ms

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.05)
    ms_flushed, per_step = timed(True)
    clocks = sampler.stop()
    ms_warm, _ = timed(False)
    if B.device_status():
        raise RuntimeError("device error word set by MLA decode")

    # end to end: q and the page table from pinned host memory, o back to it (the KV cache stays resident)
    h_in = [t.cpu().pin_memory() for t in (x.q, x.kv_indptr, x.kv_indices, x.kv_last_page_lens)]
    h_o = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e0[i].record(stream)
        for d, h in zip((x.q, x.kv_indptr, x.kv_indices, x.kv_last_page_lens), h_in):
            d.copy_(h, non_blocking=True)
        step()
        h_o.copy_(o, non_blocking=True)
        e1[i].record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(e0, e1)), world) / args.steps

    nbytes, flops = mla_work(cfg)
    peaks = load_peaks()
    hbm = peaks["hbm_gbs"]
    gbs = nbytes / (ms_flushed * 1e-3) / 1e9
    result = {
        "metric": MLA_METRIC,
        "value": cfg.B * world / (ms_flushed * 1e-3), "unit": "sequences/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_flushed, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 x bf16 -> fp32 (softmax weights rounded to bf16), bf16 out",
        "data": "synthetic (seeded)",
        "config": {"workload": cfg.name, "B": cfg.B, "heads": cfg.Hq, "kv_len": cfg.L, "page_size": cfg.page_size,
                   "qk_head_dim": cfg.Dk, "v_head_dim": cfg.Dv, "num_kv_splits": splits,
                   "l2": "flushed between steps (256 MB write)", "parallelism": f"dp{world} (independent batches)"},
        "tflops": flops / (ms_flushed * 1e-3) / 1e12,
        "l2_warm": {"ms_per_step": ms_warm, "gbs": nbytes / (ms_warm * 1e-3) / 1e9},
        "step_ms": {"median": statistics.median(per_step), "min": min(per_step), "max": max(per_step)},
        "roofline": {"kernel": "mla_decode_fwd (decode kernel + split combine, timed together)", "bound": "hbm",
                     "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm, "traffic": None,
                     "algorithmic_bytes": nbytes, "peak_source": peaks["source"]},
        "e2e": {"value": cfg.B * world / (e2e_ms * 1e-3), "unit": "sequences/s",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in h_in),
                "d2h_bytes_per_step": o.numel() * 2},
        "gpu_launches": args.steps * (2 if splits > 1 else 1),
        "clocks": clocks,
    }
    if cpu and rank == 0 and world == 1 and not args.no_cpu_baseline:
        runner = MlaOracleSample(cfg, min(cfg.B, 8))
        times = []
        while sum(times) < 5.0:
            times.append(runner.step())
        sec = sum(times) / len(times)
        result["cpu_baseline"] = {"value": runner.n / sec, "unit": "sequences/s", "cores": torch.get_num_threads(),
                                  "kind": "oracle",
                                  "sample": f"first {runner.n} sequences of {cfg.name}, {len(times)} passes in "
                                            f"{sum(times):.1f} s"}
    return result


def run_reference_mla(args, world, cfg):
    runner = MlaOracleSample(cfg, min(cfg.B, 4))
    for _ in range(args.warmup):
        runner.step()
    times = [runner.step() for _ in range(args.steps)]
    sec = statistics.mean(times)
    value = runner.n / sec
    return {
        "impl": "reference", "metric": MLA_METRIC, "value": value, "unit": "sequences/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": cfg.name, "B": cfg.B, "heads": cfg.Hq, "kv_len": cfg.L, "page_size": cfg.page_size},
        "cpu_baseline": {"value": value, "unit": "sequences/s", "cores": torch.get_num_threads(), "kind": "oracle",
                         "sample": f"first {runner.n} sequences of {cfg.name} per step"},
        "e2e": {"value": value, "unit": "sequences/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference_gemm(args, world):
    """The oracle's block-scale GEMM on a fixed sample of 8 rows of A per step (operands quantised before timing)."""
    from oracle import fp8moe_oracle as O
    cfg = I.GEMM
    a, b = I.gemm_inputs(cfg, device="cpu")
    rows = torch.arange(0, cfg.M, cfg.M // 8)
    qa, sa = O.quant_1x128(a[rows])
    qb, sb = O.quant_128x128(b)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        O.blockscale_gemm(qa, sa, qb, sb)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = statistics.mean(times)
    value = 2.0 * len(rows) * cfg.N * cfg.K / sec / 1e12
    return {
        "impl": "reference",
        "metric": "FP8 block-scale GEMM TFLOP/s at 1 B200 (C = A.B^T, 1x128 / 128x128 fp32 scales, bf16 out)",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": cfg.name, "M": cfg.M, "N": cfg.N, "K": cfg.K},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": torch.get_num_threads(), "kind": "oracle",
                         "sample": f"{len(rows)} of {cfg.M} rows of A per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference(args, world, rank):
    if args.workload == "gemm":
        return run_reference_gemm(args, world)
    if args.workload in MLA_WORKLOADS:
        return run_reference_mla(args, world, MLA_WORKLOADS[args.workload])
    cfg = workload_config(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    runner = OracleSample(cfg, args.ref_sample_tokens, device=dev)
    for _ in range(args.warmup):
        runner.step()
    times = [runner.step() for _ in range(args.steps)]
    sec = statistics.mean(times)
    n = args.ref_sample_tokens
    value = n / sec
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 (fp32 where a routing choice or an FP8 code is decided)",
        "data": "synthetic (seeded)",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "groups": cfg.G,
                   "topk_group": cfg.TG, "topk": cfg.K, "I": cfg.I, **ep_config(cfg)},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": torch.get_num_threads(), "kind": "oracle",
                         "sample": f"{n} seeded tokens of {cfg.name} per step ({len(runner.experts)} experts, "
                                   "weights quantised before timing)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(DIST_WORKLOADS) + ["gemm"] + sorted(MLA_WORKLOADS),
                    default="prefill",
                    help="MoE layer workload; gemm: the standalone block-scale GEMM (M=2048, N=4096, K=7168); "
                         "mla_decode / mla_long: MLA decode of 64 sequences of 544 / 8192 cached tokens, 16 heads")
    ap.add_argument("--tokens", type=int, default=None,
                    help="run the MoE workload's recipe at this many tokens (a batch-size sweep point; the "
                         "workloads timed beside the prefill headline are then left out)")
    ap.add_argument("--tp-reduce", choices=["peer", "nccl"], default="peer",
                    help="prefill_tp: sum the ranks' partials with the combine fused with the all-reduce over "
                         "peer memory (peer) or with NCCL's reduce-scatter and all-gather (nccl)")
    ap.add_argument("--ep-exchange", choices=["peer", "nccl"], default="peer",
                    help="prefill_ep: dispatch and return over peer memory (peer) or NCCL all-to-alls (nccl)")
    ap.add_argument("--ep-emulate", type=int, default=0,
                    help="prefill_ep on one GPU: N expert-parallel ranks over peer memory there, timed beside the "
                         "one-GPU layer on the same batches (a measurement of the exchange, not a multi-GPU number)")
    ap.add_argument("--tp-emulate", type=int, default=0,
                    help="prefill_tp on one GPU: run all N ranks there, their fused combine + all-reduce as one "
                         "launch (a kernel measurement, not a multi-GPU number)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of replaying a CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="prefill only: leave out the decode, skewed, GEMM and MLA decode workloads timed beside the "
                         "headline")
    ap.add_argument("--cpu-sample-tokens", type=int, default=8,
                    help="tokens of the workload the oracle runs for cpu_baseline")
    ap.add_argument("--ref-sample-tokens", type=int, default=1,
                    help="tokens of the workload the oracle runs per step under --impl reference")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch of the gate/up GEMM from an ncu capture (reported as is)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    if args.tokens is not None and (args.tokens < 1 or args.workload not in WORKLOADS):
        ap.error("--tokens takes a positive count and a single-GPU MoE workload")
    if args.tp_emulate and (args.workload != "prefill_tp" or args.gpus != 1 or not 2 <= args.tp_emulate <= 8
                            or DIST_WORKLOADS["prefill_tp"].I % (128 * args.tp_emulate)):
        ap.error("--tp-emulate takes 2..8 ranks that split I into 128-column blocks, with prefill_tp on one GPU")
    if args.ep_emulate and (args.workload != "prefill_ep" or args.gpus != 1 or not 2 <= args.ep_emulate <= 8
                            or DIST_WORKLOADS["prefill_ep"].E % args.ep_emulate):
        ap.error("--ep-emulate takes 2..8 ranks that split E evenly, with prefill_ep on one GPU")
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps(run_reference(args, world, rank)), flush=True)
        else:
            if args.workload == "gemm":
                res = run_gemm(args, world, rank, local)
            elif args.workload in MLA_WORKLOADS:
                res = run_mla(args, world, rank, local, MLA_WORKLOADS[args.workload])
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
