"""Host-side logic of bench.py, on the CPU: the reference arm's JSON line (one
rank and two gloo ranks), the traffic table's source check and the algorithmic
work counts the roofline divides by."""
import json
import os
import subprocess
import sys

import pytest
import torch

import bench
from fp8_block_scaled_biased_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _json_lines(text):
    out = []
    for ln in text.splitlines():
        ln = ln.strip()
        if ln.startswith("{"):
            out.append(json.loads(ln))
    return out


def test_reference_arm_line_on_one_rank():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"] == I.TINY.name
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_two_gloo_ranks_print_one_line():
    env = dict(os.environ, MASTER_ADDR="127.0.0.1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", "29541", "bench.py", "--impl", "reference",
           "--workload", "tiny", "--gpus", "2", "--steps", "1", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1 and lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2


def test_traffic_reported_only_for_unchanged_sources(monkeypatch):
    sha = bench.gemm_source_sha()
    monkeypatch.setattr(bench, "GATE_UP_TRAFFIC", {
        "w_same": {"bytes": 123.0, "sha256": sha, "capture": "c"},
        "w_old": {"bytes": 456.0, "sha256": "0" * 64, "capture": "c"},
    })
    assert bench.gate_up_traffic("w_same", None) == (123.0, "c")
    assert bench.gate_up_traffic("w_old", None)[0] is None
    assert bench.gate_up_traffic("w_none", None)[0] is None
    assert bench.gate_up_traffic("w_old", 7.0) == (7.0, "given on the command line")


def test_layer_work_counts():
    cfg = I.TINY
    ids = torch.tensor([[0, 1, 2, 3]] * cfg.T, dtype=torch.int32)
    w = bench.layer_work(cfg, ids)
    P = cfg.T * cfg.K
    assert w["n_experts"] == 4
    assert w["flops"] == 2 * P * cfg.H * 2 * cfg.I + 2 * P * cfg.I * cfg.H
    assert w["gemm1_flops"] == 2 * P * cfg.H * 2 * cfg.I
    w1 = 2 * cfg.I * cfg.H + (2 * cfg.I // 128) * (cfg.H // 128) * 4
    assert w["gemm1_bytes"] == (4 * w1 + cfg.T * cfg.H + cfg.T * (cfg.H // 128) * 4
                                + P * cfg.I + P * (cfg.I // 128) * 4)


@pytest.mark.parametrize("n", [1, 3])
def test_oracle_sample_step_is_repeatable(n):
    r = bench.OracleSample(I.TINY, n, device="cpu")
    assert r.step() > 0 and r.step() > 0
    assert len(r.experts) >= 1 and set(r.weights) == set(r.experts)


def test_reference_arm_gemm_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "gemm",
                        "--steps", "1", "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    d = _json_lines(r.stdout)[-1]
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["config"]["workload"] == I.GEMM.name


def test_layer_work_counts_only_kept_experts_under_a_mask():
    cfg = I.TINY
    ids = torch.tensor([[0, 1, 2, 3]] * cfg.T, dtype=torch.int32)
    mask = torch.tensor([1, 0, 1] + [0] * (cfg.E - 3), dtype=torch.int32)
    w = bench.layer_work(cfg, ids, mask)
    P = cfg.T * 2                                   # experts 0 and 2 only
    assert w["n_experts"] == 2
    assert w["flops"] == 2 * P * cfg.H * 2 * cfg.I + 2 * P * cfg.I * cfg.H


def test_expert_parallel_workload_mask_and_config():
    cfg = I.PREFILL_EP8
    m = I.expert_mask(cfg)
    assert m.dtype == torch.int32 and int(m.sum()) == cfg.E // 8 and bool(m[:32].all())
    assert I.expert_mask(I.PREFILL) is None and bench.ep_config(I.PREFILL) == {}
    assert "rank 0 of 8" in bench.ep_config(cfg)["expert_parallel"]


def test_tensor_parallel_workload_config_and_oracle_sample():
    assert "intermediate columns 0-255" in bench.ep_config(I.PREFILL_TP8)["tensor_parallel"]
    cfg = I.MoEConfig("host_tp2", T=8, H=256, E=4, G=2, TG=1, K=2, I=256, tp_ranks=2, tp_rank=1)
    r = bench.OracleSample(cfg, 2, device="cpu")
    assert r.step() > 0
    w1q, w1s, w2q, w2s = r.weights[r.experts[0]]
    assert w1q.shape == (256, 256) and w1s.shape == (2, 2) and w2q.shape == (256, 128) and w2s.shape == (2, 1)


def test_source_hash_ignores_comments_and_layout_only(tmp_path):
    code = "int f(int a) {\n  return a + 1;  // one more\n}\n/* block\n comment */\n"
    (tmp_path / "a.cu").write_text(code)
    (tmp_path / "b.cu").write_text("int f(int a){return a+1;}  // other words\n")
    (tmp_path / "c.cu").write_text("int f(int a){return a+2;}\n")
    h = [bench.source_sha([str(tmp_path / n)]) for n in ("a.cu", "b.cu", "c.cu")]
    assert h[0] == h[1] != h[2]


def test_tokens_option_keeps_the_recipe_at_another_batch_size():
    """--tokens T is a batch-size sweep point: the workload's recipe (shapes, routing, seed)
    at T tokens, named as such; the reference arm runs it too."""
    import argparse
    cfg = bench.workload_config(argparse.Namespace(workload="prefill", tokens=16))
    assert cfg.T == 16 and cfg.name == "prefill_t16_h7168_e256"
    assert (cfg.H, cfg.E, cfg.G, cfg.TG, cfg.K, cfg.I, cfg.seed) == (I.PREFILL.H, I.PREFILL.E, I.PREFILL.G,
                                                                    I.PREFILL.TG, I.PREFILL.K, I.PREFILL.I,
                                                                    I.PREFILL.seed)
    assert bench.workload_config(argparse.Namespace(workload="decode", tokens=None)) is I.DECODE
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--tokens", "3",
                        "--steps", "1", "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    (d,) = _json_lines(r.stdout)
    assert d["config"]["workload"] == "tiny_t3_h256_e16" and d["config"]["T"] == 3
    bad = subprocess.run([sys.executable, "bench.py", "--workload", "gemm", "--tokens", "3"], cwd=ROOT,
                         capture_output=True, text=True, timeout=600)
    assert bad.returncode != 0 and "--tokens" in bad.stderr


def test_tp_emulate_option_is_checked():
    """--tp-emulate runs the tensor-parallel workload's ranks on one GPU; it takes 2..8 ranks
    that split I into whole 128-column blocks, and only the prefill_tp workload."""
    for bad in (["--workload", "prefill", "--tp-emulate", "8"], ["--workload", "prefill_tp", "--tp-emulate", "9"],
                ["--workload", "prefill_tp", "--tp-emulate", "1"], ["--workload", "prefill_tp", "--tp-emulate", "3"]):
        r = subprocess.run([sys.executable, "bench.py", *bad], cwd=ROOT, capture_output=True, text=True, timeout=600)
        assert r.returncode != 0 and "--tp-emulate" in r.stderr, bad


def test_ep_emulate_option_is_checked():
    for bad in (["--workload", "prefill", "--ep-emulate", "8"], ["--workload", "prefill_ep", "--ep-emulate", "9"],
                ["--workload", "prefill_ep", "--ep-emulate", "3"]):
        r = subprocess.run([sys.executable, "bench.py", *bad], cwd=ROOT, capture_output=True, text=True, timeout=600)
        assert r.returncode != 0 and "--ep-emulate" in r.stderr, bad


def test_mla_work_counts_by_hand():
    """MLA decode's algorithmic bytes: KV rows once, q, o, lse and the page table."""
    nbytes, flops = bench.mla_work(I.MLA_DECODE)
    rows = 64 * 544
    assert nbytes == rows * 1152 + 64 * 16 * (1152 + 1024 + 4) + rows * 4 + (2 * 64 + 1) * 4 == 42_480_132
    assert flops == 2 * rows * 16 * (576 + 512)
    cfg = I.MlaConfig("t", B=3, Hq=32, L=(0, 5, 17), page_size=4)
    nbytes, _ = bench.mla_work(cfg)
    assert nbytes == 22 * 1152 + 3 * 32 * 2180 + (0 + 2 + 5) * 4 + 7 * 4


def test_reference_arm_mla_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "mla_decode",
                        "--steps", "2", "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "sequences/s" and line["value"] > 0
    assert line["config"]["workload"] == I.MLA_DECODE.name
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
