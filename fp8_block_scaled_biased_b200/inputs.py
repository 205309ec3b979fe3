"""Seeded synthetic inputs for the FP8 block-scaled MoE layer and the block-scale GEMM.

This module only draws random numbers. It holds none of the method's arithmetic:
no routing, no quantisation, no GEMM. Both the CUDA path (through the binding)
and the CPU oracle consume what it produces, so the two sides see the same raw
numbers and derive everything else on their own.

Workloads (DeepSeek-V3-shaped, as in "Accelerate DeepSeek-R1 Inference:
Integrate AITER into SGLang", section "Complete MoE Implementation"):

  tiny      T=16,    H=256,  E=16,  G=4, TG=2, K=4, I=128
  decode    T=64,    H=7168, E=256, G=8, TG=4, K=8, I=2048
  prefill   T=4096,  same layer as decode
  skewed    T=16384, same layer, correction bias +3.0 on 16 random experts
  gemm      M=2048, N=4096, K=7168 (single-expert block-scale GEMM)

Draw order for a MoE workload, from one CPU generator seeded with `seed`:
router logits ~N(0,1) fp32 [T,E], correction bias ~N(0,0.1) fp32 [E], hidden
states ~N(0,1) rounded to bf16 [T,H], then (skewed only) the 16 hot experts by
a random permutation. Expert weights ~N(0,0.02) are drawn per expert and per
matrix from their own generator, seeded from (seed, matrix, expert), on the
device the caller asks for; a given device always yields the same numbers, so
any single expert's raw weights can be drawn again later.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    H: int
    E: int
    G: int
    TG: int
    K: int
    I: int
    renorm: bool = True
    scale: float = 2.5
    hot_experts: int = 0        # experts that get +hot_bias on the correction bias
    hot_bias: float = 3.0
    logit_std: float = 1.0
    bias_std: float = 0.1
    x_std: float = 1.0
    w_std: float = 0.02
    seed: int = 0
    ep_ranks: int = 0           # > 0: the layer as expert-parallel rank ep_rank of ep_ranks sees it
    ep_rank: int = 0
    tp_ranks: int = 0           # > 0: tensor-parallel shard tp_rank of tp_ranks (over I)
    tp_rank: int = 0

    @property
    def P(self) -> int:
        return self.T * self.K


def expert_mask(cfg: MoEConfig):
    """int32 [E] on the CPU: the experts rank ep_rank holds when E experts are split into
    ep_ranks contiguous ranges (None when the config is not expert-parallel)."""
    if cfg.ep_ranks <= 0:
        return None
    per = cfg.E // cfg.ep_ranks
    return (torch.arange(cfg.E) // per == cfg.ep_rank).to(torch.int32)


@dataclass(frozen=True)
class GemmConfig:
    name: str
    M: int
    N: int
    K: int
    a_std: float = 1.0
    b_std: float = 0.02
    seed: int = 0


TINY = MoEConfig("tiny_t16_h256_e16", T=16, H=256, E=16, G=4, TG=2, K=4, I=128)
DECODE = MoEConfig("decode_t64_h7168_e256", T=64, H=7168, E=256, G=8, TG=4, K=8, I=2048)
PREFILL = MoEConfig("prefill_t4096_h7168_e256", T=4096, H=7168, E=256, G=8, TG=4, K=8, I=2048)
SKEWED = MoEConfig("skewed_t16384_h7168_e256", T=16384, H=7168, E=256, G=8, TG=4, K=8, I=2048,
                   hot_experts=16)
GEMM = GemmConfig("gemm_m2048_n4096_k7168", M=2048, N=4096, K=7168)

# The decode/prefill layer shape with 32 experts (1.4 GB of weights, more than
# L2) and 512 tokens: small enough for full-set profiler captures.
PROFILE = MoEConfig("profile_t512_h7168_e32", T=512, H=7168, E=32, G=8, TG=4, K=8, I=2048)

# The prefill batch as expert-parallel rank 0 of 8 computes it: experts 0-31 only
# (the expert_mask of the page's asm_moe call), a partial output for all 4096 tokens.
PREFILL_EP8 = MoEConfig("prefill_ep8_rank0_t4096_h7168_e256", T=4096, H=7168, E=256, G=8, TG=4, K=8, I=2048,
                        ep_ranks=8, ep_rank=0)

# The prefill batch on tensor-parallel rank 0 of 8 (the pages' TP8 run): every expert's
# intermediate columns 0-255, a partial output for all 4096 tokens.
PREFILL_TP8 = MoEConfig("prefill_tp8_rank0_t4096_h7168_e256", T=4096, H=7168, E=256, G=8, TG=4, K=8, I=2048,
                        tp_ranks=8, tp_rank=0)

MOE_CONFIGS = {c.name: c for c in (TINY, DECODE, PREFILL, SKEWED, PROFILE, PREFILL_EP8, PREFILL_TP8)}


@dataclass
class MoEActivations:
    logits: torch.Tensor      # fp32 [T, E]
    bias: torch.Tensor        # fp32 [E]
    x: torch.Tensor           # bf16 [T, H]
    hot: torch.Tensor = field(default_factory=lambda: torch.empty(0, dtype=torch.int64))


def moe_activations(cfg: MoEConfig) -> MoEActivations:
    """Router logits, correction bias and hidden states on the CPU, in the stated draw order."""
    g = torch.Generator(device="cpu").manual_seed(cfg.seed)
    logits = torch.randn(cfg.T, cfg.E, generator=g, dtype=torch.float32) * cfg.logit_std
    bias = torch.randn(cfg.E, generator=g, dtype=torch.float32) * cfg.bias_std
    x = (torch.randn(cfg.T, cfg.H, generator=g, dtype=torch.float32) * cfg.x_std).to(torch.bfloat16)
    hot = torch.empty(0, dtype=torch.int64)
    if cfg.hot_experts:
        hot = torch.randperm(cfg.E, generator=g)[: cfg.hot_experts]
        bias[hot] += cfg.hot_bias
    return MoEActivations(logits=logits.contiguous(), bias=bias.contiguous(), x=x.contiguous(), hot=hot)


_MATRIX_TAG = {"w1": 1, "w2": 2}


def _expert_seed(seed: int, which: str, e: int) -> int:
    return (seed * 1_000_003 + _MATRIX_TAG[which] * 65_537 + e) & 0x7FFF_FFFF_FFFF


def expert_weight_raw(cfg: MoEConfig, which: str, e: int, device="cpu") -> torch.Tensor:
    """Raw fp32 weights of one expert: w1 [2I, H] (gate rows first, then up) or w2 [H, I]."""
    rows, cols = (2 * cfg.I, cfg.H) if which == "w1" else (cfg.H, cfg.I)
    g = torch.Generator(device=device).manual_seed(_expert_seed(cfg.seed, which, e))
    return torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * cfg.w_std


def gemm_inputs(cfg: GemmConfig, device="cpu"):
    """A bf16 [M,K] ~N(0,a_std) and B fp32 [N,K] ~N(0,b_std), from one generator on `device`."""
    g = torch.Generator(device=device).manual_seed(cfg.seed)
    a = (torch.randn(cfg.M, cfg.K, generator=g, device=device) * cfg.a_std).to(torch.bfloat16)
    b = torch.randn(cfg.N, cfg.K, generator=g, device=device) * cfg.b_std
    return a, b


# ---------------------------------------------------------------------------
# MLA decode (section "Attention Mechanisms", "MLA For Decode")
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class MlaConfig:
    """A decode batch of multi-head latent attention over a paged KV buffer.

    L is the number of cached tokens of every sequence (an int) or of each one (a
    tuple of B ints, 0 allowed)."""
    name: str
    B: int
    Hq: int
    L: int | tuple
    page_size: int = 1
    Dk: int = 576
    Dv: int = 512
    q_std: float = 1.0
    kv_std: float = 1.0
    seed: int = 0

    def lengths(self) -> list[int]:
        return [self.L] * self.B if isinstance(self.L, int) else list(self.L)


# The pages' decode benchmark (bench_one_batch: batch 64, 512 input tokens, 32 output
# tokens, --tp 8): DeepSeek-R1's 128 query heads split over 8 GPUs, SGLang's page
# size of 1, and the KV length of the last decode step.
MLA_DECODE = MlaConfig("mla_decode_b64_h16_l544", B=64, Hq=16, L=544)
# The same batch with an 8K context: 604 MB of KV, more than L2.
MLA_LONG = MlaConfig("mla_decode_b64_h16_l8192", B=64, Hq=16, L=8192)
MLA_CONFIGS = {c.name: c for c in (MLA_DECODE, MLA_LONG)}


@dataclass
class MlaInputs:
    q: torch.Tensor                  # bf16 [B, Hq, Dk]
    kv_buffer: torch.Tensor          # bf16 [pages, page_size, 1, Dk]
    kv_indptr: torch.Tensor          # int32 [B + 1]
    kv_indices: torch.Tensor         # int32 [kv_indptr[B]]
    kv_last_page_lens: torch.Tensor  # int32 [B]


def mla_inputs(cfg: MlaConfig, device="cpu", spare_pages: int = 0) -> MlaInputs:
    """Seeded inputs on `device`: q ~N(0, q_std) and every KV entry ~N(0, kv_std), rounded to
    bf16, drawn in that order from one generator; then the page table, which hands the
    sequences' pages out in a random order (a permutation drawn from a CPU generator with
    the same seed), as a paged allocator would after some churn. `spare_pages` pages that
    no sequence lists are added to the buffer. A sequence of L tokens holds ceil(L /
    page_size) pages, its last one holding the rest (a full page when L is a multiple)."""
    lens = cfg.lengths()
    assert len(lens) == cfg.B
    pages_of = [(n + cfg.page_size - 1) // cfg.page_size for n in lens]
    n_pages = sum(pages_of) + spare_pages
    g = torch.Generator(device=device).manual_seed(cfg.seed)
    q = (torch.randn(cfg.B, cfg.Hq, cfg.Dk, generator=g, device=device) * cfg.q_std).to(torch.bfloat16)
    kv = (torch.randn(max(n_pages, 1), cfg.page_size, 1, cfg.Dk, generator=g, device=device)
          * cfg.kv_std).to(torch.bfloat16)
    gc = torch.Generator(device="cpu").manual_seed(cfg.seed + 1)
    perm = torch.randperm(max(n_pages, 1), generator=gc)[: sum(pages_of)].to(torch.int32)
    indptr = torch.zeros(cfg.B + 1, dtype=torch.int32)
    indptr[1:] = torch.cumsum(torch.tensor(pages_of, dtype=torch.int64), 0).to(torch.int32)
    last = torch.tensor([(n - (p - 1) * cfg.page_size) if p else 0 for n, p in zip(lens, pages_of)],
                        dtype=torch.int32)
    return MlaInputs(q=q.contiguous(), kv_buffer=kv.contiguous(), kv_indptr=indptr.to(device),
                     kv_indices=perm.to(device), kv_last_page_lens=last.to(device))
