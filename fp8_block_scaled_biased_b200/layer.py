"""The FP8 block-scaled MoE layer as one object: weights resident on the device,
buffers preallocated, forward = route -> align/sort (and, on a side stream at the same
time, 1x128 quant) -> fused g1u1 MoE.

This mirrors the composition the pages' asm_moe wrapper performs ("Accelerate
DeepSeek-R1 Inference: Integrate AITER into SGLang", section "Blockscale FP8
MoE Computation"): sorting, activation quantisation with transposed scales,
then fmoe_fp8_blockscale_g1u1. Every step is a call into the CUDA library.
"""
from __future__ import annotations

import dataclasses

import torch

from . import binding as B
from . import inputs as I


class MoELayer:
    def __init__(self, cfg: I.MoEConfig, device="cuda", max_tokens: int | None = None, weights_from=None,
                 tiled: bool = True):
        """weights_from: another MoELayer of the same layer shape whose device weights (and
        layout) are shared. tiled: keep w1 and w2 in the tiled layout of fp8_tile_weights
        ([E, N/128, K/128, 128, 128], every 128 x 128 block 16 KB of consecutive bytes), which
        the GEMMs read with one contiguous load per block; False keeps them row-major
        ([E, 2I, H], [E, H, I]), the layout the pages' fused call takes."""
        self.cfg = cfg
        self.device = torch.device(device)
        self.max_tokens = max_tokens or cfg.T
        E, H, Im = cfg.E, cfg.H, cfg.I
        dev = self.device
        if weights_from is not None:
            o = weights_from
            if (o.cfg.E, o.cfg.H, o.cfg.I) != (E, H, Im):
                raise ValueError("weights_from has a different layer shape")
            self.tiled = o.tiled
            self.w1, self.w1_scale, self.w2, self.w2_scale = o.w1, o.w1_scale, o.w2, o.w2_scale
        else:
            self.tiled = tiled
            if tiled:
                self.w1 = torch.empty(E, 2 * Im // 128, H // 128, 128, 128, dtype=B.FP8, device=dev)
                self.w2 = torch.empty(E, H // 128, Im // 128, 128, 128, dtype=B.FP8, device=dev)
            else:
                self.w1 = torch.empty(E, 2 * Im, H, dtype=B.FP8, device=dev)
                self.w2 = torch.empty(E, H, Im, dtype=B.FP8, device=dev)
            self.w1_scale = torch.empty(E, 2 * Im // 128, H // 128, dtype=torch.float32, device=dev)
            self.w2_scale = torch.empty(E, H // 128, Im // 128, dtype=torch.float32, device=dev)
        self.block_m = B.moe_block_m()
        self._alloc(self.max_tokens)
        # The activation quantisation depends only on x, so it runs on a side stream
        # while routing and sorting run on the caller's stream.
        self._side = torch.cuda.Stream(device=dev) if dev.type == "cuda" else None
        self._fork = torch.cuda.Event() if dev.type == "cuda" else None
        self._join = torch.cuda.Event() if dev.type == "cuda" else None

    def _alloc(self, T):
        cfg, dev = self.cfg, self.device
        self.topk_w = torch.empty(T, cfg.K, dtype=torch.float32, device=dev)
        self.topk_ids = torch.empty(T, cfg.K, dtype=torch.int32, device=dev)
        self.sorted = B.alloc_sorted(T, cfg.K, cfg.E, self.block_m, dev)
        self.sort_workspace = torch.empty(B.moe_align_sort_workspace_bytes(T, cfg.K, cfg.E, self.block_m),
                                          dtype=torch.uint8, device=dev)
        self.a8 = torch.empty(T, cfg.H, dtype=B.FP8, device=dev)
        self.a8_scale = torch.empty(cfg.H // 128, T, dtype=torch.float32, device=dev)
        self.out = torch.empty(T, cfg.H, dtype=torch.bfloat16, device=dev)
        ws = B.fused_moe_workspace_bytes(T, cfg.K, cfg.E, cfg.H, cfg.I, self.block_m)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev)

    def load_synthetic_weights(self, expert_offset: int = 0):
        """Draw each expert's raw fp32 weights on the device, quantise them in 128x128 blocks
        and, for a tiled layer, re-pack them (fp8_tile_weights). Slot i holds global expert
        expert_offset + i (an expert-parallel rank's experts start past 0)."""
        cfg = self.cfg
        stage1 = stage2 = None
        if self.tiled:
            stage1 = torch.empty(2 * cfg.I, cfg.H, dtype=B.FP8, device=self.device)
            stage2 = torch.empty(cfg.H, cfg.I, dtype=B.FP8, device=self.device)
        for i in range(self.w1.shape[0]):
            e = expert_offset + i
            raw1 = I.expert_weight_raw(cfg, "w1", e, self.device)
            B.fp8_per_block_quant(raw1, q=stage1 if self.tiled else self.w1[i], scales=self.w1_scale[i])
            raw2 = I.expert_weight_raw(cfg, "w2", e, self.device)
            B.fp8_per_block_quant(raw2, q=stage2 if self.tiled else self.w2[i], scales=self.w2_scale[i])
            if self.tiled:
                B.fp8_tile_weights(stage1, out=self.w1[i])
                B.fp8_tile_weights(stage2, out=self.w2[i])
        return self

    def tp_shard(self, rank: int, nranks: int) -> "MoELayer":
        """Tensor-parallel shard `rank` of `nranks` (the pages' TP8 deployment): every expert's
        intermediate columns [rank*I/n, (rank+1)*I/n), i.e. those gate and up rows of w1 and
        those columns of w2, with their 128x128 block scales, copied into a new layer. Its
        forward gives that rank's partial output; the ranks' partial outputs sum to the whole
        layer's, because the 1x128 requantisation groups of the intermediate lie inside a
        shard (I/n must be a multiple of 128). Routing and the activation quantisation are
        the same on every rank."""
        cfg = self.cfg
        if nranks < 1 or not 0 <= rank < nranks or cfg.I % (128 * nranks):
            raise ValueError(f"I={cfg.I} cannot be split into {nranks} shards of whole 128-column blocks")
        Is, I0 = cfg.I // nranks, rank * (cfg.I // nranks)
        nb, b0, nbI = Is // 128, I0 // 128, cfg.I // 128
        scfg = dataclasses.replace(cfg, name=f"{cfg.name}_tp{nranks}_rank{rank}", I=Is, tp_ranks=nranks, tp_rank=rank)
        shard = MoELayer(scfg, self.device, max_tokens=self.max_tokens, tiled=self.tiled)
        if self.tiled:                   # whole 128-blocks: gate/up row blocks of w1, K blocks of w2
            shard.w1[:, :nb].copy_(self.w1[:, b0:b0 + nb])
            shard.w1[:, nb:].copy_(self.w1[:, nbI + b0:nbI + b0 + nb])
            shard.w2.copy_(self.w2[:, :, b0:b0 + nb])
        else:
            shard.w1[:, :Is].copy_(self.w1[:, I0:I0 + Is])
            shard.w1[:, Is:].copy_(self.w1[:, cfg.I + I0:cfg.I + I0 + Is])
            shard.w2.copy_(self.w2[:, :, I0:I0 + Is])
        shard.w1_scale[:, :nb].copy_(self.w1_scale[:, b0:b0 + nb])
        shard.w1_scale[:, nb:].copy_(self.w1_scale[:, nbI + b0:nbI + b0 + nb])
        shard.w2_scale.copy_(self.w2_scale[:, :, b0:b0 + nb])
        return shard

    def forward(self, logits, bias, x, expert_mask=None):
        """logits fp32 or bf16 [T, E], bias fp32 [E], x bf16 [T, H] (all on the device) -> bf16 [T, H].

        expert_mask: optional int32 [E] on the device (nonzero = an expert this GPU holds).
        The result is then the sum over the kept experts' pairs only, the partial output
        of one expert-parallel rank."""
        self._route_sort_quant(logits, bias, x, expert_mask)
        B.fused_moe_fp8_blockscale_g1u1(self.out, self.a8, self.w1, self.w2, self.sorted, self.cfg.K, self.a8_scale,
                                        self.w1_scale, self.w2_scale, workspace=self.workspace)
        return self.out

    def forward_pairs(self, logits, bias, x):
        """forward() without the combine: routing, sorting, quantisation and
        fused_moe_fp8_blockscale_g1u1_pairs. The weighted pair rows and the pair flags are
        left in self.workspace, where moe_combine_allreduce (a tensor-parallel rank's
        combine fused with the all-reduce) reads them; returns that workspace."""
        self._route_sort_quant(logits, bias, x, None)
        return B.fused_moe_fp8_blockscale_g1u1_pairs(self.a8, self.w1, self.w2, self.sorted, self.cfg.K,
                                                      self.a8_scale, self.w1_scale, self.w2_scale,
                                                      workspace=self.workspace)

    def _route_sort_quant(self, logits, bias, x, expert_mask):
        cfg = self.cfg
        T = x.shape[0]
        if T != self.max_tokens:
            raise ValueError(f"layer buffers are sized for {self.max_tokens} tokens, got {T}")
        main = torch.cuda.current_stream(self.device)
        self._fork.record(main)
        self._side.wait_event(self._fork)
        with torch.cuda.stream(self._side):
            B.fp8_per_token_group_quant(x, 128, column_major_scales=True, q=self.a8, scales=self.a8_scale)
            self._join.record(self._side)
        B.moe_biased_grouped_topk(logits, bias, self.topk_w, self.topk_ids, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
        B.moe_align_sort(self.topk_ids, self.topk_w, cfg.E, self.block_m, out=self.sorted,
                         workspace=self.sort_workspace, expert_mask=expert_mask)
        main.wait_event(self._join)

    @property
    def launches_per_forward(self):
        """Kernels one forward launches: route, sort (count and scatter; one kernel when the
        T*topk pairs fit one 1024-pair chunk), quant, gather (slot pass and row pass), gate/up
        GEMM, down GEMM, combine."""
        sort_kernels = 1 if self.max_tokens * self.cfg.K <= 1024 else 2
        return 7 + sort_kernels
