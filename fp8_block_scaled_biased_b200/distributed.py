"""Multi-GPU forms of the FP8 block-scaled MoE layer, one process per GPU over
torch.distributed (between GPUs NCCL, or the library's kernels on peer memory from
torch's symmetric memory; gloo for the rank logic on the CPU).

"Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang" runs the layer at
TP8 (section "Performance Reproduction for AITER-Optimized in SGLang", --tp 8),
summing the ranks' outputs with the custom all-reduce of section "Other
Operators", and gives asm_moe an expert_mask (section "Blockscale FP8 MoE
Computation"), the hook of expert parallelism. Both are built here:

Tensor parallelism over I (TensorParallelMoE). Every rank routes every token and
runs its shard of each expert's intermediate columns (MoELayer.tp_shard). The
ranks' partial outputs are summed either by the library's combine fused with the
all-reduce over peer memory (reduce="peer": each rank combines its pair rows per
token and stores the bf16 partial straight into the receive buffer of the rank that
owns the token's slice, over NVLink; the owners sum in rank order and store the
result into every rank's output; TpPeerAllReduce holds the buffers, in torch's
symmetric memory), or by tp_reduce (reduce="nccl": an fp32 reduce-scatter over
NCCL, each rank summing one slice of the tokens, and a bf16 all-gather). Both sum
the same bf16 partials in fp32 and round once; the peer form fixes the order (rank
order) and saves the combine's separate pass over the partial output.

Expert parallelism over E (ExpertParallelMoE). Rank r holds experts
[r*E/n, (r+1)*E/n) and its own batch of tokens. It routes and quantises its
tokens, then one all-to-all sends every (token, owner rank) pair that has work
there: the token's FP8 row, its 1x128 scales, and its top-k ids (as the owner's
local ids; pairs of other ranks carry a sentinel id that the owner's sort drops)
and weights, packed in one byte row. The owner sorts what it received with an
expert mask and runs the fused MoE on its experts; a second all-to-all returns
each received row's partial output (the bf16 sum over that rank's pairs), and the
origin adds, per token, the partial rows in ascending rank order in fp32 and
rounds to bf16 once. The result is deterministic for a given rank count.

Expert parallelism over peer memory (ExpertParallelPeerMoE). The same split with
no all-to-all: every rank publishes its routing, activations and a return buffer
in symmetric memory; each owner reads every rank's routing (moe_ep_routing),
sorts the pairs of its experts over all ranks' tokens, gathers their activation
rows where they lie inside its fused call (fused_moe_fp8_blockscale_g1u1_multi)
and stores each pair's weighted row into its origin's return buffer
(moe_ep_return); two flag barriers (moe_ep_barrier) order the steps. Each rank
then combines its own tokens' rows exactly as one GPU does, so the output is the
one-GPU layer's bit for bit. EmulatedExpertParallel runs all ranks on one GPU.

The compute is the library's kernels (routing, quantisation, sort, fused MoE,
and for the peer forms the exchange itself); the NCCL forms' collectives are
NCCL's, with index bookkeeping and byte packing on the device (torch indexing)
between them and the local compute passed in as a callable, so that their rank
logic runs unchanged on the CPU with the oracle in its place.
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist

from . import binding as B
from . import inputs as I


def _world(group):
    return dist.get_world_size(group) if dist.is_initialized() else 1


def _rank(group):
    return dist.get_rank(group) if dist.is_initialized() else 0


# ---------------------------------------------------------------------------------- tensor parallel

def tp_reduce(partial: torch.Tensor, group=None) -> torch.Tensor:
    """Sum over the group's ranks of each rank's partial output [T, H] (bf16), returned
    on every rank as bf16 [T, H]: the tokens are split into one slice per rank, each slice
    summed over the ranks in fp32 (reduce-scatter) and rounded to bf16 once, then the
    slices gathered (all-gather). With one rank the partial is the output."""
    n = _world(group)
    if n == 1:
        return partial
    T, H = partial.shape
    Tp = -(-T // n) * n
    full = torch.zeros(Tp, H, dtype=torch.float32, device=partial.device)
    full[:T].copy_(partial)
    piece = torch.empty(Tp // n, H, dtype=torch.float32, device=partial.device)
    dist.reduce_scatter_tensor(piece, full, op=dist.ReduceOp.SUM, group=group)
    out = torch.empty(Tp, H, dtype=torch.bfloat16, device=partial.device)
    dist.all_gather_into_tensor(out, piece.to(torch.bfloat16), group=group)
    return out[:T]


@dataclasses.dataclass(frozen=True)
class TpBufferLayout:
    """Byte offsets of one rank's buffers for moe_combine_allreduce inside one allocation:
    the receive buffer bf16 [n][ceil(T/n)][H], the output bf16 [T][H] and the flag words
    (each part starting at a multiple of 256 bytes)."""
    recv: int
    out: int
    flags: int
    total: int


def tp_buffer_layout(T: int, H: int, n: int) -> TpBufferLayout:
    if not 1 <= n <= B.TP_MAX_RANKS or T < 1 or H < 1:
        raise ValueError(f"bad tensor-parallel buffer shape T={T}, H={H}, n={n}")
    up = lambda v: -(-v // 256) * 256   # noqa: E731
    Ts = -(-T // n)
    recv = 0
    out = up(n * Ts * H * 2)
    flags = out + up(T * H * 2)
    return TpBufferLayout(recv, out, flags, flags + up(B.TP_FLAG_WORDS * 8))


class TpPeerAllReduce:
    """One rank's buffers for the combine fused with the all-reduce (moe_combine_allreduce):
    the receive buffer, the output and the flag words in one allocation of torch's symmetric
    memory, exchanged over the group so that every rank's buffers are addressable from every
    GPU (over NVLink); the CTA barrier words (which also count the calls) in this GPU's
    memory. Every rank of the group must construct it and then make the same calls; nothing
    is passed from the host per call, so a forward holding it can be captured in a CUDA
    graph."""

    def __init__(self, T: int, H: int, group=None, device=None):
        import torch.distributed._symmetric_memory as symm
        n, r = _world(group), _rank(group)
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.T, self.H, self.n, self.rank = T, H, n, r
        self.layout = L = tp_buffer_layout(T, H, n)
        self.buf = symm.empty(L.total, dtype=torch.uint8, device=dev)
        self.buf.zero_()
        handle = symm.rendezvous(self.buf, group if group is not None else dist.group.WORLD)
        bases = [int(b) for b in handle.buffer_ptrs]
        self._handle = handle
        self.recv = [b + L.recv for b in bases]
        self.outs = [b + L.out for b in bases]
        self.flags = [b + L.flags for b in bases]
        self.out = self.buf[L.out:L.out + T * H * 2].view(torch.bfloat16).view(T, H)
        self.barrier = torch.zeros(B.TP_BARRIER_WORDS, dtype=torch.int64, device=dev)
        torch.cuda.synchronize(dev)
        if dist.is_initialized() and n > 1:
            dist.barrier(group)            # every rank's flags are zero before any rank's first call

    def __call__(self, workspace, capacity: int, topk: int, I: int) -> torch.Tensor:
        """Combine this rank's pair rows (left in `workspace` by the pairs call) and all-reduce
        them; returns this rank's output buffer bf16 [T, H] (rewritten by the next call)."""
        B.moe_combine_allreduce(workspace, capacity, self.T, topk, self.H, I, self.rank, self.recv, self.outs,
                                self.flags, self.barrier)
        return self.out

    @property
    def calls(self) -> int:
        """Calls made so far (the device-side counter; reading it synchronises)."""
        return int(self.barrier[2])


class EmulatedTpAllReduce:
    """Every rank of the fused combine + all-reduce on one GPU: each rank's receive buffer,
    output, flags and barrier words in this GPU's memory, all ranks run by one cooperative
    launch (moe_combine_allreduce_emulated) through the same per-rank code and flags as the
    multi-GPU form."""

    def __init__(self, T: int, H: int, n: int, device="cuda"):
        tp_buffer_layout(T, H, n)
        Ts = -(-T // n)
        self.T, self.H, self.n = T, H, n
        self.recv = [torch.empty(n, Ts, H, dtype=torch.bfloat16, device=device) for _ in range(n)]
        self.out = [torch.empty(T, H, dtype=torch.bfloat16, device=device) for _ in range(n)]
        self.flags = [torch.zeros(B.TP_FLAG_WORDS, dtype=torch.int64, device=device) for _ in range(n)]
        self.barriers = [torch.zeros(B.TP_BARRIER_WORDS, dtype=torch.int64, device=device) for _ in range(n)]

    def __call__(self, workspaces, capacity: int, topk: int, I: int):
        """workspaces[r]: rank r's pairs-call workspace. Returns the n ranks' outputs."""
        B.moe_combine_allreduce_emulated(workspaces, capacity, self.T, topk, self.H, I, self.recv, self.out,
                                         self.flags, self.barriers)
        return self.out

    @property
    def calls(self) -> int:
        """Calls made so far, by every rank's device-side counter (which must agree)."""
        counts = {int(b[2]) for b in self.barriers}
        if len(counts) != 1:
            raise RuntimeError(f"the ranks' call counters disagree: {sorted(counts)}")
        return counts.pop()


class TensorParallelMoE:
    """One rank of the layer split over I: its shard (rank, n) of every expert, the whole
    routing, and the sum of the ranks' partial outputs: reduce="peer" (the combine fused
    with the all-reduce over peer memory, TpPeerAllReduce) or reduce="nccl" (tp_reduce)."""

    def __init__(self, layer, group=None, reduce: str = "nccl"):
        """layer: the whole MoELayer (its shard is copied out) or an already-sharded one
        whose cfg.tp_ranks / tp_rank match the group."""
        if reduce not in ("peer", "nccl"):
            raise ValueError("reduce must be 'peer' or 'nccl'")
        self.group, self.reduce = group, reduce
        n, r = _world(group), _rank(group)
        if layer.cfg.tp_ranks == n and layer.cfg.tp_rank == r:
            self.shard = layer
        else:
            self.shard = layer.tp_shard(r, n) if n > 1 else layer
        self.peer = None

    def forward(self, logits, bias, x):
        if self.reduce == "nccl":
            partial = self.shard.forward(logits, bias, x)
            return tp_reduce(partial, self.group)
        sh = self.shard
        if self.peer is None:
            self.peer = TpPeerAllReduce(x.shape[0], sh.cfg.H, self.group, x.device)
        ws = sh.forward_pairs(logits, bias, x)
        return self.peer(ws, sh.sorted.capacity, sh.cfg.K, sh.cfg.I)


# ---------------------------------------------------------------------------------- expert parallel

def ep_expert_range(E: int, rank: int, n: int):
    """Experts [e0, e1) that rank `rank` of `n` holds (contiguous ranges; E % n == 0)."""
    if n < 1 or E % n:
        raise ValueError(f"E={E} experts cannot be split evenly over {n} ranks")
    per = E // n
    return rank * per, (rank + 1) * per


@dataclasses.dataclass
class EpPlan:
    """Where a rank's tokens went: for each destination rank d, the tokens (ascending)
    that have at least one pair on d's experts, in the order their rows were sent."""
    tokens: list          # per destination: int64 [n_d] token indices
    send_counts: list     # per destination: n_d
    recv_counts: list     # per source: rows received from it
    T: int
    H: int


def _row_bytes(H, K):
    return H + 4 * (H // 128) + 4 * K + 4 * K


def ep_dispatch(a8, a8_scale, topk_ids, topk_weights, E, group=None):
    """Sends each (token, owner rank) pair with work to the owner. a8 fp8 [T, H],
    a8_scale fp32 [T, H/128] (row-major), topk_ids int32 [T, K], topk_weights fp32 [T, K].

    Returns (received, plan): received = (a8 fp8 [m, H], scales fp32 [m, H/128], local ids
    int32 [m, K], weights fp32 [m, K]) for the m rows this rank received, sources in rank
    order; a pair of another rank carries the local id E/n (one past this rank's experts)."""
    n, r = _world(group), _rank(group)
    T, H = a8.shape
    K = topk_ids.shape[1]
    per = E // n
    dev = a8.device
    owner = topk_ids.long() // per                                   # [T, K]
    has = torch.zeros(T, n, dtype=torch.bool, device=dev)
    has.scatter_(1, owner.clamp(0, n - 1), True)
    tokens = [torch.nonzero(has[:, d]).flatten() for d in range(n)]
    send_counts = [int(t.numel()) for t in tokens]
    idx = torch.cat(tokens) if tokens else torch.empty(0, dtype=torch.long, device=dev)
    dest = torch.repeat_interleave(torch.arange(n, device=dev), torch.tensor(send_counts, device=dev))
    ids = topk_ids[idx].long()
    local = torch.where(ids // per == dest[:, None], ids - dest[:, None] * per, torch.full_like(ids, per))
    rb = _row_bytes(H, K)
    send = torch.empty(idx.numel(), rb, dtype=torch.uint8, device=dev)
    o1, o2, o3 = H, H + 4 * (H // 128), H + 4 * (H // 128) + 4 * K
    send[:, :o1] = a8.view(torch.uint8)[idx]
    send[:, o1:o2] = a8_scale[idx].contiguous().view(torch.uint8)
    send[:, o2:o3] = local.to(torch.int32).contiguous().view(torch.uint8)
    send[:, o3:] = topk_weights[idx].contiguous().view(torch.uint8)
    counts = torch.tensor(send_counts, dtype=torch.int64, device=dev)
    recv_c = torch.empty_like(counts)
    if n > 1:
        dist.all_to_all_single(recv_c, counts, group=group)
    else:
        recv_c.copy_(counts)
    recv_counts = [int(c) for c in recv_c.tolist()]
    recv = torch.empty(sum(recv_counts), rb, dtype=torch.uint8, device=dev)
    if n > 1:
        dist.all_to_all_single(recv, send, recv_counts, send_counts, group=group)
    else:
        recv.copy_(send)
    m = recv.shape[0]
    r_a8 = recv[:, :o1].contiguous().view(a8.dtype)
    r_sc = recv[:, o1:o2].contiguous().view(torch.float32).view(m, H // 128)
    r_ids = recv[:, o2:o3].contiguous().view(torch.int32).view(m, K)
    r_w = recv[:, o3:].contiguous().view(torch.float32).view(m, K)
    return (r_a8, r_sc, r_ids, r_w), EpPlan(tokens, send_counts, recv_counts, T, H)


def ep_combine(partials: torch.Tensor, plan: EpPlan, group=None) -> torch.Tensor:
    """Returns each received row's partial output (bf16 [m, H], rows in the order received)
    to its origin and sums, per token, the rows from all ranks in ascending rank order in
    fp32, rounded to bf16 once. A token with no pair anywhere gets a zero row."""
    n = _world(group)
    H = plan.H
    back = torch.empty(sum(plan.send_counts), H, dtype=partials.dtype, device=partials.device)
    if n > 1:
        dist.all_to_all_single(back, partials.contiguous(), plan.send_counts, plan.recv_counts, group=group)
    else:
        back.copy_(partials)
    acc = torch.zeros(plan.T, H, dtype=torch.float32, device=partials.device)
    off = 0
    for d in range(n):
        c = plan.send_counts[d]
        if c:
            # each token appears at most once per source rank: no two adds hit one row here
            acc.index_add_(0, plan.tokens[d], back[off:off + c].float())
        off += c
    return acc.to(torch.bfloat16)


class ExpertShard:
    """The experts [e0, e1) of a layer, as one expert-parallel rank holds them: w1 and w2
    (tiled as fp8_tile_weights writes them, or row-major [n_e, 2I, H], [n_e, H, I]) and
    their 128x128 block scales, on the device."""

    def __init__(self, cfg: I.MoEConfig, e0: int, e1: int, device="cuda", tiled: bool = True):
        self.cfg, self.e0, self.e1, self.tiled = cfg, e0, e1, tiled
        ne, H, Im = e1 - e0, cfg.H, cfg.I
        if tiled:
            self.w1 = torch.empty(ne, 2 * Im // 128, H // 128, 128, 128, dtype=B.FP8, device=device)
            self.w2 = torch.empty(ne, H // 128, Im // 128, 128, 128, dtype=B.FP8, device=device)
        else:
            self.w1 = torch.empty(ne, 2 * Im, H, dtype=B.FP8, device=device)
            self.w2 = torch.empty(ne, H, Im, dtype=B.FP8, device=device)
        self.w1_scale = torch.empty(ne, 2 * Im // 128, H // 128, dtype=torch.float32, device=device)
        self.w2_scale = torch.empty(ne, H // 128, Im // 128, dtype=torch.float32, device=device)
        self.block_m = B.moe_block_m()
        # sort over the rank's experts plus one sentinel expert (other ranks' pairs), masked out
        self.sort_mask = torch.ones(ne + 1, dtype=torch.int32, device=device)
        self.sort_mask[ne] = 0

    def load_synthetic_weights(self):
        """Draw and quantise the raw weights of global experts e0..e1-1 (as MoELayer does)."""
        dev = self.w1.device
        cfg = self.cfg
        stage1 = torch.empty(2 * cfg.I, cfg.H, dtype=B.FP8, device=dev) if self.tiled else None
        stage2 = torch.empty(cfg.H, cfg.I, dtype=B.FP8, device=dev) if self.tiled else None
        for i, e in enumerate(range(self.e0, self.e1)):
            B.fp8_per_block_quant(I.expert_weight_raw(cfg, "w1", e, dev), q=stage1 if self.tiled else self.w1[i],
                                  scales=self.w1_scale[i])
            B.fp8_per_block_quant(I.expert_weight_raw(cfg, "w2", e, dev), q=stage2 if self.tiled else self.w2[i],
                                  scales=self.w2_scale[i])
            if self.tiled:
                B.fp8_tile_weights(stage1, out=self.w1[i])
                B.fp8_tile_weights(stage2, out=self.w2[i])
        return self

    def __call__(self, a8, scales, ids, weights):
        """The fused MoE over received rows: a8 fp8 [m, H], scales fp32 [m, H/128], local ids
        int32 [m, K] (sentinel n_e = another rank's pair), weights fp32 [m, K] -> bf16 [m, H]."""
        m, H = a8.shape
        K = ids.shape[1]
        ne = self.e1 - self.e0
        out = torch.empty(m, H, dtype=torch.bfloat16, device=a8.device)
        if m == 0:
            return out
        sp = B.moe_align_sort(ids, weights, ne + 1, self.block_m, expert_mask=self.sort_mask)
        B.fused_moe_fp8_blockscale_g1u1(out, a8, self.w1, self.w2, sp, K, scales.t().contiguous(), self.w1_scale,
                                        self.w2_scale)
        return out


class ExpertParallelMoE:
    """One expert-parallel rank: its experts (an ExpertShard or any callable with its
    signature), the whole routing of its own tokens, and the dispatch/return all-to-alls."""

    def __init__(self, cfg: I.MoEConfig, local_experts, group=None):
        self.cfg, self.local, self.group = cfg, local_experts, group
        ep_expert_range(cfg.E, _rank(group), _world(group))

    def forward(self, logits, bias, x):
        cfg = self.cfg
        T = x.shape[0]
        w = torch.empty(T, cfg.K, dtype=torch.float32, device=x.device)
        ids = torch.empty(T, cfg.K, dtype=torch.int32, device=x.device)
        B.moe_biased_grouped_topk(logits, bias, w, ids, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
        a8, a8_scale = B.fp8_per_token_group_quant(x, 128, column_major_scales=False)
        received, plan = ep_dispatch(a8, a8_scale, ids, w, cfg.E, self.group)
        partial = self.local(*received)
        return ep_combine(partial, plan, self.group)


# ------------------------------------------------------------------ expert parallel over peer memory

@dataclasses.dataclass(frozen=True)
class EpBufferLayout:
    """Byte offsets of what one expert-parallel rank publishes to the others, in one
    allocation (each part at a multiple of 256 bytes): its routing (ids int32 [T, K],
    weights fp32 [T, K]), its activations (fp8 [T, H]) and their scales (fp32 [H/128, T]),
    its return buffer (bf16 rows [T*K, H], then a 16-byte count and one flag byte per pair)
    and its barrier words (int64 [EP_BARRIER_WORDS])."""
    ids: int
    w: int
    a8: int
    scale: int
    rows: int
    flags: int
    barrier: int
    total: int


def ep_buffer_layout(T: int, K: int, H: int) -> EpBufferLayout:
    if T < 1 or K < 1 or H < 128 or H % 128:
        raise ValueError(f"bad expert-parallel buffer shape T={T}, K={K}, H={H}")
    up = lambda v: -(-v // 256) * 256   # noqa: E731
    off, parts = 0, []
    for size in (T * K * 4, T * K * 4, T * H, (H // 128) * T * 4, T * K * H * 2, 16 + T * K, B.EP_BARRIER_WORDS * 8):
        parts.append(off)
        off = up(off + size)
    return EpBufferLayout(*parts, total=off)


class EpRankBuffers:
    """Typed views of one rank's published buffers (a uint8 tensor laid out by
    ep_buffer_layout) and their addresses."""

    def __init__(self, buf: torch.Tensor, T: int, K: int, H: int):
        L = ep_buffer_layout(T, K, H)
        self.layout, self.buf = L, buf
        self.ids = buf[L.ids:L.ids + T * K * 4].view(torch.int32).view(T, K)
        self.w = buf[L.w:L.w + T * K * 4].view(torch.float32).view(T, K)
        self.a8 = buf[L.a8:L.a8 + T * H].view(B.FP8).view(T, H)
        self.scale = buf[L.scale:L.scale + (H // 128) * T * 4].view(torch.float32).view(H // 128, T)
        self.rows = buf[L.rows:L.rows + T * K * H * 2].view(torch.bfloat16).view(T * K, H)
        self.flags = buf[L.flags:L.flags + 16 + T * K]
        self.barrier = buf[L.barrier:L.barrier + B.EP_BARRIER_WORDS * 8].view(torch.int64)

    @staticmethod
    def addresses(base: int, T: int, K: int, H: int) -> dict:
        L = ep_buffer_layout(T, K, H)
        return {name: base + getattr(L, name) for name in ("ids", "w", "a8", "scale", "rows", "flags", "barrier")}


class EpPeerRank:
    """One expert-parallel rank's steps over peer memory (include/fp8moe.h): publish its
    routing and activations, gather every rank's pairs of its own experts (routing read
    from the other ranks, activation rows pulled by the fused call's gather), return each
    pair's weighted row to its origin, and combine its own tokens' rows. `peers` maps each
    buffer name to the n ranks' addresses, as this GPU sees them."""

    def __init__(self, cfg: I.MoEConfig, shard: "ExpertShard", n: int, rank: int, T: int, mine: EpRankBuffers,
                 peers: dict, return_in_gemm: bool = True):
        """return_in_gemm: the down GEMM stores each pair's row into its origin's buffer (True),
        or the rows stay in the workspace and moe_ep_return copies them there (False)."""
        self.cfg, self.shard, self.n, self.rank, self.T, self.mine, self.peers = cfg, shard, n, rank, T, mine, peers
        dev = mine.buf.device
        self.return_in_gemm = return_in_gemm
        self.ret_rows = torch.tensor(peers["rows"], dtype=torch.int64, device=dev)
        self.ret_flags = torch.tensor([f + 16 for f in peers["flags"]], dtype=torch.int64, device=dev)
        K, ne = cfg.K, shard.e1 - shard.e0
        self.ids_g = torch.empty(n * T, K, dtype=torch.int32, device=dev)
        self.w_g = torch.empty(n * T, K, dtype=torch.float32, device=dev)
        self.sorted = B.alloc_sorted(n * T, K, ne + 1, shard.block_m, dev)
        self.sort_ws = torch.empty(B.moe_align_sort_workspace_bytes(n * T, K, ne + 1, shard.block_m),
                                   dtype=torch.uint8, device=dev)
        self.workspace = torch.empty(B.fused_moe_workspace_bytes(n * T, K, ne, cfg.H, cfg.I, shard.block_m,
                                                                 capacity=self.sorted.capacity),
                                     dtype=torch.uint8, device=dev)
        self.out = torch.empty(T, cfg.H, dtype=torch.bfloat16, device=dev)

    def publish(self, logits, bias, x):
        if x.shape[0] != self.T or logits.shape[0] != self.T:
            raise ValueError(f"this rank's buffers are sized for {self.T} tokens, got {x.shape[0]}")
        cfg, m = self.cfg, self.mine
        B.moe_biased_grouped_topk(logits, bias, m.w, m.ids, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
        B.fp8_per_token_group_quant(x, 128, column_major_scales=True, q=m.a8, scales=m.scale)
        m.flags.zero_()

    def compute(self):
        cfg, sh, p = self.cfg, self.shard, self.peers
        ne = sh.e1 - sh.e0
        B.moe_ep_routing(p["ids"], p["w"], self.T, cfg.K, cfg.E, sh.e0, ne, self.ids_g, self.w_g)
        B.moe_align_sort(self.ids_g, self.w_g, ne + 1, sh.block_m, out=self.sorted, workspace=self.sort_ws,
                         expert_mask=sh.sort_mask)
        if self.return_in_gemm:
            B.fused_moe_fp8_blockscale_g1u1_multi(p["a8"], p["scale"], self.T, cfg.H, sh.w1, sh.w2, self.sorted,
                                                  cfg.K, sh.w1_scale, sh.w2_scale, workspace=self.workspace,
                                                  return_rows=self.ret_rows, return_flags=self.ret_flags)
        else:
            B.fused_moe_fp8_blockscale_g1u1_multi(p["a8"], p["scale"], self.T, cfg.H, sh.w1, sh.w2, self.sorted,
                                                  cfg.K, sh.w1_scale, sh.w2_scale, workspace=self.workspace)
            B.moe_ep_return(self.workspace, self.sorted.capacity, self.T, cfg.K, cfg.H, cfg.I, self.sorted,
                            p["rows"], [f + 16 for f in p["flags"]])

    def combine(self):
        return B.moe_combine_pairs(self.mine.rows, self.mine.flags, self.T, self.cfg.K, self.out)


class ExpertParallelPeerMoE:
    """One expert-parallel rank over peer memory: its experts, its own batch of T tokens, the
    published buffers in torch's symmetric memory (rendezvoused over the group), and the
    forward publish -> barrier -> gather/compute/return -> barrier -> combine. The output is
    the one-GPU layer's for this rank's tokens, bit for bit."""

    def __init__(self, cfg: I.MoEConfig, shard: "ExpertShard", T: int, group=None):
        import torch.distributed._symmetric_memory as symm
        n, r = _world(group), _rank(group)
        ep_expert_range(cfg.E, r, n)
        dev = shard.w1.device
        L = ep_buffer_layout(T, cfg.K, cfg.H)
        self.buf = symm.empty(L.total, dtype=torch.uint8, device=dev)
        self.buf.zero_()
        handle = symm.rendezvous(self.buf, group if group is not None else dist.group.WORLD)
        self._handle = handle
        bases = [int(b) for b in handle.buffer_ptrs]
        addrs = [EpRankBuffers.addresses(b, T, cfg.K, cfg.H) for b in bases]
        peers = {k: [a[k] for a in addrs] for k in addrs[0]}
        self.rank = EpPeerRank(cfg, shard, n, r, T, EpRankBuffers(self.buf, T, cfg.K, cfg.H), peers)
        self.r = r
        torch.cuda.synchronize(dev)
        if dist.is_initialized() and n > 1:
            dist.barrier(group)            # every rank's barrier words are zero before the first forward

    def forward(self, logits, bias, x):
        """This rank's tokens -> its output bf16 [T, H] (a buffer the next forward rewrites)."""
        rk = self.rank
        rk.publish(logits, bias, x)
        B.moe_ep_barrier(self.r, rk.peers["barrier"])
        rk.compute()
        B.moe_ep_barrier(self.r, rk.peers["barrier"])
        return rk.combine()

    @property
    def barriers_passed(self) -> int:
        """Barrier calls made so far (this rank's device-side counter; reading synchronises)."""
        return int(self.rank.mine.barrier[B.EP_BARRIER_WORDS - 1])


class EmulatedExpertParallel:
    """All n expert-parallel ranks on one GPU, each with its own published buffers in this
    GPU's memory and its own experts; the steps run rank after rank on one stream and the
    two barriers as one launch over all ranks (moe_ep_barrier_emulated)."""

    def __init__(self, cfg: I.MoEConfig, shards, T: int, device="cuda", return_in_gemm: bool = True):
        n = len(shards)
        L = ep_buffer_layout(T, cfg.K, cfg.H)
        self.bufs = [torch.zeros(L.total, dtype=torch.uint8, device=device) for _ in range(n)]
        addrs = [EpRankBuffers.addresses(b.data_ptr(), T, cfg.K, cfg.H) for b in self.bufs]
        peers = {k: [a[k] for a in addrs] for k in addrs[0]}
        self.ranks = [EpPeerRank(cfg, sh, n, r, T, EpRankBuffers(self.bufs[r], T, cfg.K, cfg.H), peers,
                                 return_in_gemm) for r, sh in enumerate(shards)]
        self.peers = peers

    def forward(self, inputs):
        """inputs[r] = (logits, bias, x) of rank r; returns the n ranks' outputs."""
        if len(inputs) != len(self.ranks):
            raise ValueError(f"one input set per rank ({len(self.ranks)}), got {len(inputs)}")
        for rk, args in zip(self.ranks, inputs):
            rk.publish(*args)
        B.moe_ep_barrier_emulated(self.peers["barrier"])
        for rk in self.ranks:
            rk.compute()
        B.moe_ep_barrier_emulated(self.peers["barrier"])
        return [rk.combine() for rk in self.ranks]

    @property
    def barriers_passed(self) -> int:
        """Barrier calls made so far, by every rank's device-side counter (which must agree)."""
        counts = {int(rk.mine.barrier[B.EP_BARRIER_WORDS - 1]) for rk in self.ranks}
        if len(counts) != 1:
            raise RuntimeError(f"the ranks' barrier counters disagree: {sorted(counts)}")
        return counts.pop()
