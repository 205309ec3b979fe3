"""GPU side of the multi-GPU forms, on one GPU: the expert shard each expert-parallel rank
runs (its experts' weights only, the received rows' local ids with other ranks' pairs as a
sentinel that the masked sort drops) against the oracle's partial outputs, for every rank of
a four-way split, and the one-rank expert- and tensor-parallel layers against the oracle. The
collectives between ranks are tested with gloo ranks on the CPU."""
import contextlib
import dataclasses

import pytest
import torch

from oracle import fp8moe_oracle as O
from fp8_block_scaled_biased_b200 import binding as B
from fp8_block_scaled_biased_b200 import distributed as D
from fp8_block_scaled_biased_b200 import inputs as I
from fp8_block_scaled_biased_b200.layer import MoELayer
from tests.gpu_helpers import assert_moe_close, oracle_moe_rows

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]
DEV = "cuda"
MID = I.MoEConfig("mid_t256_h1024_e32", T=256, H=1024, E=32, G=4, TG=2, K=4, I=512, seed=1)


@pytest.fixture(autouse=True)
def _device_status_clean():
    yield
    assert B.device_status() == 0


@pytest.mark.parametrize("n", [4])
def test_expert_shards_give_the_ranks_partials_and_sum_to_the_layer(n):
    cfg = MID
    act = I.moe_activations(cfg)
    w, ids = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    a8, sc = B.fp8_per_token_group_quant(act.x.to(DEV), 128)          # row-major scales, as dispatched
    total = torch.zeros(cfg.T, cfg.H, dtype=torch.float64)
    per = cfg.E // n
    for r in range(n):
        e0, e1 = D.ep_expert_range(cfg.E, r, n)
        shard = D.ExpertShard(cfg, e0, e1, DEV).load_synthetic_weights()
        rows = torch.nonzero((ids // per == r).any(dim=1)).flatten()
        loc = torch.where(ids[rows] // per == r, ids[rows] - e0, torch.full_like(ids[rows], per)).to(torch.int32)
        part = shard(a8[rows.to(DEV)], sc[rows.to(DEV)], loc.to(DEV), w[rows].to(DEV))
        mask = torch.zeros(cfg.E, dtype=torch.int32)
        mask[e0:e1] = 1
        ref, _, _ = oracle_moe_rows(cfg, act, rows, expert_mask=mask)
        assert_moe_close(part, ref)
        total[rows] += part.double().cpu()
    ref_full, _, _ = oracle_moe_rows(cfg, act, None)
    assert_moe_close(total, ref_full)


def test_one_rank_expert_and_tensor_parallel_layers_match_the_oracle():
    cfg = MID
    act = I.moe_activations(cfg)
    args = (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
    ref, _, _ = oracle_moe_rows(cfg, act, None)
    ep = D.ExpertParallelMoE(cfg, D.ExpertShard(cfg, 0, cfg.E, DEV).load_synthetic_weights())
    assert_moe_close(ep.forward(*args), ref)
    tp = D.TensorParallelMoE(MoELayer(cfg, DEV).load_synthetic_weights())
    out = tp.forward(*args)
    assert_moe_close(out, ref)


# ---------------------------------------------------------------- combine fused with the TP all-reduce
TPCFG = I.MoEConfig("tp_t300_h1024_e16", T=300, H=1024, E=16, G=4, TG=2, K=4, I=1024, seed=7)


def _rank_partials_and_workspaces(shards, args):
    """Each shard's combined partial (the fused call's own combine) and then its pairs-call
    workspace (the same pair rows, left uncombined)."""
    partials = [sh.forward(*args).clone() for sh in shards]
    workspaces = [sh.forward_pairs(*args) for sh in shards]
    return partials, workspaces


@pytest.mark.parametrize("n", [2, 4, 8])
def test_emulated_tp_combine_allreduce_is_the_rank_order_sum_of_the_partials(n):
    """Every rank of the fused combine + all-reduce on one GPU (one cooperative launch, each
    rank's CTAs running the one-rank code through the shared flags): every rank's output must
    equal, bit for bit, bf16 of the fp32 sum in rank order of the ranks' bf16 partials (each
    the fused call's own combine of that rank's pair rows), over three calls whose inputs
    alternate (each call's flag value comes from the ranks' device-side call counters); and
    the result must match the whole layer's oracle."""
    cfg = TPCFG
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    shards = [layer.tp_shard(r, n) for r in range(n)]
    emu = D.EmulatedTpAllReduce(cfg.T, cfg.H, n, DEV)
    sets = []
    for seed in (cfg.seed, cfg.seed + 50):
        act = I.moe_activations(dataclasses.replace(cfg, seed=seed))
        sets.append((act, (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))))
    for call in range(3):
        act, args = sets[call % 2]
        partials, workspaces = _rank_partials_and_workspaces(shards, args)
        outs = emu(workspaces, shards[0].sorted.capacity, cfg.K, cfg.I // n)
        torch.cuda.synchronize()
        want = partials[0].float()
        for p in partials[1:]:
            want = want + p.float()
        want = want.to(torch.bfloat16)
        for r in range(n):
            assert torch.equal(outs[r], want), f"call {call}, rank {r}"
        if call < 2:
            ref, _, _ = oracle_moe_rows(cfg, act, None)
            assert_moe_close(outs[0], ref)
    assert emu.calls == 3


def test_tp_combine_allreduce_bounded_wait_runs_out_without_its_peer():
    """Failure handling without a fault: rank 0 of 2 launched alone (rank 1's buffers are
    local stand-ins that nothing else touches) waits for rank 1's flags, which nothing sets;
    each bounded wait expires (about 2 s), FP8MOE_DEVERR_TIMEOUT is raised and the kernel
    ends; the context stays usable."""
    cfg = TPCFG
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    shard = layer.tp_shard(0, 2)
    act = I.moe_activations(cfg)
    ws = shard.forward_pairs(act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
    Ts = -(-cfg.T // 2)
    recv = [torch.empty(2, Ts, cfg.H, dtype=torch.bfloat16, device=DEV) for _ in range(2)]
    out = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=DEV) for _ in range(2)]
    flags = [torch.zeros(B.TP_FLAG_WORDS, dtype=torch.int64, device=DEV) for _ in range(2)]
    barrier = torch.zeros(B.TP_BARRIER_WORDS, dtype=torch.int64, device=DEV)
    B.moe_combine_allreduce(ws, shard.sorted.capacity, cfg.T, cfg.K, cfg.H, cfg.I // 2, 0, recv, out, flags,
                            barrier)
    assert B.device_status() & 1                       # FP8MOE_DEVERR_TIMEOUT (read and cleared)
    assert B.device_status() == 0
    assert int(flags[1][0]) == 1 and int(flags[0][0]) == 1    # rank 0 published its partials to both
    got = layer.forward(act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
    ref, _, _ = oracle_moe_rows(cfg, act, None)
    assert_moe_close(got, ref)                         # the context is intact


def test_tp_combine_allreduce_rejects_bad_arguments():
    cfg = TPCFG
    shard = MoELayer(cfg, DEV).tp_shard(0, 1)
    t = torch.zeros(16, dtype=torch.int64, device=DEV)
    buf = torch.zeros(1 << 20, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(B.Fp8MoeError):                 # H not a multiple of 128
        B.moe_combine_allreduce(shard.workspace, shard.sorted.capacity, cfg.T, cfg.K, cfg.H - 8, cfg.I, 0, [buf],
                                [buf], [t], t)
    with pytest.raises(B.Fp8MoeError):                 # rank outside [0, nranks)
        B.moe_combine_allreduce(shard.workspace, shard.sorted.capacity, cfg.T, cfg.K, cfg.H, cfg.I, 1, [buf], [buf],
                                [t], t)
    with pytest.raises(ValueError):                    # more ranks than the protocol takes
        B.moe_combine_allreduce(shard.workspace, shard.sorted.capacity, cfg.T, cfg.K, cfg.H, cfg.I, 0, [buf] * 9,
                                [buf] * 9, [t] * 9, t)
    assert B.device_status() == 0


@contextlib.contextmanager
def _one_rank_nccl_group(tmp_path):
    """A one-rank NCCL process group on this GPU over a file store (no TCP port to race for)."""
    import torch.distributed as dist
    store = dist.FileStore(str(tmp_path / "store"), 1)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, device_id=torch.device(DEV, 0))
    try:
        yield
    finally:
        dist.destroy_process_group()


def test_one_rank_peer_all_reduce_through_symmetric_memory(tmp_path):
    """The multi-GPU form's host side on a one-rank NCCL group: the buffers come from torch's
    symmetric memory and the pointers from its rendezvous; with one rank the fused combine +
    all-reduce is the combine, so the output equals the layer's own bit for bit."""
    import gc
    cfg = TPCFG
    with _one_rank_nccl_group(tmp_path):
        layer = MoELayer(cfg, DEV).load_synthetic_weights()
        act = I.moe_activations(cfg)
        args = (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
        want = layer.forward(*args).clone()
        tp = D.TensorParallelMoE(layer, reduce="peer")
        for _ in range(2):
            got = tp.forward(*args)
            torch.cuda.synchronize()
            assert torch.equal(got, want)
        assert tp.peer.calls == 2
        del tp, got
        gc.collect()
        torch.cuda.synchronize()


# ---------------------------------------------------------------- expert parallelism over peer memory
EPCFG = I.MoEConfig("ep_t100_h1024_e16", T=100, H=1024, E=16, G=4, TG=2, K=4, I=512, seed=9)
EP_HOT = I.MoEConfig("ep_hot_t96_h512_e32", T=96, H=512, E=32, G=4, TG=2, K=6, I=256, hot_experts=3, seed=11)


@pytest.mark.parametrize("cfg,n", [(EPCFG, 2), (EPCFG, 4), (EP_HOT, 4), (EP_HOT, 8)], ids=lambda v: str(getattr(v, "name", v)))
def test_emulated_peer_expert_parallel_equals_the_one_gpu_layer(cfg, n):
    """Every rank of the peer-memory expert-parallel form on one GPU (each with its own tokens
    and only its experts' weights; routing read across ranks, activation rows pulled by the
    owner's gather, pair rows returned to their origin, the two flag barriers as one launch
    over the ranks): each rank's output must equal the one-GPU layer's output for its tokens
    bit for bit, over two forwards. EP_HOT's boosted experts load the ranks unevenly."""
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    shards = [D.ExpertShard(cfg, *D.ep_expert_range(cfg.E, r, n), DEV).load_synthetic_weights() for r in range(n)]
    emu = D.EmulatedExpertParallel(cfg, shards, cfg.T, DEV)
    for call in range(2):
        inputs, wants = [], []
        for r in range(n):
            act = I.moe_activations(dataclasses.replace(cfg, seed=cfg.seed + 10 * r + 100 * call))
            args = (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
            inputs.append(args)
            wants.append(layer.forward(*args).clone())
        outs = emu.forward(inputs)
        torch.cuda.synchronize()
        for r in range(n):
            assert torch.equal(outs[r], wants[r]), f"forward {call}, rank {r}"
    assert emu.barriers_passed == 4


def test_ep_barrier_bounded_wait_runs_out_without_its_peer():
    """Rank 0 of 2 at the flag barrier alone: rank 1's word is never set, the bounded wait
    expires (about 2 s), FP8MOE_DEVERR_TIMEOUT is raised and the context stays usable."""
    words = [torch.zeros(B.EP_BARRIER_WORDS, dtype=torch.int64, device=DEV) for _ in range(2)]
    B.moe_ep_barrier(0, words)
    assert B.device_status() & 1
    assert B.device_status() == 0
    assert int(words[0][0]) == 1 and int(words[1][0]) == 1     # rank 0 published to both
    assert int(words[0][B.EP_BARRIER_WORDS - 1]) == 1          # and counted its call
    with pytest.raises(B.Fp8MoeError):
        B.moe_ep_barrier(2, words)                              # rank outside [0, n)


def test_one_rank_peer_expert_parallel_through_symmetric_memory(tmp_path):
    """The multi-GPU expert-parallel form's host side on a one-rank NCCL group (buffers from
    torch's symmetric memory, addresses from its rendezvous): with one rank it is the whole
    layer, so the output equals the layer's bit for bit."""
    import gc
    cfg = EPCFG
    with _one_rank_nccl_group(tmp_path):
        layer = MoELayer(cfg, DEV).load_synthetic_weights()
        act = I.moe_activations(cfg)
        args = (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
        want = layer.forward(*args).clone()
        ep = D.ExpertParallelPeerMoE(cfg, D.ExpertShard(cfg, 0, cfg.E, DEV).load_synthetic_weights(), cfg.T)
        for _ in range(2):
            got = ep.forward(*args)
            torch.cuda.synchronize()
            assert torch.equal(got, want)
        assert ep.barriers_passed == 4
        del ep, got
        gc.collect()
        torch.cuda.synchronize()


def test_emulated_peer_expert_parallel_with_the_return_kernel():
    """The same exchange with the pair rows left in each owner's workspace and copied to their
    origins by moe_ep_return instead of stored there by the down GEMM: the same outputs."""
    cfg, n = EP_HOT, 4
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    shards = [D.ExpertShard(cfg, *D.ep_expert_range(cfg.E, r, n), DEV).load_synthetic_weights() for r in range(n)]
    emu = D.EmulatedExpertParallel(cfg, shards, cfg.T, DEV, return_in_gemm=False)
    inputs, wants = [], []
    for r in range(n):
        act = I.moe_activations(dataclasses.replace(cfg, seed=cfg.seed + 7 * r))
        args = (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
        inputs.append(args)
        wants.append(layer.forward(*args).clone())
    outs = emu.forward(inputs)
    torch.cuda.synchronize()
    for r in range(n):
        assert torch.equal(outs[r], wants[r]), f"rank {r}"


# ---------------------------------------------------------------- degenerate splits
EP_EDGE = I.MoEConfig("ep_edge_t20_h256_e16", T=20, H=256, E=16, G=4, TG=1, K=4, I=256, seed=13)


def test_emulated_peer_expert_parallel_with_idle_owners():
    """Every pair on one rank's experts: the bias makes group 0 (experts 0-3, all of rank 0's
    four) the only group chosen, so ranks 1-3 own no pair at all (empty sorted lists, GEMMs
    with no tile) while still publishing, returning nothing and combining. Outputs must still
    equal the one-GPU layer's."""
    cfg, n = EP_EDGE, 4
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    shards = [D.ExpertShard(cfg, *D.ep_expert_range(cfg.E, r, n), DEV).load_synthetic_weights() for r in range(n)]
    emu = D.EmulatedExpertParallel(cfg, shards, cfg.T, DEV)
    inputs, wants = [], []
    for r in range(n):
        act = I.moe_activations(dataclasses.replace(cfg, seed=cfg.seed + r))
        bias = act.bias.clone()
        bias[:4] += 100.0
        args = (act.logits.to(DEV), bias.to(DEV), act.x.to(DEV))
        inputs.append(args)
        wants.append(layer.forward(*args).clone())
    assert int((layer.topk_ids >= 4).sum()) == 0                # the last input set: all on experts 0-3
    outs = emu.forward(inputs)
    torch.cuda.synchronize()
    for r in range(n):
        assert torch.equal(outs[r], wants[r]), f"rank {r}"
    assert [int(rk.sorted.num_valid_ids.item()) for rk in emu.ranks[1:]] == [0, 0, 0]


def test_emulated_tp_combine_allreduce_with_fewer_tokens_than_ranks():
    """T = 5 tokens over 8 ranks: slices of one token, and ranks 5-7 own no token (they still
    combine, publish and wait). Every rank's output must be the rank-order sum."""
    cfg = dataclasses.replace(TPCFG, name="tp_t5_h1024_e16", T=5)
    n = 8
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    shards = [layer.tp_shard(r, n) for r in range(n)]
    emu = D.EmulatedTpAllReduce(cfg.T, cfg.H, n, DEV)
    act = I.moe_activations(cfg)
    args = (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
    partials, workspaces = _rank_partials_and_workspaces(shards, args)
    outs = emu(workspaces, shards[0].sorted.capacity, cfg.K, cfg.I // n)
    torch.cuda.synchronize()
    want = partials[0].float()
    for p in partials[1:]:
        want = want + p.float()
    for r in range(n):
        assert torch.equal(outs[r], want.to(torch.bfloat16)), f"rank {r}"


# ---------------------------------------------------------------- the peer forms inside CUDA graphs
def test_tp_combine_allreduce_replays_in_a_cuda_graph():
    """The ranks' forwards and the fused combine + all-reduce captured in one CUDA graph: no
    value comes from the host per call (each call's flag value is the ranks' device-side call
    count plus one), so every replay runs the protocol afresh. Two input sets alternate between
    replays; every rank's output must be that set's rank-order sum each time."""
    cfg, n = TPCFG, 4
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    shards = [layer.tp_shard(r, n) for r in range(n)]
    emu = D.EmulatedTpAllReduce(cfg.T, cfg.H, n, DEV)
    cap, Is = shards[0].sorted.capacity, cfg.I // n
    sets, wants = [], []
    for seed in (cfg.seed, cfg.seed + 1):
        act = I.moe_activations(dataclasses.replace(cfg, seed=seed))
        args = (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
        want = None
        for sh in shards:
            p = sh.forward(*args).float()
            want = p if want is None else want + p
        sets.append(args)
        wants.append(want.to(torch.bfloat16))
    bufs = tuple(t.clone() for t in sets[0])

    def step():
        return emu([sh.forward_pairs(*bufs) for sh in shards], cap, cfg.K, Is)

    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        outs = step()
    for i in range(4):
        for b, a in zip(bufs, sets[i % 2]):
            b.copy_(a)
        graph.replay()
        torch.cuda.synchronize()
        for r in range(n):
            assert torch.equal(outs[r], wants[i % 2]), f"replay {i}, rank {r}"
    assert emu.calls == 5                               # one eager call and four replays
    del graph


def test_peer_expert_parallel_replays_in_a_cuda_graph():
    """The peer-memory expert-parallel forward of all ranks (routing read across ranks, the
    pulled gather, the rows stored into their origins by the down GEMM, both barriers) captured
    in one CUDA graph and replayed with alternating inputs: every rank's output equals the
    one-GPU layer's for its tokens on every replay."""
    cfg, n = EP_HOT, 4
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    shards = [D.ExpertShard(cfg, *D.ep_expert_range(cfg.E, r, n), DEV).load_synthetic_weights() for r in range(n)]
    emu = D.EmulatedExpertParallel(cfg, shards, cfg.T, DEV)
    sets, wants = [], []
    for call in range(2):
        inputs, want = [], []
        for r in range(n):
            act = I.moe_activations(dataclasses.replace(cfg, seed=cfg.seed + 10 * r + 100 * call))
            args = (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
            inputs.append(args)
            want.append(layer.forward(*args).clone())
        sets.append(inputs)
        wants.append(want)
    bufs = [tuple(t.clone() for t in args) for args in sets[0]]
    emu.forward(bufs)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        outs = emu.forward(bufs)
    for i in range(4):
        for rb, ra in zip(bufs, sets[i % 2]):
            for b, a in zip(rb, ra):
                b.copy_(a)
        graph.replay()
        torch.cuda.synchronize()
        for r in range(n):
            assert torch.equal(outs[r], wants[i % 2][r]), f"replay {i}, rank {r}"
    assert emu.barriers_passed == 10                    # two barriers per forward, five forwards
    del graph
