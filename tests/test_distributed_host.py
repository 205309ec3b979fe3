"""Rank logic of the multi-GPU forms on the CPU: two or four gloo ranks, the oracle as
each rank's local compute.

Tensor parallelism: each rank's oracle partial output over its shard of I, rounded to bf16
as the device layer returns it, summed by tp_reduce, must equal the whole layer's oracle
output within the MoE tolerance on every rank. Expert parallelism: each rank routes and
quantises its own tokens with the oracle, ep_dispatch sends them to the experts' owners, each
owner's oracle computes the partial outputs of what it received (its experts only; the
sentinel id of other ranks' pairs masked out), ep_combine returns and sums them; the result
must equal the whole layer's oracle output for the rank's tokens. Nothing here touches a GPU.
"""
import os
import socket
import traceback

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import fp8moe_oracle as O
from fp8_block_scaled_biased_b200 import inputs as I
from fp8_block_scaled_biased_b200 import distributed as D
from tests.gpu_helpers import moe_error, oracle_expert

CFG = I.MoEConfig("host_dist_t48_h256_e8", T=48, H=256, E=8, G=2, TG=2, K=3, I=256, seed=7)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_full(cfg):
    act = I.moe_activations(cfg)
    w, ids = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    a8, asc = O.quant_1x128(act.x)
    ref = O.moe_layer(a8, asc, ids, w, lambda e: oracle_expert(cfg, e, "cpu"), round_bf16=False)
    return act, w, ids, a8, asc, ref


def _tp_rank(rank, n, cfg):
    act, w, ids, a8, asc, ref = _oracle_full(cfg)
    Is, nb = cfg.I // n, cfg.I // n // 128
    rows = torch.cat([torch.arange(rank * Is, (rank + 1) * Is), cfg.I + torch.arange(rank * Is, (rank + 1) * Is)])
    brows = torch.cat([torch.arange(rank * nb, (rank + 1) * nb), cfg.I // 128 + torch.arange(rank * nb, (rank + 1) * nb)])

    def shard(e):
        w1q, w1s, w2q, w2s = oracle_expert(cfg, e, "cpu")
        return w1q[rows], w1s[brows], w2q[:, rank * Is:(rank + 1) * Is], w2s[:, rank * nb:(rank + 1) * nb]

    partial = O.bf16_round(O.moe_layer(a8, asc, ids, w, shard, round_bf16=False)).to(torch.bfloat16)
    out = D.tp_reduce(partial)
    dmax, bound, mre = moe_error(out, ref)
    assert dmax <= bound and mre <= 5e-3, (dmax, bound, mre)
    everyone = [torch.empty_like(out) for _ in range(n)]
    dist.all_gather(everyone, out)
    assert all(torch.equal(o, out) for o in everyone)          # the same output on every rank
    return mre


def _ep_rank(rank, n, cfg):
    act, w, ids, a8, asc, ref = _oracle_full(cfg)
    tok = torch.arange(cfg.T).chunk(n)[rank]                     # this rank's own tokens
    e0, e1 = D.ep_expert_range(cfg.E, rank, n)
    received, plan = D.ep_dispatch(a8[tok], asc[tok], ids[tok], w[tok], cfg.E)
    r_a8, r_sc, r_ids, r_w = received
    # bookkeeping: one row per (token, owner) pair with work, from every source
    owners = ids.long() // (cfg.E // n)
    expect = sum(int(((owners[src_tok] == rank).any(dim=1)).sum()) for src_tok in torch.arange(cfg.T).chunk(n))
    assert r_a8.shape[0] == expect == sum(plan.recv_counts)
    assert int(r_ids.max()) <= e1 - e0 and int(r_ids.min()) >= 0
    # the owner's compute: its experts only, the sentinel id (e1 - e0) masked out
    mask = torch.ones(e1 - e0 + 1, dtype=torch.int32)
    mask[-1] = 0
    part = O.moe_layer(r_a8, r_sc, r_ids, r_w, lambda e: oracle_expert(cfg, e0 + e, "cpu"), round_bf16=False,
                       expert_mask=mask)
    out = D.ep_combine(O.bf16_round(part).to(torch.bfloat16), plan)
    dmax, bound, mre = moe_error(out, ref[tok])
    assert dmax <= bound and mre <= 5e-3, (dmax, bound, mre)
    return mre


def _worker(rank, n, port, which, cfg, errors):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.set_num_threads(2)
    try:
        import datetime
        dist.init_process_group("gloo", rank=rank, world_size=n, timeout=datetime.timedelta(seconds=60))
        (_tp_rank if which == "tp" else _ep_rank)(rank, n, cfg)
        dist.barrier()
    except Exception:  # noqa: BLE001 - reported to the parent
        errors.put(f"rank {rank}: {traceback.format_exc()}")
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def _run(which, n, cfg=CFG):
    ctx = mp.get_context("spawn")
    errors = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, n, port, which, cfg, errors)) for r in range(n)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    msgs = []
    while not errors.empty():
        msgs.append(errors.get())
    assert not alive, "a rank did not finish"
    assert not msgs, "\n".join(msgs)
    assert all(p.exitcode == 0 for p in procs)


@pytest.mark.parametrize("n", [2])
def test_tensor_parallel_shards_reduce_to_the_layer(n):
    _run("tp", n)


@pytest.mark.parametrize("n", [2, 4])
def test_expert_parallel_dispatch_and_combine_give_the_layer(n):
    _run("ep", n)


def test_single_rank_forms_need_no_process_group():
    """Without a process group tp_reduce returns the partial and the expert-parallel
    dispatch/combine pair is the identity around the local compute."""
    p = torch.randn(5, 128).to(torch.bfloat16)
    assert D.tp_reduce(p) is p
    cfg = CFG
    act, w, ids, a8, asc, ref = _oracle_full(cfg)
    (r_a8, r_sc, r_ids, r_w), plan = D.ep_dispatch(a8, asc, ids, w, cfg.E)
    assert torch.equal(r_a8, a8) and torch.equal(r_ids, ids) and torch.equal(r_w, w)
    rows = torch.randn(cfg.T, cfg.H).to(torch.bfloat16)
    assert torch.equal(D.ep_combine(rows, plan), rows)
    with pytest.raises(ValueError):
        D.ep_expert_range(10, 0, 4)


def test_tensor_parallel_buffer_layout():
    """One allocation per rank for the fused combine + all-reduce: the receive buffer bf16
    [n][ceil(T/n)][H], the output bf16 [T][H] and the flag words, each 256-byte aligned and
    not overlapping."""
    for T, H, n in ((4096, 7168, 8), (300, 1024, 8), (1, 128, 1), (37, 640, 3)):
        L = D.tp_buffer_layout(T, H, n)
        Ts = -(-T // n)
        assert L.recv == 0 and L.out >= n * Ts * H * 2 and L.flags >= L.out + T * H * 2
        assert L.total >= L.flags + 16 * 8
        assert L.out % 256 == 0 and L.flags % 256 == 0
    assert D.tp_buffer_layout(4096, 7168, 8).total == 117440768
    for bad in ((0, 128, 1), (16, 128, 0), (16, 128, 9)):
        with pytest.raises(ValueError):
            D.tp_buffer_layout(*bad)


def test_tensor_parallel_reduce_choice_is_checked():
    class _Layer:
        cfg = I.MoEConfig("t", T=4, H=128, E=4, G=1, TG=1, K=2, I=128, tp_ranks=1, tp_rank=0)
    assert D.TensorParallelMoE(_Layer(), reduce="peer").reduce == "peer"
    with pytest.raises(ValueError):
        D.TensorParallelMoE(_Layer(), reduce="ring")


def test_expert_parallel_buffer_layout():
    """What an expert-parallel rank publishes, in one allocation: routing ids and weights
    [T, K], activations [T, H] and scales [H/128, T], return rows [T*K, H] with a 16-byte
    count and T*K flag bytes, and the barrier words; 256-byte aligned, in that order."""
    for T, K, H in ((4096, 8, 7168), (100, 4, 1024), (1, 1, 128)):
        L = D.ep_buffer_layout(T, K, H)
        ends = [(L.ids, T * K * 4), (L.w, T * K * 4), (L.a8, T * H), (L.scale, H // 128 * T * 4),
                (L.rows, T * K * H * 2), (L.flags, 16 + T * K), (L.barrier, 8 * 8)]
        for (a, size), (b, _) in zip(ends, ends[1:] + [(L.total, 0)]):
            assert a % 256 == 0 and a + size <= b
    for bad in ((0, 8, 7168), (16, 0, 128), (16, 8, 100)):
        with pytest.raises(ValueError):
            D.ep_buffer_layout(*bad)
