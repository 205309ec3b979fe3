"""GPU side of the multi-GPU forms, on one GPU: the expert shard each expert-parallel rank
runs (its experts' weights only, the received rows' local ids with other ranks' pairs as a
sentinel that the masked sort drops) against the oracle's partial outputs, for every rank of
a four-way split, and the one-rank expert- and tensor-parallel layers against the oracle. The
collectives between ranks are tested with gloo ranks on the CPU."""
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
