"""GPU parity of the expert mask (the expert_mask argument of the page's asm_moe call: an
expert-parallel rank's partial output) and of bf16 router logits (the page's routing test
runs over a dtype), against the CPU oracle through the C ABI."""
import pytest
import torch

from oracle import fp8moe_oracle as O
from fp8_block_scaled_biased_b200 import binding as B
from fp8_block_scaled_biased_b200 import inputs as I
from fp8_block_scaled_biased_b200.layer import MoELayer
from tests.gpu_helpers import assert_moe_close, blocks_covered, full_size_tokens, oracle_moe_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"
MID = I.MoEConfig("mid_t256_h1024_e32", T=256, H=1024, E=32, G=4, TG=2, K=4, I=512, seed=1)
FEW = I.MoEConfig("few_t300_h256_e6_k2", T=300, H=256, E=6, G=2, TG=1, K=2, I=256, seed=5)
ODD = I.MoEConfig("odd_t37_h640_e24_k5", T=37, H=640, E=24, G=4, TG=3, K=5, I=384, seed=4)


@pytest.fixture(autouse=True)
def _device_status_clean():
    yield
    assert B.device_status() == 0


def rank_mask(E, rank, nranks):
    """Experts of one expert-parallel rank: e % nranks == rank."""
    return (torch.arange(E) % nranks == rank).to(torch.int32)


# ---------------------------------------------------------------- bf16 router logits
@pytest.mark.parametrize("cfg", [I.TINY, I.DECODE, I.PREFILL, ODD], ids=lambda c: c.name)
@pytest.mark.parametrize("pad", [0, 3])
def test_routing_bf16_logits_bit_exact(cfg, pad):
    act = I.moe_activations(cfg)
    # pad 3: row stride E + 3, so rows are not 8-byte aligned (scalar loads)
    wide = act.logits.to(torch.bfloat16)
    if pad:
        wide = torch.cat([wide, torch.zeros(cfg.T, pad, dtype=torch.bfloat16)], dim=1)
    lg = wide.to(DEV)[:, : cfg.E]
    ld = cfg.K + 10
    wbuf = torch.full((cfg.T, ld), -7.0, device=DEV)
    ibuf = torch.full((cfg.T, ld), -7, dtype=torch.int32, device=DEV)
    w, ids = wbuf[:, : cfg.K], ibuf[:, : cfg.K]
    B.moe_biased_grouped_topk(lg, act.bias.to(DEV), w, ids, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    w_ref, ids_ref = O.biased_grouped_topk(lg.cpu(), act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    assert torch.equal(ids.cpu(), ids_ref)
    assert torch.equal(w.cpu().view(torch.int32), w_ref.view(torch.int32))
    assert (wbuf[:, cfg.K:] == -7.0).all() and (ibuf[:, cfg.K:] == -7).all()


def test_fused_layer_with_bf16_logits():
    cfg = MID
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    act = I.moe_activations(cfg)
    lg = act.logits.to(torch.bfloat16)
    out = layer.forward(lg.to(DEV), act.bias.to(DEV), act.x.to(DEV)).clone()
    act16 = I.MoEActivations(logits=lg.float(), bias=act.bias, x=act.x)
    ref, _, ids_ref = oracle_moe_rows(cfg, act16, None)
    assert torch.equal(layer.topk_ids.cpu(), ids_ref)
    assert_moe_close(out, ref)


# ---------------------------------------------------------------- expert mask: sort
@pytest.mark.parametrize("cfg,block_m,nranks", [(I.TINY, 4, 4), (I.DECODE, 128, 8), (I.PREFILL, 128, 8),
                                                (I.SKEWED, 128, 8), (FEW, 16, 3)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_masked_sort_bit_exact(cfg, block_m, nranks):
    act = I.moe_activations(cfg)
    w_ref, ids_ref = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    for rank in (0, nranks - 1):
        mask = rank_mask(cfg.E, rank, nranks)
        sp = B.alloc_sorted(cfg.T, cfg.K, cfg.E, block_m, DEV)
        sp.sorted_ids.fill_(-5)
        B.moe_align_sort(ids_ref.to(DEV), w_ref.to(DEV), cfg.E, block_m, out=sp, expert_mask=mask.to(DEV))
        sid, sw, se, nv = O.align_sort(ids_ref, w_ref, cfg.E, block_m, expert_mask=mask)
        assert sp.num_valid_ids.item() == nv
        assert torch.equal(sp.sorted_ids[:nv].cpu(), sid)
        assert torch.equal(sp.sorted_weights[:nv].cpu().view(torch.int32), sw.view(torch.int32))
        assert torch.equal(sp.sorted_expert_ids[: nv // block_m].cpu(), se)
        assert (sp.sorted_ids[nv:] == -5).all()


def test_masked_sort_all_masked_is_empty():
    cfg = I.DECODE
    act = I.moe_activations(cfg)
    w_ref, ids_ref = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    sp = B.moe_align_sort(ids_ref.to(DEV), w_ref.to(DEV), cfg.E, 128,
                          expert_mask=torch.zeros(cfg.E, dtype=torch.int32, device=DEV))
    assert sp.num_valid_ids.item() == 0


# ---------------------------------------------------------------- expert mask: fused layer
@pytest.mark.parametrize("cfg,nranks", [(I.TINY, 4), (MID, 4), (FEW, 3)], ids=lambda v: getattr(v, "name", str(v)))
def test_fused_moe_expert_parallel_partials(cfg, nranks):
    """Each rank's masked output matches the oracle's partial output, and the ranks' outputs
    add up to the whole layer's (each partial is rounded to bf16 once)."""
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    act = I.moe_activations(cfg)
    args = (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
    total = torch.zeros(cfg.T, cfg.H, dtype=torch.float64)
    for rank in range(nranks):
        mask = rank_mask(cfg.E, rank, nranks)
        out = layer.forward(*args, expert_mask=mask.to(DEV)).clone()
        ref, _, _ = oracle_moe_rows(cfg, act, None, expert_mask=mask)
        assert_moe_close(out, ref)
        assert torch.equal(out, layer.forward(*args, expert_mask=mask.to(DEV)))   # deterministic
        total += out.double().cpu()
    ref_full, _, _ = oracle_moe_rows(cfg, act, None)
    assert_moe_close(total, ref_full)


def test_fused_moe_expert_mask_full_size_many_tokens():
    """Expert-parallel rank 5 of 8 on the prefill layer: 256 seeded tokens, the first and
    last token and every token of the rank's most-loaded kept expert, chosen from the
    oracle's routing, against the oracle's partial output."""
    cfg = I.PREFILL
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    act = I.moe_activations(cfg)
    mask = rank_mask(cfg.E, 5, 8)
    out = layer.forward(act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV), expert_mask=mask.to(DEV)).clone()
    _, ids_ref = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    tokens, roles = full_size_tokens(cfg, ids_ref, 256, seed=7, m64_tail=False, expert_mask=mask)
    assert int(mask[roles["most_loaded"]]) == 1 and tokens.numel() >= 256
    hit, nblocks = blocks_covered(ids_ref, tokens, cfg.E, expert_mask=mask)
    assert hit >= 0.75 * nblocks, (hit, nblocks)
    ref, _, _ = oracle_moe_rows(cfg, act, tokens, expert_mask=mask)
    assert_moe_close(out.cpu()[tokens], ref)


def test_fused_moe_leaves_out_dropped_pairs():
    """Ids outside [0, E) are dropped by the sort (and flagged); the fused layer sums the rest."""
    cfg = MID
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    act = I.moe_activations(cfg)
    w, ids = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    ids = ids.clone()
    ids[0, 1] = cfg.E + 3
    ids[5, 0] = -1
    ids[9, :] = cfg.E                       # a token with no valid pair: zero row
    sp = B.moe_align_sort(ids.to(DEV), w.to(DEV), cfg.E, layer.block_m)
    assert B.device_status() & 2            # FP8MOE_DEVERR_EXPERT_ID (read and cleared)
    a8, a1 = B.fp8_per_token_group_quant(act.x.to(DEV), 128, column_major_scales=True)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=DEV)
    B.fused_moe_fp8_blockscale_g1u1(out, a8, layer.w1, layer.w2, sp, cfg.K, a1, layer.w1_scale, layer.w2_scale)
    assert B.device_status() == 0
    a8r, ascr = O.quant_1x128(act.x)
    from tests.gpu_helpers import oracle_expert
    ref = O.moe_layer(a8r, ascr, ids, w, lambda e: oracle_expert(cfg, e), round_bf16=False,
                      expert_mask=torch.ones(cfg.E, dtype=torch.int32))
    assert (out[9] == 0).all()
    assert_moe_close(out, ref)
