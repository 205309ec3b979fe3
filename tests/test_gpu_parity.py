"""GPU parity: every step of the CUDA path, called through the C ABI, against the oracle.

Bit-exact for routing ids/weights, the sort, and FP8 codes and scales; the
stated tolerance for the GEMM and the fused MoE output. Inputs come from the
seeded generator; each side quantises raw numbers with its own code.
"""
import dataclasses

import pytest
import torch

from oracle import fp8moe_oracle as O
from fp8_block_scaled_biased_b200 import binding as B
from fp8_block_scaled_biased_b200 import inputs as I
from fp8_block_scaled_biased_b200.layer import MoELayer
from tests.gpu_helpers import (assert_moe_close, blocks_covered, e4m3_ordinal, full_size_tokens,
                                fused_workspace_intermediate, m64_tail_expert, oracle_expert, oracle_moe_rows,
                                tokens_of_expert)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device"),
              pytest.mark.filterwarnings("ignore")]

DEV = "cuda"
MOE = [I.TINY, I.DECODE, I.PREFILL, I.SKEWED]


def u8(t):
    return t.view(torch.uint8).cpu() if t.dtype == B.FP8 else t.cpu()


@pytest.fixture(autouse=True)
def _device_status_clean():
    yield
    assert B.device_status() == 0


# ---------------------------------------------------------------- FP8 conversion and sigmoid recipe
def test_hardware_e4m3_conversion_matches_oracle_encoder():
    g = torch.Generator().manual_seed(11)
    vals = torch.cat([torch.randn(1 << 20, generator=g) * 40, torch.randn(1 << 18, generator=g) * 1e-2,
                      (torch.rand(1 << 16, generator=g) - 0.5) * 2 ** -6,
                      O.e4m3_decode(torch.arange(0, 0x7E, dtype=torch.int64)),        # grid points
                      ]).float().clamp(-448, 448)
    mids = O.e4m3_decode(torch.arange(0, 0x7E, dtype=torch.int64))
    mids = ((mids[1:] + mids[:-1]) / 2).float()
    vals = torch.cat([vals, mids, -mids])
    n = (vals.numel() + 16383) // 16384 * 16384
    w = torch.zeros(n, dtype=torch.float32)
    w[: vals.numel()] = vals
    w = w.view(-1, 128)
    w[::128, 0] = 448.0            # every 128x128 block holds 448, so its scale is exactly 1
    q, s = B.fp8_per_block_quant(w.to(DEV))
    assert (s.cpu() == 1.0).all()
    assert torch.equal(u8(q), O.e4m3_encode(w))


def test_sigmoid_recipe_is_bit_identical():
    # one group, all experts kept, no bias, no renorm: the weights are the sigmoid values
    T, E = 1 << 15, 32
    g = torch.Generator().manual_seed(12)
    logits = torch.cat([torch.randn(T // 2, E, generator=g) * 4, (torch.rand(T // 2, E, generator=g) - 0.5) * 190])
    bias = torch.zeros(E)
    w = torch.empty(T, E, device=DEV)
    ids = torch.empty(T, E, dtype=torch.int32, device=DEV)
    B.moe_biased_grouped_topk(logits.to(DEV), bias.to(DEV), w, ids, 1, 1, False, 1.0)
    w_ref, ids_ref = O.biased_grouped_topk(logits, bias, E, 1, 1, False, 1.0)
    assert torch.equal(ids.cpu(), ids_ref)
    assert torch.equal(w.cpu().view(torch.int32), w_ref.view(torch.int32))


# ---------------------------------------------------------------- S1 routing
@pytest.mark.parametrize("cfg", MOE, ids=lambda c: c.name)
def test_routing_bit_exact_with_strided_outputs(cfg):
    act = I.moe_activations(cfg)
    ld = cfg.K + 10                                   # strided outputs, as the pages' test allocates them
    wbuf = torch.full((cfg.T, ld), -7.0, device=DEV)
    ibuf = torch.full((cfg.T, ld), -7, dtype=torch.int32, device=DEV)
    w, ids = wbuf[:, : cfg.K], ibuf[:, : cfg.K]
    B.moe_biased_grouped_topk(act.logits.to(DEV), act.bias.to(DEV), w, ids, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    w_ref, ids_ref = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    assert torch.equal(ids.cpu(), ids_ref)
    assert torch.equal(w.cpu().view(torch.int32), w_ref.view(torch.int32))
    assert (wbuf[:, cfg.K:] == -7.0).all() and (ibuf[:, cfg.K:] == -7).all()


@pytest.mark.parametrize("E,G,TG,K", [(256, 8, 4, 8), (64, 8, 3, 6), (16, 1, 1, 4), (24, 4, 2, 5)])
def test_routing_ties_resolve_like_the_oracle(E, G, TG, K):
    """Logits and biases on a few levels, so equal biased scores and equal group scores are
    common: the kernel must break ties toward the lower group and expert index."""
    g = torch.Generator().manual_seed(E + K)
    T = 512
    logits = torch.randint(-2, 3, (T, E), generator=g).float() * 0.5
    bias = torch.randint(0, 2, (E,), generator=g).float() * 0.25
    w = torch.empty(T, K, device=DEV)
    ids = torch.empty(T, K, dtype=torch.int32, device=DEV)
    B.moe_biased_grouped_topk(logits.to(DEV), bias.to(DEV), w, ids, G, TG, True, 2.5)
    w_ref, ids_ref = O.biased_grouped_topk(logits, bias, K, G, TG, True, 2.5)
    assert torch.equal(ids.cpu(), ids_ref)
    assert torch.equal(w.cpu().view(torch.int32), w_ref.view(torch.int32))


@pytest.mark.parametrize("E,G,TG,K", [(512, 16, 4, 32), (512, 1, 1, 32), (384, 32, 32, 32)],
                         ids=["e512_g16_k32", "e512_g1_k32", "e384_g32_k32"])
def test_routing_at_the_size_limits(E, G, TG, K):
    """The routing kernel's limits: 512 experts (16 per lane), topk 32, 32 groups, and a group
    size (12) that takes the kernel's generic experts-per-lane path."""
    g = torch.Generator().manual_seed(E * K + G)
    T = 300
    logits = torch.randn(T, E, generator=g) * 2
    bias = torch.randn(E, generator=g) * 0.1
    w = torch.empty(T, K, device=DEV)
    ids = torch.empty(T, K, dtype=torch.int32, device=DEV)
    B.moe_biased_grouped_topk(logits.to(DEV), bias.to(DEV), w, ids, G, TG, True, 2.5)
    w_ref, ids_ref = O.biased_grouped_topk(logits, bias, K, G, TG, True, 2.5)
    assert torch.equal(ids.cpu(), ids_ref)
    assert torch.equal(w.cpu().view(torch.int32), w_ref.view(torch.int32))


# ---------------------------------------------------------------- S2 align/sort
@pytest.mark.parametrize("cfg,block_m", [(I.TINY, 4), (I.TINY, 128), (I.DECODE, 128), (I.DECODE, 16),
                                         (I.PREFILL, 128), (I.PREFILL, 64), (I.SKEWED, 128)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_sort_bit_exact(cfg, block_m):
    act = I.moe_activations(cfg)
    w_ref, ids_ref = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    sp = B.alloc_sorted(cfg.T, cfg.K, cfg.E, block_m, DEV)
    sp.sorted_ids.fill_(-5)
    sp.sorted_weights.fill_(-5.0)
    sp.sorted_expert_ids.fill_(-5)
    B.moe_align_sort(ids_ref.to(DEV), w_ref.to(DEV), cfg.E, block_m, out=sp)
    sid, sw, se, nv = O.align_sort(ids_ref, w_ref, cfg.E, block_m)
    assert sp.num_valid_ids.item() == nv
    assert torch.equal(sp.sorted_ids[:nv].cpu(), sid)
    assert torch.equal(sp.sorted_weights[:nv].cpu().view(torch.int32), sw.view(torch.int32))
    assert torch.equal(sp.sorted_expert_ids[: nv // block_m].cpu(), se)
    assert (sp.sorted_ids[nv:] == -5).all() and (sp.sorted_expert_ids[nv // block_m:] == -5).all()


@pytest.mark.parametrize("T", [30, 100], ids=["one_chunk", "four_chunks"])
def test_sort_at_the_size_limits(T):
    """1024 experts (the sort's limit) and topk 32: 960 pairs take the one-CTA path, 3200 the
    count + scatter path; both bit-exact against the oracle."""
    E, K = 1024, 32
    g = torch.Generator().manual_seed(T)
    ids = torch.stack([torch.randperm(E, generator=g)[:K] for _ in range(T)]).to(torch.int32)
    w = torch.rand(T, K, generator=g)
    sp = B.moe_align_sort(ids.to(DEV), w.to(DEV), E, 128)
    sid, sw, se, nv = O.align_sort(ids, w, E, 128)
    assert sp.num_valid_ids.item() == nv
    assert torch.equal(sp.sorted_ids[:nv].cpu(), sid)
    assert torch.equal(sp.sorted_weights[:nv].cpu().view(torch.int32), sw.view(torch.int32))
    assert torch.equal(sp.sorted_expert_ids[: nv // 128].cpu(), se)


def test_sort_empty_and_single_token():
    for T in (0, 1):
        ids = torch.arange(T * 4, dtype=torch.int32).view(T, 4) % 16
        w = torch.ones(T, 4)
        sp = B.moe_align_sort(ids.to(DEV), w.to(DEV), 16, 8)
        sid, sw, se, nv = O.align_sort(ids, w, 16, 8)
        assert sp.num_valid_ids.item() == nv
        assert torch.equal(sp.sorted_ids[:nv].cpu(), sid)


# ---------------------------------------------------------------- S3 quantisation
@pytest.mark.parametrize("M,K", [(16, 256), (64, 7168), (2048, 7168), (37, 200), (5, 136), (1, 8)])
@pytest.mark.parametrize("col_major", [False, True])
def test_quant_1x128_bit_exact(M, K, col_major):
    g = torch.Generator().manual_seed(M * 7 + K)
    x = (torch.randn(M, K, generator=g) * torch.logspace(-4, 3, M)[:, None]).to(torch.bfloat16)
    if M > 2:
        x[1, : min(K, 128)] = 0                      # an all-zero group
    q, s = B.fp8_per_token_group_quant(x.to(DEV), 128, column_major_scales=col_major)
    q_ref, s_ref = O.quant_1x128(x)
    assert torch.equal(u8(q), q_ref)
    s_gpu = s.cpu().t() if col_major else s.cpu()
    assert torch.equal(s_gpu.contiguous().view(torch.int32), s_ref.view(torch.int32))


def test_quant_1x128_quotients_near_e4m3_midpoints():
    """Groups holding elements whose fp32 quotient x / scale lies within 4 ulps of a midpoint
    between two E4M3 values, or below the E4M3 normal range: the quotients whose code a
    division rounded differently (for instance x times a rounded reciprocal) would change."""
    g = torch.Generator().manual_seed(11)
    x = torch.randn(16384, 128, generator=g).to(torch.bfloat16)
    y = (x.float() / (x.float().abs().amax(1, keepdim=True) / 448.0)).abs()
    below = y.view(torch.int32) & 0xFFFFF
    near = (((below - 0x80000).abs() <= 4) & (y >= 2.0 ** -6)) | ((y < 2.0 ** -6) & (y > 0))
    rows = near.any(1)
    assert int(rows.sum()) > 1000
    xs = x[rows].contiguous()
    q, s = B.fp8_per_token_group_quant(xs.to(DEV), 128)
    q_ref, s_ref = O.quant_1x128(xs)
    assert torch.equal(u8(q), q_ref)
    assert torch.equal(s.cpu().view(torch.int32), s_ref.view(torch.int32))


def test_quant_strided_rows():
    x = torch.randn(40, 512).to(torch.bfloat16)
    q, s = B.fp8_per_token_group_quant(x.to(DEV)[:, :384], 128)
    q_ref, s_ref = O.quant_1x128(x[:, :384])
    assert torch.equal(u8(q), q_ref) and torch.equal(s.cpu(), s_ref)


@pytest.mark.parametrize("which", ["random_300x260", "w1_4096x7168", "w2_7168x2048"])
def test_quant_128x128_bit_exact(which):
    if which.startswith("random"):
        w = (torch.randn(300, 260, generator=torch.Generator().manual_seed(3)) * 0.02).to(DEV)
    else:
        w = I.expert_weight_raw(I.DECODE, which[:2], 7, DEV)
    q, s = B.fp8_per_block_quant(w)
    q_ref, s_ref = O.quant_128x128(w.cpu())
    assert torch.equal(u8(q), q_ref)
    assert torch.equal(s.cpu().view(torch.int32), s_ref.view(torch.int32))


# ---------------------------------------------------------------- S0 block-scale GEMM
def _gemm_case(M, N, K, seed, sample_rows=None):
    g = torch.Generator().manual_seed(seed)
    a = (torch.randn(M, K, generator=g)).to(torch.bfloat16)
    b = torch.randn(N, K, generator=g) * 0.02
    qa, sa = B.fp8_per_token_group_quant(a.to(DEV), 128)
    qb, sb = B.fp8_per_block_quant(b.to(DEV))
    c = B.fp8_blockscale_gemm(qa, qb, sa, sb)
    rows = torch.arange(M) if sample_rows is None else sample_rows
    qa_ref, sa_ref = O.quant_1x128(a[rows])
    qb_ref, sb_ref = O.quant_128x128(b)
    ref = O.blockscale_gemm(qa_ref, sa_ref, qb_ref, sb_ref)
    got = c.cpu()[rows].double()
    return got, ref


def _assert_gemm_close(got, ref):
    d = (got - ref).abs()
    # bf16 output rounding (2^-9 relative) plus fp32 accumulation
    assert (d <= ref.abs() * 2.0 ** -8 + 1e-5 * ref.abs().max()).all(), d.max()
    assert d.max() <= 2e-2 * ref.abs().max() + 1e-3
    assert d.sum() / ref.abs().sum() <= 5e-3


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (200, 300, 400), (1, 8, 16), (257, 1000, 1024), (130, 520, 272)])
def test_gemm_small_and_ragged(M, N, K):
    got, ref = _gemm_case(M, N, K, seed=M + N + K)
    _assert_gemm_close(got, ref)


def test_gemm_2048x4096x7168_every_element():
    """The standalone GEMM workload (M=2048, N=4096, K=7168) compared in full: all
    8,388,608 outputs, every one of its 16 x 16 tiles and 56 K blocks."""
    got, ref = _gemm_case(2048, 4096, 7168, seed=0)
    _assert_gemm_close(got, ref)


def test_gemm_is_deterministic():
    g = torch.Generator().manual_seed(5)
    a = torch.randn(512, 1024, generator=g).to(torch.bfloat16).to(DEV)
    b = (torch.randn(768, 1024, generator=g) * 0.02).to(DEV)
    qa, sa = B.fp8_per_token_group_quant(a, 128)
    qb, sb = B.fp8_per_block_quant(b)
    c1 = B.fp8_blockscale_gemm(qa, qb, sa, sb).clone()
    c2 = B.fp8_blockscale_gemm(qa, qb, sa, sb)
    assert torch.equal(c1, c2)


def test_gemm_bounded_wait_runs_out_and_the_context_stays_usable():
    """Failure handling without a fault: the test hook withholds one K block's scales, the
    epilogue's bounded wait for them runs out (about 2 s), every CTA stops, frees its tensor
    memory and flags FP8MOE_DEVERR_TIMEOUT; the next GEMMs run normally."""
    g = torch.Generator().manual_seed(21)
    a = torch.randn(256, 512, generator=g).to(torch.bfloat16).to(DEV)
    b = (torch.randn(512, 512, generator=g) * 0.02).to(DEV)
    qa, sa = B.fp8_per_token_group_quant(a, 128)
    qb, sb = B.fp8_per_block_quant(b)
    c = torch.empty(256, 512, dtype=torch.bfloat16, device=DEV)
    B.selftest_gemm_stall(qa, qb, sa, sb, c, stall_kb=1)
    assert B.device_status() & 1                       # FP8MOE_DEVERR_TIMEOUT (read and cleared)
    assert B.device_status() == 0
    got, ref = _gemm_case(257, 1000, 1024, seed=3)     # TMEM and the context are intact
    _assert_gemm_close(got, ref)


# ---------------------------------------------------------------- S4-S7 fused MoE
MID = I.MoEConfig("mid_t256_h1024_e32", T=256, H=1024, E=32, G=4, TG=2, K=4, I=512, seed=1)
SKEW_SMALL = I.MoEConfig("skew_t512_h512_e64", T=512, H=512, E=64, G=8, TG=4, K=8, I=256, hot_experts=4, seed=2)


# Odd shapes: one token and one expert with H % 256 == 128 (the down GEMM's last column
# tile is half valid) and a single I block; E not a power of two with topk 5 and a ragged T;
# few experts, so each holds several row blocks (multi-block groups, M=64 tails).
ODD_ONE = I.MoEConfig("odd_t1_h384_e8_k1", T=1, H=384, E=8, G=1, TG=1, K=1, I=128, renorm=False, scale=1.0, seed=3)
ODD_E24 = I.MoEConfig("odd_t37_h640_e24_k5", T=37, H=640, E=24, G=4, TG=3, K=5, I=384, seed=4)
FEW_EXPERTS = I.MoEConfig("few_t300_h256_e6_k2", T=300, H=256, E=6, G=2, TG=1, K=2, I=256, seed=5)
# topk at its limit (32): every token picks half the experts
TOPK32 = I.MoEConfig("topk32_t40_h256_e64", T=40, H=256, E=64, G=1, TG=1, K=32, I=256, seed=8)


@pytest.mark.parametrize("cfg", [I.TINY, MID, SKEW_SMALL, ODD_ONE, ODD_E24, FEW_EXPERTS, TOPK32],
                         ids=lambda c: c.name)
def test_fused_moe_full_small_layers(cfg):
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    act = I.moe_activations(cfg)
    out = layer.forward(act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV)).clone()
    ref, w_ref, ids_ref = oracle_moe_rows(cfg, act, None)
    assert torch.equal(layer.topk_ids.cpu(), ids_ref)
    assert_moe_close(out, ref)
    out2 = layer.forward(act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
    assert torch.equal(out, out2)                      # deterministic combine


@pytest.mark.parametrize("E,N,K", [(1, 128, 128), (3, 384, 256), (2, 4096, 7168), (2, 7168, 2048)])
def test_tile_weights_layout(E, N, K):
    """fp8_tile_weights against the tiled layout's definition: block (e, nb, kb) holds rows
    nb*128.. and columns kb*128.. of matrix e, row-major inside the block."""
    g = torch.Generator().manual_seed(E * N + K)
    w = torch.randint(0, 256, (E, N, K), generator=g, dtype=torch.uint8)
    t = B.fp8_tile_weights(w.to(DEV).view(B.FP8))
    ref = w.view(E, N // 128, 128, K // 128, 128).permute(0, 1, 3, 2, 4).contiguous()
    assert torch.equal(t.view(torch.uint8).cpu(), ref)
    with pytest.raises(ValueError):
        B.fp8_tile_weights(torch.empty(1, 200, 128, dtype=B.FP8, device=DEV))


@pytest.mark.parametrize("cfg", [MID, SKEW_SMALL, ODD_ONE, ODD_E24, FEW_EXPERTS], ids=lambda c: c.name)
def test_fused_moe_tiled_weights_equal_row_major_bit_for_bit(cfg):
    """The fused call on tiled weights computes exactly what it computes on row-major ones:
    only the order in which the weight bytes sit in memory differs."""
    act = I.moe_activations(cfg)
    args = (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
    rm = MoELayer(cfg, DEV, tiled=False).load_synthetic_weights()
    tl = MoELayer(cfg, DEV, tiled=True).load_synthetic_weights()
    assert tl.tiled and tl.w1.dim() == 5
    out_rm = rm.forward(*args).clone()
    assert torch.equal(tl.forward(*args), out_rm)


@pytest.fixture(scope="module")
def big_layer():
    layer = MoELayer(I.DECODE, DEV).load_synthetic_weights()
    yield layer
    del layer
    torch.cuda.empty_cache()


def test_fused_moe_decode_every_token(big_layer):
    """The decode layer (T=64) compared in full: all 64 tokens, all 512 pairs."""
    cfg = I.DECODE
    layer = MoELayer(cfg, DEV, weights_from=big_layer)
    act = I.moe_activations(cfg)
    out = layer.forward(act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV)).clone()
    ref, w_ref, ids_ref = oracle_moe_rows(cfg, act, None)
    assert torch.equal(layer.topk_ids.cpu(), ids_ref)
    assert_moe_close(out, ref)
    out2 = layer.forward(act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
    assert torch.equal(out, out2)


@pytest.mark.parametrize("cfg", [I.PREFILL, I.SKEWED], ids=lambda c: c.name)
def test_fused_moe_full_size_many_tokens(big_layer, cfg):
    """The prefill (T=4096) and skewed (T=16384) layers: 512 seeded tokens and the first and
    last token; at prefill also every token of the most-loaded expert (1249 pairs, ten row
    blocks) and of the least-loaded expert with whole row blocks and an M=64 tail. The
    tokens are chosen from the oracle's routing; their pairs reach nearly every row block.
    (Every skewed expert carries thousands of pairs: its whole experts are compared pair by
    pair in the next test.)"""
    layer = MoELayer(cfg, DEV, weights_from=big_layer)
    act = I.moe_activations(cfg)
    out = layer.forward(act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV)).clone()
    _, ids_ref = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    assert torch.equal(layer.topk_ids.cpu(), ids_ref)
    whole = cfg is I.PREFILL
    tokens, roles = full_size_tokens(cfg, ids_ref, 512, seed=99, most_loaded=whole, m64_tail=whole)
    if whole:
        assert set(roles) == {"most_loaded", "m64_tail"}
    hit, nblocks = blocks_covered(ids_ref, tokens, cfg.E)
    assert hit >= 0.95 * nblocks, (hit, nblocks)
    ref, _, _ = oracle_moe_rows(cfg, act, tokens)
    assert_moe_close(out.cpu()[tokens], ref)
    out2 = layer.forward(act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
    assert torch.equal(out, out2)


def test_fused_moe_skewed_whole_experts_every_pair(big_layer):
    """Every pair of two skewed experts: the most-loaded one (12,856 pairs, 101 row blocks)
    and the least-loaded one whose last block runs as an M=64 tile (6,785 pairs). The expert
    mask keeps these two alone, so each token's output is the weighted sum of its pairs on
    them; the oracle computes it for every token they serve, and every other row is zero."""
    cfg = I.SKEWED
    layer = MoELayer(cfg, DEV, weights_from=big_layer)
    act = I.moe_activations(cfg)
    _, ids_ref = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    e_max = int(torch.bincount(ids_ref.flatten().long(), minlength=cfg.E).argmax())
    e_tail = m64_tail_expert(ids_ref, cfg.E)
    assert e_tail is not None and e_tail != e_max
    mask = torch.zeros(cfg.E, dtype=torch.int32)
    mask[[e_max, e_tail]] = 1
    out = layer.forward(act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV), expert_mask=mask.to(DEV)).clone()
    tokens = torch.unique(torch.cat([tokens_of_expert(ids_ref, e_max), tokens_of_expert(ids_ref, e_tail)]))
    assert tokens.numel() >= 100 * 128
    others = torch.ones(cfg.T, dtype=torch.bool)
    others[tokens] = False
    assert (out[others.to(DEV)] == 0).all()           # tokens without a pair on them: zero rows
    ref, _, _ = oracle_moe_rows(cfg, act, tokens, expert_mask=mask)
    assert_moe_close(out.cpu()[tokens], ref)


@pytest.mark.parametrize("which", ["mid", "decode"])
def test_requantised_intermediate_against_the_oracle(big_layer, which):
    """The gate/up GEMM's epilogue output (SiLU(gate) * up re-quantised 1x128 along I: codes
    a2 and scales s2 in the workspace) against the oracle's intermediate for every listed
    pair. The kernel takes SiLU with the fast exponential and division and quantises
    h * RN(1/scale) where the oracle divides exactly and works in fp64 before the final fp32
    rounding of h, so: every scale within 2e-5 relative (the fp32 accumulation of GEMM1),
    at most 0.5% of the codes different, none by more than one E4M3 step."""
    cfg = MID if which == "mid" else I.DECODE
    layer = (MoELayer(cfg, DEV).load_synthetic_weights() if which == "mid"
             else MoELayer(cfg, DEV, weights_from=big_layer))
    act = I.moe_activations(cfg)
    layer.forward(act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
    torch.cuda.synchronize()
    sp = layer.sorted
    cap = sp.capacity
    a2, s2 = fused_workspace_intermediate(layer.workspace, cap, cfg.T, cfg.K, cfg.H, cfg.I)
    a2, s2 = a2.cpu(), s2.cpu()
    nv = int(sp.num_valid_ids.item())
    sid = sp.sorted_ids[:nv].cpu().long()
    blk = sp.sorted_expert_ids[: nv // layer.block_m].cpu().long()
    P = cfg.T * cfg.K
    a8r, ascr = O.quant_1x128(act.x)
    diff_codes = total = 0
    worst_step = 0
    worst_scale = 0.0
    for e in torch.unique(blk).tolist():
        slots = torch.nonzero(blk.repeat_interleave(layer.block_m) == e).flatten()
        slots = slots[sid[slots] < P]
        t = sid[slots] // cfg.K
        w1q, w1s, _, _ = oracle_expert(cfg, e)
        q_ref, s_ref = O.expert_intermediate(a8r[t], ascr[t], w1q, w1s)
        s_gpu = s2[:, slots].t()
        rel = ((s_gpu.double() - s_ref.double()).abs() / s_ref.double().clamp_min(1e-30)).max().item()
        worst_scale = max(worst_scale, rel)
        q_gpu = a2[slots]
        diff = q_gpu != q_ref
        diff_codes += int(diff.sum())
        total += diff.numel()
        if diff.any():
            worst_step = max(worst_step, int((e4m3_ordinal(q_gpu) - e4m3_ordinal(q_ref)).abs().max()))
    print(f"{cfg.name}: scales within {worst_scale:.2e} relative, {diff_codes} of {total} codes differ "
          f"({diff_codes / total:.2e}), by at most {worst_step} step")
    assert worst_scale <= 2e-5, worst_scale
    assert worst_step <= 1, worst_step
    assert diff_codes <= 5e-3 * total, (diff_codes, total)


def test_timing_hook_reports_each_fused_kernel():
    """The measurement hook times gather, gate/up GEMM, down GEMM and combine of the latest call."""
    cfg = MID
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    act = I.moe_activations(cfg)
    args = (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
    layer.forward(*args)
    B.timing_enable(True)
    try:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        layer.forward(*args)
        end.record()
        ms = B.timing_last()
        torch.cuda.synchronize()
    finally:
        B.timing_enable(False)
    assert len(ms) == 4 and all(m > 0 for m in ms), ms
    assert sum(ms) <= start.elapsed_time(end) * 1.05 + 0.01


@pytest.mark.parametrize("cfg", [ODD_ONE, MID, SKEW_SMALL], ids=lambda c: c.name)
def test_graph_replays_follow_their_inputs(cfg):
    """The layer's forward captured in a CUDA graph (as the bench replays it: quantisation on
    a side stream joined before the fused call) gives on every replay exactly the eager
    forward's output for the inputs then in its buffers. Two input sets with different
    routings alternate between replays, so a kernel that read a buffer before its producer
    wrote it, or a sorted list left from the previous replay, would show the other set's
    values."""
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    sets = []
    for seed in (cfg.seed, cfg.seed + 100):
        act = I.moe_activations(dataclasses.replace(cfg, seed=seed))
        args = (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
        sets.append((args, layer.forward(*args).clone()))
    assert not torch.equal(sets[0][1], sets[1][1])
    bufs = tuple(t.clone() for t in sets[0][0])
    layer.forward(*bufs)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out = layer.forward(*bufs)
    for i in range(16):
        args, want = sets[i % 2]
        for b, a in zip(bufs, args):
            b.copy_(a)
        graph.replay()
        assert torch.equal(out, want), f"replay {i}"
    del graph


def test_fused_moe_zero_tokens_is_a_no_op():
    cfg = I.TINY
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    out = torch.full((0, cfg.H), 7.0, dtype=torch.bfloat16, device=DEV)
    a8 = torch.empty(0, cfg.H, dtype=torch.float8_e4m3fn, device=DEV)
    a1 = torch.empty(cfg.H // 128, 0, dtype=torch.float32, device=DEV)
    sorted_pairs = B.alloc_sorted(0, cfg.K, cfg.E, layer.block_m, DEV)
    B.fused_moe_fp8_blockscale_g1u1(out, a8, layer.w1, layer.w2, sorted_pairs, cfg.K, a1, layer.w1_scale,
                                    layer.w2_scale)
    torch.cuda.synchronize()
    assert out.numel() == 0


def test_fused_moe_flags_unsorted_block_experts():
    """Block expert ids that decrease (not a moe_align_sort result) raise the device error bit."""
    cfg = MID
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    act = I.moe_activations(cfg)
    layer.forward(act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
    assert B.device_status() == 0
    sp = layer.sorted
    nblocks = int(sp.num_valid_ids.item()) // layer.block_m
    ids = sp.sorted_expert_ids[:nblocks].clone()
    assert nblocks >= 2 and int(ids[0]) < int(ids[-1])
    sp.sorted_expert_ids[:nblocks] = torch.flip(ids, [0])
    B.fused_moe_fp8_blockscale_g1u1(layer.out, layer.a8, layer.w1, layer.w2, sp, cfg.K, layer.a8_scale,
                                    layer.w1_scale, layer.w2_scale, workspace=layer.workspace)
    assert B.device_status() & 16
    assert B.device_status() == 0          # read and cleared
