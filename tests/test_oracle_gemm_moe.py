"""Pins for the oracle's block-scale GEMM and the fused g1u1 MoE layer.

The GEMM is pinned to a dense fp64 matmul of the dequantised operands (the
identity sum_kb sa*sb*S_kb = sum_k (qa*sa)(qb*sb)); the MoE layer to dense
per-expert FFNs computed with plain matmuls, to permutation equivariances and
to closed-form special cases.
"""
import pytest
import torch

from oracle import fp8moe_oracle as O
from fp8_block_scaled_biased_b200 import inputs as I

pytestmark = pytest.mark.filterwarnings("ignore")


def _q_act(x):
    return O.quant_1x128(x)


def _dense(q, s, block_rows):
    return O.dequant_rows(q, s, block_rows)


@pytest.mark.parametrize("M,N,K", [(5, 7, 128), (130, 260, 384), (64, 200, 300), (3, 129, 16)])
def test_blockscale_gemm_equals_dense_dequantised_matmul(M, N, K):
    g = torch.Generator().manual_seed(M + N + K)
    a = torch.randn(M, K, generator=g) * torch.logspace(-2, 1, M)[:, None]
    b = torch.randn(N, K, generator=g) * 0.02
    b[: min(N, 128), : min(K, 128)] *= 50                   # blocks with very different scales
    qa, sa = O.quant_1x128(a)
    qb, sb = O.quant_128x128(b)
    C = O.blockscale_gemm(qa, sa, qb, sb)
    Ad = O.dequant_rows(qa, sa, 1)                           # per-row scales
    Bd = O.dequant_rows(qb, sb, 128)
    ref = Ad @ Bd.T
    assert torch.allclose(C, ref, rtol=1e-12, atol=1e-12 * ref.abs().max().item())
    # operand roles: swapping A and B transposes C only when both use the same scale shape
    assert C.shape == (M, N)


def test_blockscale_gemm_block_sums_are_exact():
    g = torch.Generator().manual_seed(9)
    qa = torch.randint(0, 0x7E, (4, 256), generator=g, dtype=torch.int32).to(torch.uint8)
    qb = torch.randint(0, 0x7E, (3, 256), generator=g, dtype=torch.int32).to(torch.uint8)
    one_a = torch.ones(4, 2)
    one_b = torch.ones(1, 2)
    C = O.blockscale_gemm(qa, one_a, qb, one_b)
    # exact integer arithmetic in units of 2^-18 gives the same value
    ia = (O.e4m3_decode(qa) * 2 ** 9).long()
    ib = (O.e4m3_decode(qb) * 2 ** 9).long()
    exact = (ia @ ib.T).double() * 2.0 ** -18
    assert torch.equal(C, exact)


def _layer(cfg, act, dev="cpu"):
    w, ids = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    a8, asc = O.quant_1x128(act.x)
    experts = {}
    for e in range(cfg.E):
        w1q, w1s = O.quant_128x128(I.expert_weight_raw(cfg, "w1", e, dev))
        w2q, w2s = O.quant_128x128(I.expert_weight_raw(cfg, "w2", e, dev))
        experts[e] = (w1q, w1s, w2q, w2s)
    return w, ids, a8, asc, experts


def _dense_ffn(a8, asc, ex):
    """Expert FFN written densely: dequantise everything, then plain fp64 matmuls."""
    w1q, w1s, w2q, w2s = ex
    I_ = w2q.shape[1]
    x = O.dequant_rows(a8, asc, 1)
    g1 = x @ O.dequant_rows(w1q, w1s, 128).T
    gate, up = g1[:, :I_], g1[:, I_:]
    h = gate * torch.sigmoid(gate) * up
    a2, s2 = O.quant_1x128(h.float())
    return O.dequant_rows(a2, s2, 1) @ O.dequant_rows(w2q, w2s, 128).T


def test_moe_layer_equals_dense_all_expert_evaluation():
    cfg = I.MoEConfig("pin_small", T=10, H=256, E=4, G=2, TG=1, K=2, I=128, seed=3)
    act = I.moe_activations(cfg)
    w, ids, a8, asc, ex = _layer(cfg, act)
    out = O.moe_layer(a8, asc, ids, w, lambda e: ex[e], round_bf16=False)
    # every expert on every token, then pick each token's experts by id
    ys = torch.stack([_dense_ffn(a8, asc, ex[e]) for e in range(cfg.E)])   # [E, T, H]
    ref = torch.zeros(cfg.T, cfg.H, dtype=torch.float64)
    for t in range(cfg.T):
        for k in range(cfg.K):
            ref[t] += w[t, k].double() * ys[ids[t, k].item(), t]
    scale = ref.abs().max().item()
    # only GEMM1 rounding order and exp differ; they can move an FP8 code of h by one step
    d = (out - ref).abs()
    assert d.max() <= 2e-3 * scale
    assert d.sum() <= 1e-4 * ref.abs().sum()


def test_moe_layer_single_expert_closed_form():
    cfg = I.MoEConfig("pin_e1", T=6, H=128, E=1, G=1, TG=1, K=1, I=128, scale=2.5, seed=4)
    act = I.moe_activations(cfg)
    w, ids, a8, asc, ex = _layer(cfg, act)
    assert (ids == 0).all() and torch.equal(w, torch.full((6, 1), 2.5))   # renorm -> factor
    out = O.moe_layer(a8, asc, ids, w, lambda e: ex[e], round_bf16=False)
    ref = 2.5 * _dense_ffn(a8, asc, ex[0])
    assert torch.allclose(out, ref, rtol=1e-3, atol=1e-6 * ref.abs().max().item())


def test_moe_layer_equivariances_and_zero_input():
    cfg = I.TINY
    act = I.moe_activations(cfg)
    w, ids, a8, asc, ex = _layer(cfg, act)
    get = lambda e: ex[e]
    out = O.moe_layer(a8, asc, ids, w, get, round_bf16=False)
    # token permutation permutes the output rows
    perm = torch.randperm(cfg.T, generator=torch.Generator().manual_seed(0))
    out_p = O.moe_layer(a8[perm], asc[perm], ids[perm], w[perm], get, round_bf16=False)
    assert torch.equal(out_p, out[perm])
    # relabelling experts (and their ids) changes nothing
    rel = torch.randperm(cfg.E, generator=torch.Generator().manual_seed(1))
    inv = torch.argsort(rel)
    out_r = O.moe_layer(a8, asc, rel[ids.long()].int(), w, lambda e: ex[inv[e].item()], round_bf16=False)
    assert torch.equal(out_r, out)
    # weights enter linearly; a power-of-two factor is exact
    out_2 = O.moe_layer(a8, asc, ids, w * 2, get, round_bf16=False)
    assert torch.equal(out_2, out * 2)
    # zero hidden states give zero output
    z8, zs = O.quant_1x128(torch.zeros(cfg.T, cfg.H, dtype=torch.bfloat16))
    assert (O.moe_layer(z8, zs, ids, w, get) == 0).all()
    # token subsets give the same rows
    sub = [1, 5, 9]
    assert torch.equal(O.moe_layer(a8, asc, ids, w, get, tokens=sub, round_bf16=False), out[sub])


def test_moe_layer_expert_mask_against_dense_evaluation_and_partition():
    """Expert mask (the page's asm_moe expert_mask): only kept experts' pairs add. Pinned to the
    dense all-expert evaluation restricted to kept experts, and to the expert-parallel identity:
    the partial outputs of a partition of the experts sum to the unmasked output."""
    cfg = I.MoEConfig("pin_mask", T=12, H=256, E=8, G=2, TG=2, K=3, I=128, seed=6)
    act = I.moe_activations(cfg)
    w, ids, a8, asc, ex = _layer(cfg, act)
    get = lambda e: ex[e]
    mask = torch.tensor([1, 0, 0, 1, 1, 0, 1, 0], dtype=torch.int32)
    out = O.moe_layer(a8, asc, ids, w, get, round_bf16=False, expert_mask=mask)
    ys = torch.stack([_dense_ffn(a8, asc, ex[e]) for e in range(cfg.E)])
    ref = torch.zeros(cfg.T, cfg.H, dtype=torch.float64)
    for t in range(cfg.T):
        for k in range(cfg.K):
            e = ids[t, k].item()
            if mask[e]:
                ref[t] += w[t, k].double() * ys[e, t]
    scale = ref.abs().max().item()
    d = (out - ref).abs()
    assert d.max() <= 2e-3 * scale and d.sum() <= 1e-4 * ref.abs().sum()
    full = O.moe_layer(a8, asc, ids, w, get, round_bf16=False)
    parts = [O.moe_layer(a8, asc, ids, w, get, round_bf16=False,
                         expert_mask=(torch.arange(cfg.E) % 4 == r).int()) for r in range(4)]
    assert torch.allclose(sum(parts), full, rtol=1e-12, atol=1e-12 * full.abs().max().item())
    none = O.moe_layer(a8, asc, ids, w, get, expert_mask=torch.zeros(cfg.E, dtype=torch.int32))
    assert (none == 0).all()


def test_moe_layer_tensor_parallel_shards_sum_to_the_layer():
    """TP over I (the pages' TP8 run): each rank holds every expert's I/n intermediate columns
    (gate and up rows of w1, columns of w2, with their block scales). The 1x128 requantisation
    groups lie inside a shard, so the ranks' partial outputs sum to the whole layer's output."""
    cfg = I.MoEConfig("pin_tp", T=9, H=256, E=4, G=2, TG=1, K=2, I=512, seed=8)
    act = I.moe_activations(cfg)
    w, ids, a8, asc, ex = _layer(cfg, act)
    full = O.moe_layer(a8, asc, ids, w, lambda e: ex[e], round_bf16=False)
    for n in (2, 4):
        Is, nb = cfg.I // n, cfg.I // n // 128

        def shard(e, r):
            w1q, w1s, w2q, w2s = ex[e]
            rows = torch.cat([torch.arange(r * Is, (r + 1) * Is), cfg.I + torch.arange(r * Is, (r + 1) * Is)])
            brows = torch.cat([torch.arange(r * nb, (r + 1) * nb), cfg.I // 128 + torch.arange(r * nb, (r + 1) * nb)])
            return (w1q[rows], w1s[brows], w2q[:, r * Is:(r + 1) * Is], w2s[:, r * nb:(r + 1) * nb])

        total = sum(O.moe_layer(a8, asc, ids, w, lambda e, r=r: shard(e, r), round_bf16=False) for r in range(n))
        assert torch.allclose(total, full, rtol=1e-12, atol=1e-12 * full.abs().max().item())
