"""Pins for the oracle's fp32 exponential/sigmoid recipe and its grouped top-k routing."""
import itertools
import math

import pytest
import torch

from oracle import fp8moe_oracle as O
from fp8_block_scaled_biased_b200 import inputs as I

pytestmark = pytest.mark.filterwarnings("ignore")


def _ulp32(x):
    """Spacing of fp32 numbers at |x| (fp64)."""
    a = x.abs().to(torch.float64)
    _, k = torch.frexp(torch.where(a > 0, a, torch.ones_like(a)))
    return torch.pow(torch.tensor(2.0, dtype=torch.float64), (torch.clamp(k - 1, min=-126) - 23).double())


def test_exp_f32_within_2ulp_of_exact_on_a_sweep():
    # every 97th fp32 bit pattern in [-87, 88], plus the reduction boundaries
    lo, hi = torch.tensor(-87.0).view(torch.int32).item(), torch.tensor(88.0).view(torch.int32).item()
    pos = torch.arange(0, hi, 97, dtype=torch.int32).view(torch.float32)
    neg = torch.arange(torch.tensor(0.0).view(torch.int32).item() | 0, 0x7F800000, 97, dtype=torch.int64)
    neg = neg[neg <= (lo & 0x7FFFFFFF)].to(torch.int32).view(torch.float32).neg()
    k = torch.arange(-125, 127, dtype=torch.float64)
    edges = torch.cat([k * math.log(2), (k + 0.5) * math.log(2)]).to(torch.float32)
    y = torch.cat([pos, neg, edges[(edges >= -87) & (edges <= 88)]])
    got = O.exp_f32(y).double()
    ref = torch.exp(y.double())
    err = (got - ref).abs() / _ulp32(ref)
    assert err.max() <= 2.0, err.max()


def test_exp_f32_special_values():
    e = O.exp_f32(torch.tensor([0.0, 1.0, -1.0, 100.0, -100.0]))
    assert e[0] == 1.0
    assert abs(e[1].item() - math.e) <= 2 * 2.4e-7 and abs(e[2].item() - 1 / math.e) <= 2 * 3e-8
    assert torch.isfinite(e).all() and e[3] == O.exp_f32(torch.tensor([88.0]))[0]


def test_sigmoid_f32_matches_exact_and_is_monotone():
    x = torch.linspace(-30, 30, 200001, dtype=torch.float32)
    s = O.sigmoid_f32(x)
    ref = 1.0 / (1.0 + torch.exp(-x.double()))
    err = (s.double() - ref).abs() / _ulp32(ref)
    assert err.max() <= 3.0
    assert (s[1:] >= s[:-1]).all()
    assert O.sigmoid_f32(torch.tensor([0.0]))[0] == 0.5


def _route_bruteforce(logits, bias, K, G, TG, renorm, factor):
    """Routing by pairwise 'beats' counts and an exhaustive pair search, no sorting."""
    T, E = logits.shape
    per = E // G
    s = O.sigmoid_f32(logits)
    b = s + bias[None, :]
    ids = torch.empty(T, K, dtype=torch.int32)
    ws = torch.empty(T, K)
    for t in range(T):
        bt = b[t].tolist()
        bt32 = b[t]
        # group score: the largest fp32 sum over pairs of distinct members (rounding is monotone)
        gs = []
        for g in range(G):
            m = range(g * per, (g + 1) * per)
            best = None
            for i, j in itertools.combinations(m, 2):
                v = (bt32[i] + bt32[j]).item()
                best = v if best is None or v > best else best
            gs.append(best)
        beats = lambda vals, i, j: vals[j] > vals[i] or (vals[j] == vals[i] and j < i)
        chosen_g = [g for g in range(G) if sum(beats(gs, g, h) for h in range(G)) < TG]
        cand = [e for e in range(E) if e // per in chosen_g]
        rank = {e: sum(beats(bt, e, f) for f in cand) for e in cand}
        pick = sorted([e for e in cand if rank[e] < K], key=lambda e: rank[e])
        ids[t] = torch.tensor(pick, dtype=torch.int32)
        w = s[t, pick]
        if renorm:
            den = w[0]
            for j in range(1, K):
                den = den + w[j]
            w = w / den
        ws[t] = w * torch.tensor(factor, dtype=torch.float32)
    return ws, ids


@pytest.mark.parametrize("T,E,G,TG,K,renorm,factor,seed", [
    (16, 16, 4, 2, 4, True, 2.5, 0),
    (20, 32, 8, 3, 5, False, 1.0, 1),
    (12, 24, 3, 2, 6, True, 1.5, 2),
    (9, 64, 8, 4, 8, True, 2.5, 3),
])
def test_routing_matches_bruteforce(T, E, G, TG, K, renorm, factor, seed):
    g = torch.Generator().manual_seed(seed)
    logits = torch.randn(T, E, generator=g)
    bias = torch.randn(E, generator=g) * 0.1
    # plant exact ties: duplicated logits inside and across groups, equal group scores
    logits[0, 1] = logits[0, 0]
    logits[1, :] = logits[1, 0]
    bias[5] = bias[4]
    w, ids = O.biased_grouped_topk(logits, bias, K, G, TG, renorm, factor)
    wb, idb = _route_bruteforce(logits, bias, K, G, TG, renorm, factor)
    assert torch.equal(ids, idb)
    assert torch.equal(w, wb)


def test_routing_reduces_to_plain_topk_with_one_group_and_no_bias():
    g = torch.Generator().manual_seed(7)
    logits = torch.randn(50, 40, generator=g)
    w, ids = O.biased_grouped_topk(logits, torch.zeros(40), 6, 1, 1, False, 1.0)
    ref = torch.topk(logits, 6, dim=1)                        # sigmoid is monotone
    assert torch.equal(ids.long(), ref.indices)
    assert torch.allclose(w.double(), torch.sigmoid(ref.values.double()), rtol=3e-7, atol=0)


def test_routing_invariants_on_tiny_workload():
    cfg = I.TINY
    act = I.moe_activations(cfg)
    w, ids = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, True, cfg.scale)
    per = cfg.E // cfg.G
    for t in range(cfg.T):
        row = ids[t].tolist()
        assert len(set(row)) == cfg.K
        assert len({e // per for e in row}) <= cfg.TG
    assert torch.allclose(w.sum(1).double(), torch.full((cfg.T,), cfg.scale, dtype=torch.float64), rtol=1e-6)
    # the bias shifts selection only: adding a constant to every expert's bias changes nothing
    w2, ids2 = O.biased_grouped_topk(act.logits, act.bias + 0.25, cfg.K, cfg.G, cfg.TG, True, cfg.scale)
    assert torch.equal(ids, ids2) and torch.equal(w, w2)
    # the weights are the unbiased scores, renormalised
    s = O.sigmoid_f32(act.logits).gather(1, ids.long())
    assert torch.allclose(w.double(), (s / s.sum(1, keepdim=True) * cfg.scale).double(), rtol=1e-6)


def test_skewed_bias_concentrates_pairs():
    cfg = I.MoEConfig("skew_small", T=512, H=128, E=256, G=8, TG=4, K=8, I=128, hot_experts=16)
    act = I.moe_activations(cfg)
    _, ids = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, True, cfg.scale)
    hot = set(act.hot.tolist())
    frac_hot = sum(1 for e in ids.flatten().tolist() if e in hot) / ids.numel()
    assert frac_hot > 0.5
