"""Pins for the oracle's MoE align/sort: a library stable argsort and counting invariants."""
import pytest
import torch

from oracle import fp8moe_oracle as O


@pytest.mark.parametrize("T,K,E,BM,seed", [(16, 4, 16, 4, 0), (64, 8, 256, 16, 1), (300, 8, 32, 128, 2),
                                           (5, 2, 64, 32, 3), (1, 1, 8, 8, 4)])
def test_sort_matches_stable_argsort_and_invariants(T, K, E, BM, seed):
    g = torch.Generator().manual_seed(seed)
    # skewed ids: half the pairs on expert 3
    ids = torch.randint(0, E, (T, K), generator=g, dtype=torch.int32)
    ids[: T // 2, 0] = 3
    w = torch.rand(T, K, generator=g)
    sid, sw, se, nv = O.align_sort(ids, w, E, BM)
    P = T * K
    flat = ids.flatten().long()
    order = torch.argsort(flat, stable=True)                 # library stable sort by expert
    valid = sid < P
    assert torch.equal(sid[valid].long(), order)             # same pairs, same order
    assert torch.equal(sw[valid], w.flatten()[order])
    assert (sw[~valid] == 0).all()
    cnt = torch.bincount(flat, minlength=E)
    assert nv == int(((cnt + BM - 1) // BM * BM).sum())
    assert nv <= O.align_sort_capacity(T, K, E, BM) and nv % BM == 0
    # every block holds one expert's pairs, padding only at a segment's tail
    for j in range(nv // BM):
        blk = sid[j * BM:(j + 1) * BM].long()
        v = blk < P
        assert (flat[blk[v]] == se[j]).all()
        assert v[0] and torch.equal(v, torch.sort(v.int(), descending=True, stable=True).values.bool())
    assert torch.equal(torch.unique_consecutive(se.long()), torch.nonzero(cnt).flatten())


def test_sort_empty_input():
    sid, sw, se, nv = O.align_sort(torch.empty(0, 4, dtype=torch.int32), torch.empty(0, 4), 8, 16)
    assert nv == 0 and sid.numel() == 0 and se.numel() == 0


@pytest.mark.parametrize("T,K,E,BM,seed", [(64, 8, 256, 16, 1), (300, 8, 32, 128, 2), (16, 4, 16, 4, 5)])
def test_masked_sort_is_the_stable_sort_of_the_kept_pairs(T, K, E, BM, seed):
    """Expert mask (the page's asm_moe expert_mask): the kept pairs in a library stable argsort."""
    g = torch.Generator().manual_seed(seed)
    ids = torch.randint(0, E, (T, K), generator=g, dtype=torch.int32)
    w = torch.rand(T, K, generator=g)
    mask = (torch.rand(E, generator=g) < 0.4).int()
    mask[ids[0, 0]] = 1
    sid, sw, se, nv = O.align_sort(ids, w, E, BM, expert_mask=mask)
    P = T * K
    flat = ids.flatten().long()
    kept = torch.nonzero(mask.bool()[flat]).flatten()
    order = kept[torch.argsort(flat[kept], stable=True)]
    valid = sid < P
    assert torch.equal(sid[valid].long(), order)
    assert torch.equal(sw[valid], w.flatten()[order])
    cnt = torch.bincount(flat[kept], minlength=E)
    assert nv == int(((cnt + BM - 1) // BM * BM).sum())
    assert set(se.tolist()) <= set(torch.nonzero(mask).flatten().tolist())
    # an all-ones mask is no mask
    full = O.align_sort(ids, w, E, BM)
    ones = O.align_sort(ids, w, E, BM, expert_mask=torch.ones(E, dtype=torch.int32))
    assert all(torch.equal(a, b) for a, b in zip(full[:3], ones[:3])) and full[3] == ones[3]


def test_sort_leaves_out_of_range_ids():
    ids = torch.tensor([[0, 5], [-1, 1], [7, 0]], dtype=torch.int32)     # E = 4: 5, -1 and 7 belong to no expert
    w = torch.tensor([[0.1, 0.2], [0.3, 0.4], [0.5, 0.6]])
    sid, sw, se, nv = O.align_sort(ids, w, 4, 2)
    assert sid.tolist() == [0, 5, 3, 6] and se.tolist() == [0, 1] and nv == 4
    assert sw.tolist()[:2] == pytest.approx([0.1, 0.6]) and sw[3] == 0 and sw[2] == pytest.approx(0.4)
