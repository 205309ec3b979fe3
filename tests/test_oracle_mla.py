"""Pins for the MLA decode oracle.

Each test checks the oracle against something other than itself: a case worked
out by hand, a closed form (zero query, one token), the library softmax, and
invariances the definition fixes (page layout, per-head independence, the value
being the first 512 entries of the key row, the rows past the last page's
length, the score scale, the soft cap).
"""
import math

import pytest
import torch

from oracle import mla_oracle as M
from fp8_block_scaled_biased_b200 import inputs as I

F64 = torch.float64


def _one_sequence(rows: torch.Tensor, page_size: int = 1, order=None):
    """A paged buffer holding one sequence's rows [L, D] (pages in `order`, default as listed)."""
    L, D = rows.shape
    n = (L + page_size - 1) // page_size
    order = list(range(n)) if order is None else list(order)
    kv = torch.full((n, page_size, 1, D), 1e30, dtype=rows.dtype)   # poison the unused slots
    for i, page in enumerate(order):
        chunk = rows[i * page_size:(i + 1) * page_size]
        kv[page, :chunk.shape[0], 0] = chunk
    indptr = torch.tensor([0, n], dtype=torch.int32)
    last = torch.tensor([L - (n - 1) * page_size], dtype=torch.int32)
    return kv, indptr, torch.tensor(order, dtype=torch.int32), last


def test_two_tokens_worked_by_hand():
    # scores 0 and ln 3 -> weights 1/4 and 3/4; lse = ln(1 + 3) = ln 4
    q = torch.tensor([[[1.0, 0.0]]], dtype=F64)                       # B=1, Hq=1, Dk=2
    rows = torch.tensor([[0.0, 5.0], [math.log(3.0), -2.0]], dtype=F64)
    kv, ip, ix, last = _one_sequence(rows)
    o, lse = M.mla_decode(q, kv, ip, ix, last, sm_scale=1.0, v_head_dim=1)
    assert o[0, 0, 0].item() == pytest.approx(0.25 * 0.0 + 0.75 * math.log(3.0), rel=1e-15)
    assert lse[0, 0].item() == pytest.approx(math.log(4.0), rel=1e-15)
    # the second key entry enters the score only through q, which is zero there
    o2, _ = M.mla_decode(q, kv, ip, ix, last, sm_scale=1.0, v_head_dim=2)
    assert o2[0, 0, 1].item() == pytest.approx(0.25 * 5.0 + 0.75 * -2.0, rel=1e-15)


def test_one_token_returns_its_value_row():
    g = torch.Generator().manual_seed(1)
    q = torch.randn(1, 3, 576, generator=g, dtype=F64)
    rows = torch.randn(1, 576, generator=g, dtype=F64)
    kv, ip, ix, last = _one_sequence(rows)
    o, lse = M.mla_decode(q, kv, ip, ix, last)
    for h in range(3):
        assert torch.equal(o[0, h], rows[0, :512])
        assert lse[0, h].item() == pytest.approx((q[0, h] @ rows[0]).item() / 24.0, rel=1e-13)


def test_zero_query_averages_the_values():
    g = torch.Generator().manual_seed(2)
    rows = torch.randn(37, 576, generator=g, dtype=F64)
    kv, ip, ix, last = _one_sequence(rows, page_size=8)
    o, lse = M.mla_decode(torch.zeros(1, 2, 576, dtype=F64), kv, ip, ix, last)
    assert torch.allclose(o[0, 0], rows[:, :512].mean(0), rtol=0, atol=1e-14)
    assert lse[0, 1].item() == pytest.approx(math.log(37.0), rel=1e-15)


def test_matches_library_softmax_with_default_scale():
    g = torch.Generator().manual_seed(3)
    q = torch.randn(1, 4, 576, generator=g, dtype=F64) * 3
    rows = torch.randn(50, 576, generator=g, dtype=F64)
    kv, ip, ix, last = _one_sequence(rows)
    o, lse = M.mla_decode(q, kv, ip, ix, last)
    s = (q[0] @ rows.T) / math.sqrt(576.0)
    assert torch.allclose(o[0], torch.softmax(s, dim=1) @ rows[:, :512], rtol=1e-12, atol=1e-13)
    assert torch.allclose(lse[0], torch.logsumexp(s, dim=1), rtol=1e-14, atol=0)


@pytest.mark.parametrize("page_size", [1, 3, 16, 64])
def test_page_layout_does_not_change_the_result(page_size):
    g = torch.Generator().manual_seed(4)
    q = torch.randn(1, 2, 576, generator=g, dtype=F64)
    rows = torch.randn(45, 576, generator=g, dtype=F64)
    kv0, ip0, ix0, last0 = _one_sequence(rows, page_size=45)            # one page, in order
    o0, l0 = M.mla_decode(q, kv0, ip0, ix0, last0)
    n = (45 + page_size - 1) // page_size
    order = torch.randperm(n, generator=g).tolist()
    kv, ip, ix, last = _one_sequence(rows, page_size=page_size, order=order)
    o, l = M.mla_decode(q, kv, ip, ix, last)
    assert torch.allclose(o, o0, rtol=1e-13, atol=1e-14)
    assert torch.allclose(l, l0, rtol=1e-14, atol=0)


def test_rows_past_the_last_page_length_are_ignored():
    g = torch.Generator().manual_seed(5)
    q = torch.randn(1, 2, 576, generator=g, dtype=F64)
    rows = torch.randn(10, 576, generator=g, dtype=F64)
    kv, ip, ix, last = _one_sequence(rows, page_size=4)                 # last page holds 2
    assert last.item() == 2
    kv[int(ix[-1]), 2:, 0] = 1e6                                         # junk in the unused slots
    o, _ = M.mla_decode(q, kv, ip, ix, last)
    s = (q[0] @ rows.T) / 24.0
    assert torch.allclose(o[0], torch.softmax(s, 1) @ rows[:, :512], rtol=1e-12, atol=1e-13)


def test_value_is_the_first_512_entries_and_rope_entries_only_score():
    g = torch.Generator().manual_seed(6)
    q = torch.randn(1, 2, 576, generator=g, dtype=F64)
    rows = torch.randn(20, 576, generator=g, dtype=F64)
    kv, ip, ix, last = _one_sequence(rows)
    o, _ = M.mla_decode(q, kv, ip, ix, last)
    # with q's last 64 entries zero, the keys' last 64 entries do not matter at all
    q0 = q.clone()
    q0[..., 512:] = 0
    kv2 = kv.clone()
    kv2[..., 512:] = torch.randn(kv2[..., 512:].shape, generator=g, dtype=F64) * 10
    a, _ = M.mla_decode(q0, kv, ip, ix, last)
    b, _ = M.mla_decode(q0, kv2, ip, ix, last)
    assert torch.equal(a, b)
    # with them nonzero, the same change moves the weights (so the output)
    c, _ = M.mla_decode(q, kv2, ip, ix, last)
    assert (c - o).abs().max() > 1e-3


def test_heads_and_sequences_are_independent():
    cfg = I.MlaConfig("t", B=3, Hq=4, L=(7, 1, 12), page_size=4)
    x = I.mla_inputs(cfg)
    o, lse = M.mla_decode(x.q, x.kv_buffer, x.kv_indptr, x.kv_indices, x.kv_last_page_lens)
    for b in range(3):
        ip = torch.tensor([0, int(x.kv_indptr[b + 1] - x.kv_indptr[b])], dtype=torch.int32)
        ix = x.kv_indices[int(x.kv_indptr[b]):int(x.kv_indptr[b + 1])]
        for h in (0, 3):
            ob, lb = M.mla_decode(x.q[b:b + 1, h:h + 1], x.kv_buffer, ip, ix, x.kv_last_page_lens[b:b + 1])
            assert torch.equal(ob[0, 0], o[b, h])
            assert lb[0, 0].item() == lse[b, h].item()


def test_score_scale_and_soft_cap():
    g = torch.Generator().manual_seed(7)
    q = torch.randn(1, 2, 576, generator=g, dtype=F64)
    rows = torch.randn(30, 576, generator=g, dtype=F64)
    kv, ip, ix, last = _one_sequence(rows)
    # sm_scale multiplies the score: scaling q by 2 and sm_scale by 1/2 changes nothing
    a, la = M.mla_decode(q, kv, ip, ix, last, sm_scale=0.1)
    b, lb = M.mla_decode(2 * q, kv, ip, ix, last, sm_scale=0.05)
    assert torch.allclose(a, b, rtol=1e-13, atol=1e-14) and torch.allclose(la, lb, rtol=1e-14)
    # a huge cap is no cap; a cap c gives the softmax of c*tanh(s/c)
    c, _ = M.mla_decode(q, kv, ip, ix, last, sm_scale=0.1, logit_cap=1e9)
    assert torch.allclose(c, a, rtol=1e-12, atol=1e-13)
    d, ld = M.mla_decode(q, kv, ip, ix, last, sm_scale=0.1, logit_cap=1.5)
    s = 1.5 * torch.tanh(0.1 * (q[0] @ rows.T) / 1.5)
    assert torch.allclose(d[0], torch.softmax(s, 1) @ rows[:, :512], rtol=1e-12, atol=1e-13)
    assert torch.allclose(ld[0], torch.logsumexp(s, 1), rtol=1e-14)


def test_empty_sequence_and_lengths():
    cfg = I.MlaConfig("t", B=3, Hq=2, L=(0, 5, 8), page_size=4)
    x = I.mla_inputs(cfg)
    assert M.sequence_lengths(x.kv_indptr, x.kv_last_page_lens, 4) == [0, 5, 8]
    o, lse = M.mla_decode(x.q, x.kv_buffer, x.kv_indptr, x.kv_indices, x.kv_last_page_lens)
    assert torch.equal(o[0], torch.zeros_like(o[0])) and torch.isneginf(lse[0]).all()
    assert torch.isfinite(lse[1:]).all()


def test_weighted_magnitude_bounds_the_output():
    cfg = I.MlaConfig("t", B=2, Hq=3, L=(9, 33), page_size=1)
    x = I.mla_inputs(cfg)
    o, _, mag = M.mla_decode(x.q, x.kv_buffer, x.kv_indptr, x.kv_indices, x.kv_last_page_lens, return_abs=True)
    assert (o.abs() <= mag + 1e-15).all()
    # a positive value column: the magnitude is the output itself
    x.kv_buffer[..., 0] = x.kv_buffer[..., 0].abs()
    o, _, mag = M.mla_decode(x.q, x.kv_buffer, x.kv_indptr, x.kv_indices, x.kv_last_page_lens, return_abs=True)
    assert torch.allclose(o[..., 0], mag[..., 0], rtol=1e-14, atol=0)


def test_inputs_page_table_is_a_partition():
    cfg = I.MlaConfig("t", B=4, Hq=16, L=(1, 64, 65, 0), page_size=16)
    x = I.mla_inputs(cfg, spare_pages=3)
    assert x.kv_buffer.shape == (1 + 4 + 5 + 0 + 3, 16, 1, 576)
    assert x.kv_indptr.tolist() == [0, 1, 5, 10, 10]
    assert x.kv_last_page_lens.tolist() == [1, 16, 1, 0]
    idx = x.kv_indices.tolist()
    assert len(set(idx)) == len(idx) == 10 and all(0 <= i < 13 for i in idx)
