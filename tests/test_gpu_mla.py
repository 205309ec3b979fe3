"""GPU parity of MLA decode (mla_decode_fwd through the C ABI) against the oracle.

Criterion, from the kernel's arithmetic: the scores are fp32 sums of exact
bf16 x bf16 products, and each softmax weight is rounded to bf16 (relative error
at most 2^-9) before it multiplies the values, the running sum adding the same
rounded weights. The effective weight of row j is then within about 2^-8 of its
exact value, relatively, so |o - o_ref| <= 2^-8 * sum_j p_j |v_j|; the bf16 output
adds 2^-9 |o_ref|. The test allows twice each term (fp32 accumulation, exp2f):
|o - o_ref| <= 2^-7 * sum_j p_j |v_j| + 2^-8 |o_ref| + 1e-6, element by element,
and |lse - lse_ref| <= 2^-8 + 1e-6 |lse_ref| (a rounded-weight sum within 2^-9).
"""
import pytest
import torch

from oracle import mla_oracle as M
from fp8_block_scaled_biased_b200 import binding as B
from fp8_block_scaled_biased_b200 import inputs as I

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device"),
              pytest.mark.filterwarnings("ignore")]

DEV = "cuda"


@pytest.fixture(autouse=True)
def _device_status_clean():
    yield
    assert B.device_status() == 0


def _to(x: I.MlaInputs, dev=DEV):
    return I.MlaInputs(*(t.to(dev) for t in (x.q, x.kv_buffer, x.kv_indptr, x.kv_indices, x.kv_last_page_lens)))


def _run(xd: I.MlaInputs, **kw):
    Bn, Hq = xd.q.shape[0], xd.q.shape[1]
    o = torch.full((Bn, Hq, 512), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((Bn, Hq), float("nan"), dtype=torch.float32, device=DEV)
    B.mla_decode_fwd(xd.q, xd.kv_buffer, o, xd.kv_indptr, xd.kv_indices, xd.kv_last_page_lens, lse=lse, **kw)
    torch.cuda.synchronize()
    return o.cpu().double(), lse.cpu().double()


def _check(x: I.MlaInputs, o, lse, sm_scale=None, logit_cap=0.0):
    ref, ref_lse, mag = M.mla_decode(x.q, x.kv_buffer, x.kv_indptr, x.kv_indices, x.kv_last_page_lens,
                                     sm_scale=sm_scale, logit_cap=logit_cap, return_abs=True)
    bound = 2.0 ** -7 * mag + 2.0 ** -8 * ref.abs() + 1e-6
    d = (o - ref).abs()
    assert torch.isfinite(o).all()
    worst = (d / bound).max().item()
    assert (d <= bound).all(), f"worst |d|/bound {worst:.3f}"
    empty = torch.isneginf(ref_lse)
    assert torch.equal(torch.isneginf(lse), empty)
    assert (o[empty] == 0).all()
    fin = ~empty
    assert ((lse[fin] - ref_lse[fin]).abs() <= 2.0 ** -8 + 1e-6 * ref_lse[fin].abs()).all()
    return worst


RAGGED = I.MlaConfig("mla_ragged_b9_h16", B=9, Hq=16, L=(0, 1, 31, 32, 33, 100, 257, 544, 1000))


@pytest.mark.parametrize("splits", [0, 1, 3, 7])
def test_ragged_lengths_every_element(splits):
    x = I.mla_inputs(RAGGED, spare_pages=5)
    o, lse = _run(_to(x), num_kv_splits=splits)
    _check(x, o, lse)


@pytest.mark.parametrize("page_size,Hq", [(16, 32), (64, 128), (3, 48)])
def test_page_sizes_and_head_counts(page_size, Hq):
    cfg = I.MlaConfig(f"mla_ps{page_size}_h{Hq}", B=5, Hq=Hq, L=(1, 64, 65, 200, 511), page_size=page_size, seed=3)
    x = I.mla_inputs(cfg, spare_pages=2)
    o, lse = _run(_to(x))
    _check(x, o, lse)


def test_sharp_scores_with_soft_cap_and_explicit_scale():
    cfg = I.MlaConfig("mla_sharp", B=4, Hq=16, L=(40, 300, 77, 1), q_std=4.0, seed=5)
    x = I.mla_inputs(cfg)
    xd = _to(x)
    o, lse = _run(xd, sm_scale=0.1)
    _check(x, o, lse, sm_scale=0.1)
    o, lse = _run(xd, sm_scale=0.1, logit_cap=2.0, num_kv_splits=3)
    _check(x, o, lse, sm_scale=0.1, logit_cap=2.0)


@pytest.mark.parametrize("cfg", [I.MLA_DECODE, I.MLA_LONG], ids=lambda c: c.name)
def test_workloads_every_element(cfg):
    """The pages' decode batch (64 sequences of 544 tokens, 16 heads, page size 1) and
    its 8K-context version, every output element against the oracle, in the launch
    configuration the bench times (automatic split count)."""
    x = I.mla_inputs(cfg)
    o, lse = _run(_to(x))
    _check(x, o, lse)


def test_deterministic_and_lse_optional():
    x = I.mla_inputs(RAGGED)
    xd = _to(x)
    o1, l1 = _run(xd, num_kv_splits=4)
    o2, l2 = _run(xd, num_kv_splits=4)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o3 = torch.empty(9, 16, 512, dtype=torch.bfloat16, device=DEV)
    B.mla_decode_fwd(xd.q, xd.kv_buffer, o3, xd.kv_indptr, xd.kv_indices, xd.kv_last_page_lens, num_kv_splits=4)
    assert torch.equal(o3.cpu().double(), o1)


def test_page_table_entry_out_of_range_is_flagged_not_read():
    x = I.mla_inputs(I.MlaConfig("mla_bad", B=2, Hq=16, L=(5, 9)))
    xd = _to(x)
    xd.kv_indices[3] = x.kv_buffer.shape[0] + 1000            # past the buffer
    o = torch.empty(2, 16, 512, dtype=torch.bfloat16, device=DEV)
    B.mla_decode_fwd(xd.q, xd.kv_buffer, o, xd.kv_indptr, xd.kv_indices, xd.kv_last_page_lens)
    torch.cuda.synchronize()
    assert B.device_status() == 32                             # FP8MOE_DEVERR_PAGE, then cleared
    xd.kv_indices[3] = int(x.kv_indices[3])
    xd.kv_last_page_lens[1] = 0                                # a last page must hold >= 1 token
    B.mla_decode_fwd(xd.q, xd.kv_buffer, o, xd.kv_indptr, xd.kv_indices, xd.kv_last_page_lens)
    torch.cuda.synchronize()
    assert B.device_status() == 32
