"""CPU oracle for multi-head latent attention (MLA) at decode.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links
this module: only the tests, the smoke check in __graft_entry__ and bench.py's
CPU-baseline leg do. It shares no code with the CUDA library and never reads a
value the CUDA library produced.

What it computes follows "Accelerate DeepSeek-R1 Inference: Integrate AITER
into SGLang" (rocm.blogs.amd.com), section "Attention Mechanisms", subsection
"MLA For Decode": the decode call takes the queries q [batch, heads, 576], a
paged latent KV buffer viewed as [pages, page_size, 1, 576] (one KV head shared
by every query head), the page table (kv_indptr, kv_indices), the number of
tokens held by each sequence's last page (kv_last_page_lens), sm_scale (by
default one over the square root of the 576-wide query/key head) and logit_cap,
and writes o [batch, heads, 512]: with weights absorbed, the values are the
first 512 entries (the latent part) of the same rows that serve as keys.

Readings taken where the section is silent:
  * sequence b's tokens are the rows of its pages kv_indices[kv_indptr[b] ..
    kv_indptr[b+1]) in list order; every page is full except the last, which
    holds kv_last_page_lens[b] tokens (the section fills that array with ones
    for a page size of 1);
  * the score of token j is s_j = sm_scale * <q, k_j> over all 576 entries; a
    positive logit_cap bounds it as logit_cap * tanh(s_j / logit_cap) (the soft
    cap of the SGLang decode kernel the call plugs into); zero leaves it alone;
  * o = sum_j softmax(s)_j v_j, and the log-sum-exp lse = log sum_j exp(s_j)
    (the per-split partials the section's call returns reduce to these);
  * a sequence with no token gets o = 0 and lse = -inf.
Arithmetic is fp64 on the exact values of the (bf16) inputs; exp and log are
the library's. Pinned by tests/test_oracle_mla.py (hand-computed cases, closed
forms, invariances and a library softmax).
"""
from __future__ import annotations

import math

import torch

F64 = torch.float64

QK_HEAD_DIM = 576       # 512 latent + 64 rotary entries per query/key row
V_HEAD_DIM = 512        # the latent part, used as the value


def sequence_rows(kv_buffer: torch.Tensor, kv_indptr, kv_indices, kv_last_page_lens, b: int) -> torch.Tensor:
    """The KV rows of sequence b in token order, [L_b, D] (fp64)."""
    page_size = kv_buffer.shape[1]
    lo, hi = int(kv_indptr[b]), int(kv_indptr[b + 1])
    rows = []
    for i in range(lo, hi):
        page = int(kv_indices[i])
        n = page_size if i < hi - 1 else int(kv_last_page_lens[b])
        rows.append(kv_buffer[page, :n, 0, :].to(F64))
    if not rows:
        return torch.zeros(0, kv_buffer.shape[-1], dtype=F64)
    return torch.cat(rows, 0)


def mla_decode(q: torch.Tensor, kv_buffer: torch.Tensor, kv_indptr, kv_indices, kv_last_page_lens,
               sm_scale: float | None = None, logit_cap: float = 0.0, v_head_dim: int = V_HEAD_DIM,
               return_abs: bool = False):
    """o [B, Hq, Dv] and lse [B, Hq] in fp64 (and, with return_abs, sum_j p_j |v_j| [B, Hq, Dv]:
    the softmax-weighted magnitude that bounds how far a rounded weight can move o).

    q: [B, Hq, Dk]; kv_buffer: [pages, page_size, 1, Dk]; Dv <= Dk."""
    B, Hq, Dk = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(Dk)
    o = torch.zeros(B, Hq, v_head_dim, dtype=F64)
    lse = torch.full((B, Hq), -math.inf, dtype=F64)
    mag = torch.zeros(B, Hq, v_head_dim, dtype=F64)
    for b in range(B):
        rows = sequence_rows(kv_buffer, kv_indptr, kv_indices, kv_last_page_lens, b)
        if rows.shape[0] == 0:
            continue
        keys = rows[:, :Dk]
        values = rows[:, :v_head_dim]
        s = sm_scale * (q[b].to(F64) @ keys.T)                  # [Hq, L]
        if logit_cap > 0:
            s = logit_cap * torch.tanh(s / logit_cap)
        m = s.max(dim=1, keepdim=True).values
        e = torch.exp(s - m)
        den = e.sum(dim=1, keepdim=True)
        p = e / den
        o[b] = p @ values
        lse[b] = m[:, 0] + torch.log(den[:, 0])
        if return_abs:
            mag[b] = p @ values.abs()
    if return_abs:
        return o, lse, mag
    return o, lse


def sequence_lengths(kv_indptr, kv_last_page_lens, page_size: int) -> list[int]:
    """L_b = (pages_b - 1) * page_size + last_len_b (0 for a sequence with no page)."""
    out = []
    for b in range(len(kv_last_page_lens)):
        n = int(kv_indptr[b + 1]) - int(kv_indptr[b])
        out.append(0 if n == 0 else (n - 1) * page_size + int(kv_last_page_lens[b]))
    return out
