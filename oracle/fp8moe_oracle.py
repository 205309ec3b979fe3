"""CPU oracle for the FP8 block-scaled biased MoE layer.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links
this module: only the tests, the smoke check in __graft_entry__ and bench.py's
CPU-baseline leg do. It shares no code with the CUDA library and never reads a
value the CUDA library produced.

It is a plain, slow, step-by-step statement of what the layer computes, written
from "Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang"
(rocm.blogs.amd.com), sections "Complete MoE Implementation" (Top-K routing,
MoE Sorting, Blockscale FP8 MoE Computation) and "General Linear Layer"
(FP8 blockscale GEMM), with the FP8 format fixed to OCP E4M3 "fn" (max 448) as
opposed to the MI300X "fnuz" variant that the zaynews.com article on running V4
Flash on one MI300X describes. Where the pages leave a step open, the reading
taken is stated at the function. Floating point is fp64 unless the step decides
an integer (a routing choice, an FP8 code), in which case that decision is taken
in fp32, the precision the kernels use, one IEEE-rounded operation at a time.

Library primitives used as steps: torch CPU matmul (fp64), stable sort, exp.
Every function is pinned by tests/test_oracle_*.py against something other than
itself (brute force, closed forms, library routines, invariants).
"""
from __future__ import annotations

import math

import torch

F32 = torch.float32
F64 = torch.float64

FP8_E4M3FN_MAX = 448.0      # OCP E4M3 "fn": largest finite magnitude, S.1111.110
QUANT_GROUP = 128           # 1x128 activation groups and 128x128 weight blocks


# ---------------------------------------------------------------------------
# OCP FP8 E4M3 ("fn") codec
# ---------------------------------------------------------------------------

def _e4m3_value_of_code(c: torch.Tensor) -> torch.Tensor:
    """OCP E4M3: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no
    infinities; exponent field 0 holds subnormals m/8 * 2^-6; S.1111.111 is NaN."""
    sign = torch.where((c >> 7) == 1, -1.0, 1.0).to(F64)
    exp = (c >> 3) & 0xF
    man = (c & 0x7).to(F64)
    normal = (1.0 + man / 8.0) * torch.pow(torch.tensor(2.0, dtype=F64), (exp - 7).to(F64))
    sub = (man / 8.0) * 2.0 ** -6
    val = torch.where(exp == 0, sub, normal) * sign
    return torch.where((exp == 0xF) & ((c & 7) == 7), torch.tensor(float("nan"), dtype=F64), val)


_E4M3_TABLE = _e4m3_value_of_code(torch.arange(256, dtype=torch.int64))


def e4m3_decode(codes: torch.Tensor) -> torch.Tensor:
    """Value of each FP8 E4M3fn code, in fp64 (looked up in the 256-entry table above)."""
    return _E4M3_TABLE[codes.to(torch.int64) & 0xFF]


def e4m3_encode(x: torch.Tensor) -> torch.Tensor:
    """Round fp32 values to E4M3fn codes: round-to-nearest-even, saturating to +-448.

    Magnitudes above 448 (and +-inf) become +-448 (code 0x7E/0xFE), which is the
    "satfinite" conversion; NaN becomes 0x7F. For |x| in [2^e, 2^(e+1)) with
    e >= -6 the grid step is 2^(e-3); below 2^-6 it is the subnormal step 2^-9.
    Each value is scaled by 1/step (a power of two: exact in fp32), rounded to an
    integer half to even (the only rounding), and the code is assembled from
    that integer and e.
    """
    x = x.to(F32)
    sign = torch.signbit(x).to(torch.int32) << 7
    a = x.abs()
    # e = floor(log2(a)) read from the fp32 exponent field (subnormal fp32 inputs
    # are far below the FP8 range and fall in the e < -6 branch either way)
    e = ((a.view(torch.int32) >> 23) & 0xFF) - 127
    e_grid = torch.clamp(e, min=-6, max=8)
    inv_step = ((3 - e_grid + 127) << 23).view(F32)        # 2^(3 - e_grid), exact
    n = torch.round(a * inv_step).to(torch.int32)          # 0..16 (16 = carry into next binade)
    carry = n == 16
    e_grid = torch.where(carry, e_grid + 1, e_grid)
    n = torch.where(carry, torch.full_like(n, 8), n)
    is_sub = n < 8                                          # only possible when e_grid == -6
    code = torch.where(is_sub, n, ((e_grid + 7) << 3) | (n - 8))
    code = torch.where(a > FP8_E4M3FN_MAX, torch.full_like(code, 0x7E), code)
    code = code | sign
    code = torch.where(torch.isnan(x), torch.full_like(code, 0x7F), code)
    return code.to(torch.uint8)


# ---------------------------------------------------------------------------
# Dynamic FP8 quantisation: 1x128 activation groups, 128x128 weight blocks
# ---------------------------------------------------------------------------

def _quant_with_scale(vals_f32: torch.Tensor, scale_f32: torch.Tensor) -> torch.Tensor:
    """q = E4M3fn(x / scale) with the division in fp32; q = 0 where scale == 0."""
    safe = torch.where(scale_f32 == 0, torch.ones_like(scale_f32), scale_f32)
    q = e4m3_encode(vals_f32 / safe)                        # fp32 / fp32: one IEEE rounding
    return torch.where(scale_f32 == 0, torch.zeros_like(q), q)


def quant_1x128(x: torch.Tensor):
    """Per-token-group FP8 quantisation of x [M, K] (groups of 128 along K).

    Returns q uint8 [M, K] (E4M3fn codes) and scales fp32 [M, ceil(K/128)]
    (row-major; the MoE call takes the transpose).

    Follows the page's section "Blockscale FP8 MoE Computation" (hidden states
    viewed as [M*H/128, 128], one scale per 128 values, then
    dynamic_per_token_scaled_fp8_quant) and "General Linear Layer" (one scale per
    1x128 activation block). The formula is not printed; the reading taken is
    scale = amax / 448 in fp32 and q = RNE-satfinite(x / scale), an all-zero
    group giving scale 0 and codes 0. A last group shorter than 128 uses its
    valid elements only.
    """
    x = x.to(F32)
    M, K = x.shape
    KB = (K + QUANT_GROUP - 1) // QUANT_GROUP
    q = torch.empty(M, K, dtype=torch.uint8)
    scales = torch.empty(M, KB, dtype=F32)
    for kb in range(KB):
        cols = slice(kb * QUANT_GROUP, min(K, (kb + 1) * QUANT_GROUP))
        vals = x[:, cols]
        amax = vals.abs().amax(dim=1, keepdim=True)         # exact in fp32
        scale = amax / torch.tensor(FP8_E4M3FN_MAX, dtype=F32)   # fp32 IEEE division
        q[:, cols] = _quant_with_scale(vals, scale)
        scales[:, kb] = scale[:, 0]
    return q, scales


def quant_128x128(w: torch.Tensor):
    """Per-block FP8 quantisation of a weight matrix w [N, K] in 128x128 blocks.

    Returns q uint8 [N, K] and scales fp32 [ceil(N/128), ceil(K/128)], with
    scale = amax / 448 over the block (fp32) and q = RNE-satfinite(w / scale).
    The dequantised weight is q * scale: the pages' "*_weight_scale_inv" tensors
    are multipliers. Edge blocks use their valid elements.
    """
    w = w.to(F32)
    N, K = w.shape
    NB = (N + QUANT_GROUP - 1) // QUANT_GROUP
    KB = (K + QUANT_GROUP - 1) // QUANT_GROUP
    # pad to whole blocks with zeros (zeros never raise an amax)
    wp = torch.zeros(NB * QUANT_GROUP, KB * QUANT_GROUP, dtype=F32)
    wp[:N, :K] = w
    blocks = wp.view(NB, QUANT_GROUP, KB, QUANT_GROUP)
    amax = blocks.abs().amax(dim=(1, 3))                    # [NB, KB]
    scales = amax / torch.tensor(FP8_E4M3FN_MAX, dtype=F32)
    sfull = scales[:, None, :, None].expand_as(blocks)
    q = _quant_with_scale(blocks, sfull).reshape(NB * QUANT_GROUP, KB * QUANT_GROUP)[:N, :K]
    return q.contiguous(), scales


def dequant_rows(q: torch.Tensor, scales: torch.Tensor, block_rows: int) -> torch.Tensor:
    """fp64 value of a quantised matrix: dec(q[r, k]) * scales[r // block_rows, k // 128]."""
    R, K = q.shape
    ridx = torch.arange(R) // block_rows
    kidx = torch.arange(K) // QUANT_GROUP
    return e4m3_decode(q) * scales.to(F64)[ridx][:, kidx]


# ---------------------------------------------------------------------------
# Block-scaled FP8 GEMM
# ---------------------------------------------------------------------------

def blockscale_gemm(qa: torch.Tensor, sa: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor) -> torch.Tensor:
    """C[m, n] = sum_kb sa[m, kb] * sb[n // 128, kb] * S_kb[m, n], in fp64.

    S_kb = sum over the 128 k of block kb of dec(qa[m, k]) * dec(qb[n, k]).
    qa [M, K] with per-row 1x128 scales sa [M, ceil(K/128)]; qb [N, K] with
    128x128 block scales sb [ceil(N/128), ceil(K/128)]; Y = XQ * WQ^T as in the
    page's section "General Linear Layer" (gemm_a8w8_blockscale(XQ, WQ, x_scale,
    w_scale)). Every E4M3 value is a multiple of 2^-9 and |S_kb| <= 128*448^2,
    so S_kb is exact in fp64 whatever the summation order; the scales are then
    applied and the blocks summed in fp64.
    """
    M, K = qa.shape
    N = qb.shape[0]
    A = e4m3_decode(qa)
    B = e4m3_decode(qb)
    KB = (K + QUANT_GROUP - 1) // QUANT_GROUP
    nblk = torch.arange(N) // QUANT_GROUP
    C = torch.zeros(M, N, dtype=F64)
    for kb in range(KB):
        cols = slice(kb * QUANT_GROUP, min(K, (kb + 1) * QUANT_GROUP))
        S = A[:, cols] @ B[:, cols].T
        f = sa[:, kb].to(F64)[:, None] * sb[nblk, kb].to(F64)[None, :]
        C += f * S
    return C


def bf16_round(x: torch.Tensor) -> torch.Tensor:
    """Round fp64 values to bfloat16 (8 significant bits, round half to even), once.

    Returned as fp64 holding the bf16 value. bf16 shares fp32's exponent range:
    the quantum is 2^(e-7) for x in [2^e, 2^(e+1)), and 2^-133 below 2^-126.
    Magnitudes that round above the largest bf16 become inf.
    """
    x = x.to(F64)
    a = x.abs()
    _, k = torch.frexp(torch.where(a > 0, a, torch.ones_like(a)))
    e = (k - 1).to(torch.int64)
    quantum = torch.pow(torch.tensor(2.0, dtype=F64), (torch.clamp(e, min=-126) - 7).to(F64))
    r = torch.round(a / quantum) * quantum
    bf16_max = (2.0 - 2.0 ** -7) * 2.0 ** 127
    r = torch.where(r > bf16_max, torch.tensor(float("inf"), dtype=F64), r)
    return torch.where(torch.signbit(x), -r, r)


# ---------------------------------------------------------------------------
# Routing: sigmoid + correction bias, group-limited top-k
# ---------------------------------------------------------------------------

# fp32 constants of the exponential below (Cody & Waite argument reduction,
# "Software Manual for the Elementary Functions", 1980; Taylor series for e^r).
_LOG2E = 1.4426950408889634          # rounded to fp32 where used
_LN2_HI = 0.693359375                # 355/512: n * _LN2_HI is exact for |n| < 2^14
_LN2_LO = -2.1219444005469057e-4     # ln 2 - _LN2_HI, rounded to fp32
_TAYLOR = [1.0 / math.factorial(k) for k in range(8)]   # 1/k!, k = 0..7, rounded to fp32
EXP_ARG_MIN = -87.0
EXP_ARG_MAX = 88.0


def exp_f32(y: torch.Tensor) -> torch.Tensor:
    """e^y in fp32 by a fixed sequence of IEEE fp32 operations (one rounding each).

    Reading: the pages do not say how the routing score is computed bit by bit,
    and bit-exact expert ids need the same fp32 score on the CPU and the GPU.
    This is the recipe both sides implement, each in its own code:
      y <- clamp(y, -87, 88)
      n <- round_half_even(y * log2e)
      r <- (y - n * LN2_HI) - n * LN2_LO
      p <- Horner with c7..c0 = 1/7!..1/0!: p = c7; p = p*r + c_k (multiply,
           then add; no fused multiply-add)
      e^y = p * 2^n
    """
    t32 = lambda v: torch.tensor(v, dtype=F32)
    y = torch.clamp(y.to(F32), EXP_ARG_MIN, EXP_ARG_MAX)
    n = torch.round(y * t32(_LOG2E))                         # fp32 multiply, then half-even
    r = y - n * t32(_LN2_HI)                                 # product exact
    r = r - n * t32(_LN2_LO)
    p = t32(_TAYLOR[7]).expand_as(r).clone()
    for k in range(6, -1, -1):
        p = p * r                                            # rounded to fp32
        p = p + t32(_TAYLOR[k])                              # rounded to fp32
    two_n = ((n.to(torch.int32) + 127) << 23).view(F32)      # 2^n, n in [-126, 127]
    return p * two_n


def sigmoid_f32(x: torch.Tensor) -> torch.Tensor:
    """s = 1 / (1 + e^-x) in fp32, with exp_f32, an fp32 add and an fp32 division."""
    one = torch.tensor(1.0, dtype=F32)
    return one / (one + exp_f32(-x.to(F32)))


def biased_grouped_topk(logits: torch.Tensor, bias: torch.Tensor, topk: int,
                        num_expert_group: int, topk_group: int,
                        need_renorm: bool, routed_scaling_factor: float):
    """Biased grouped top-k routing of logits [T, E] with correction bias [E].

    From the page's section "Top-K routing": each token keeps a fixed number of
    expert groups (topk_group of num_expert_group) and picks its top-k experts
    inside them; outputs are fp32 weights and int32 ids [T, topk]; the weights
    are multiplied by routed_scaling_factor. The pages do not give the scoring;
    the readings taken (DeepSeek-V3 style) are:
      s = sigmoid(logit), b = s + bias (fp32); the bias steers selection only;
      group score = sum of the two largest b of the group (fp32 add);
      groups ranked by (score desc, group index asc), keep topk_group;
      experts of kept groups ranked by (b desc, expert index asc), keep topk,
      in that rank order;
      w = s of the chosen experts; if need_renorm, w /= (w_0 + ... + w_{k-1})
      summed left to right in fp32 (left as is if that sum is 0); then
      w *= routed_scaling_factor (fp32).
    """
    logits = logits.to(F32)
    T, E = logits.shape
    G = num_expert_group
    per = E // G
    s = sigmoid_f32(logits)
    b = s + bias.to(F32)[None, :]
    bg = b.view(T, G, per)
    top = torch.sort(bg, dim=2, descending=True, stable=True).values
    gscore = top[:, :, 0] + top[:, :, 1] if per >= 2 else top[:, :, 0]
    gorder = torch.sort(gscore, dim=1, descending=True, stable=True).indices[:, :topk_group]
    gmask = torch.zeros(T, G, dtype=torch.bool)
    gmask.scatter_(1, gorder, True)
    emask = gmask[:, :, None].expand(T, G, per).reshape(T, E)
    bm = torch.where(emask, b, torch.tensor(float("-inf"), dtype=F32))
    ids = torch.sort(bm, dim=1, descending=True, stable=True).indices[:, :topk]
    w = torch.gather(s, 1, ids)
    if need_renorm:
        denom = w[:, 0].clone()
        for j in range(1, topk):
            denom = denom + w[:, j]
        safe = torch.where(denom == 0, torch.ones_like(denom), denom)
        w = torch.where(denom[:, None] == 0, w, w / safe[:, None])
    w = w * torch.tensor(routed_scaling_factor, dtype=F32)
    return w.contiguous(), ids.to(torch.int32).contiguous()


# ---------------------------------------------------------------------------
# MoE align / sort
# ---------------------------------------------------------------------------

def align_sort(topk_ids: torch.Tensor, topk_weights: torch.Tensor, num_experts: int, block_m: int,
               expert_mask: torch.Tensor | None = None):
    """Group the T*topk token-expert pairs by expert into block_m-padded segments.

    From the page's section "MoE Sorting" (moe_sorting returns sorted_token_ids,
    sorted_weight_buf, sorted_expert_ids and num_valid_ids). The layout is not
    printed; the reading taken: a pair (t, k) is named by its flat id
    p = t*topk + k; experts in ascending order, each expert's pairs in ascending
    p, each segment padded to a multiple of block_m with the sentinel id T*topk
    and weight 0; experts with no pair get no block; one expert id per block;
    num_valid_ids = total padded length. Ids outside [0, num_experts) belong to
    no expert and are left out. expert_mask (the expert_mask argument of the
    page's asm_moe call, the experts one GPU holds under expert parallelism):
    when given, experts e with expert_mask[e] == 0 are left out with their pairs.

    Returns (sorted_ids int32 [L], sorted_weights fp32 [L], sorted_expert_ids
    int32 [L/block_m], num_valid_ids int).
    """
    T, K = topk_ids.shape
    P = T * K
    flat = topk_ids.reshape(-1).to(torch.int64)
    wflat = topk_weights.reshape(-1).to(F32)
    ids_out, w_out, blocks = [], [], []
    for e in range(num_experts):
        if expert_mask is not None and int(expert_mask[e]) == 0:
            continue
        pairs = torch.nonzero(flat == e).flatten()          # ascending p
        cnt = pairs.numel()
        if cnt == 0:
            continue
        padded = -(-cnt // block_m) * block_m
        ids_out.append(torch.cat([pairs, torch.full((padded - cnt,), P, dtype=torch.int64)]))
        w_out.append(torch.cat([wflat[pairs], torch.zeros(padded - cnt, dtype=F32)]))
        blocks.append(torch.full((padded // block_m,), e, dtype=torch.int64))
    sorted_ids = torch.cat(ids_out).to(torch.int32) if ids_out else torch.empty(0, dtype=torch.int32)
    sorted_w = torch.cat(w_out) if w_out else torch.empty(0, dtype=F32)
    sorted_e = torch.cat(blocks).to(torch.int32) if blocks else torch.empty(0, dtype=torch.int32)
    return sorted_ids, sorted_w, sorted_e, int(sorted_ids.numel())


def align_sort_capacity(T: int, topk: int, num_experts: int, block_m: int) -> int:
    """Largest padded length: every pair plus at most block_m - 1 pad slots per expert."""
    return T * topk + num_experts * (block_m - 1)


# ---------------------------------------------------------------------------
# The fused g1u1 MoE computation
# ---------------------------------------------------------------------------

def silu(z: torch.Tensor) -> torch.Tensor:
    """silu(z) = z / (1 + e^-z) in fp64."""
    z = z.to(F64)
    return z / (1.0 + torch.exp(-z))


def expert_intermediate(a8_rows, a_scale_rows, w1q, w1s):
    """The first half of one expert: the re-quantised intermediate (a2 codes [rows, I],
    scales fp32 [rows, I/128]) that the second GEMM takes.

    From the page's section "Blockscale FP8 MoE Computation" (g1u1: w1 holds gate
    and up, w2.shape[2] * 2 == w1.shape[1]; activation silu). Readings: w1 rows
    [0, I) are gate and [I, 2I) are up; GEMM1 stays fp64 (no rounding before the
    activation); h = silu(gate) * up in fp64, rounded to fp32 and re-quantised per
    row in 1x128 groups along I by quant_1x128 (the second GEMM's activation
    quantisation is not printed; it is taken to be the same dynamic recipe as the
    first).
    """
    I = w1q.shape[0] // 2
    g1 = blockscale_gemm(a8_rows, a_scale_rows, w1q, w1s)
    h = silu(g1[:, :I]) * g1[:, I:]
    return quant_1x128(h.to(F32))


def expert_ffn(a8_rows, a_scale_rows, w1q, w1s, w2q, w2s):
    """One expert applied to quantised token rows; returns y [rows, H] in fp64:
    expert_intermediate, then GEMM2 = blockscale_gemm(a2, s2, w2q, w2s) (same page
    section)."""
    a2, s2 = expert_intermediate(a8_rows, a_scale_rows, w1q, w1s)
    return blockscale_gemm(a2, s2, w2q, w2s)


def moe_combine(y_slots: torch.Tensor, topk_weights: torch.Tensor) -> torch.Tensor:
    """out[t] = sum over k = 0..topk-1, in that order, of w[t, k] * y[t, k, :] in fp64.

    y_slots [T, topk, H]; the weighted sum of the experts' outputs ("moe_buf" in
    the page). Returned unrounded (fp64); bf16_round gives the bf16 output.
    """
    T, K, H = y_slots.shape
    out = torch.zeros(T, H, dtype=F64)
    for k in range(K):
        out = out + topk_weights[:, k].to(F64)[:, None] * y_slots[:, k, :]
    return out


def moe_layer(a8, a_scale, topk_ids, topk_weights, get_expert, tokens=None, round_bf16=True, expert_mask=None):
    """Fused g1u1 MoE of quantised hidden states a8 [T, H] (scales [T, H/128]).

    get_expert(e) -> (w1q [2I, H], w1s [2I/128, H/128], w2q [H, I], w2s [H/128, I/128])
    supplies expert e's quantised weights (so that large layers can be streamed).
    tokens: optional sorted list of token indices to compute (others are skipped);
    the result then has one row per listed token.
    expert_mask: optional [E]; when given, only pairs whose id e lies in [0, E)
    with expert_mask[e] != 0 contribute (the others add nothing), which is the
    partial output of one expert-parallel rank.
    Output: bf16-rounded (fp64 tensor of bf16 values) or unrounded fp64.
    """
    T, K = topk_ids.shape
    tok = torch.arange(T) if tokens is None else torch.as_tensor(tokens, dtype=torch.int64)
    ids = topk_ids[tok].to(torch.int64)
    H = a8.shape[1]
    y = torch.zeros(len(tok), K, H, dtype=F64)
    for e in torch.unique(ids).tolist():
        if expert_mask is not None and not (0 <= e < len(expert_mask) and int(expert_mask[e]) != 0):
            continue
        rows, slots = torch.nonzero(ids == e, as_tuple=True)
        w1q, w1s, w2q, w2s = get_expert(e)
        t = tok[rows]
        y[rows, slots] = expert_ffn(a8[t], a_scale[t], w1q, w1s, w2q, w2s)
    out = moe_combine(y, topk_weights[tok])
    return bf16_round(out) if round_bf16 else out
