"""Shared pieces of the GPU parity tests: oracle-side expert weights, the token
selections of the full-size comparisons and the output criterion. The oracle
always quantises raw weights itself; raw weights drawn on the device by the
input generator are copied to the host for it."""
import torch

from oracle import fp8moe_oracle as O
from fp8_block_scaled_biased_b200 import inputs as I

# Oracle-quantised experts, kept for the whole test session: the decode, prefill
# and skewed layers (and their expert- and tensor-parallel variants) share one
# weight set, and quantising an expert on the host is the slowest step of their
# oracle. The cache stops growing before it would take half the host memory that
# was free when it started.
_EXPERTS = {}
_BUDGET = None


def _cache_budget():
    global _BUDGET
    if _BUDGET is None:
        try:
            import psutil
            _BUDGET = psutil.virtual_memory().available // 2
        except Exception:  # noqa: BLE001 - without psutil nothing is cached
            _BUDGET = 0
    return _BUDGET


def _expert_bytes(cfg):
    return 3 * cfg.I * cfg.H + 4 * (3 * cfg.I * cfg.H // (128 * 128))


def oracle_expert(cfg, e, device="cuda"):
    """Oracle-quantised weights of expert e from the same raw numbers the device layer used."""
    key = (cfg.seed, cfg.H, cfg.I, cfg.w_std, e, str(device))
    hit = _EXPERTS.get(key)
    if hit is not None:
        return hit
    w1 = I.expert_weight_raw(cfg, "w1", e, device).cpu()
    w2 = I.expert_weight_raw(cfg, "w2", e, device).cpu()
    q1, s1 = O.quant_128x128(w1)
    q2, s2 = O.quant_128x128(w2)
    val = (q1, s1, q2, s2)
    if (len(_EXPERTS) + 1) * _expert_bytes(cfg) <= _cache_budget():
        _EXPERTS[key] = val
    return val


def moe_error(gpu_out: torch.Tensor, ref: torch.Tensor):
    """(max |gpu - ref|, its bound 2e-2 * max|ref| + 1e-3, mean relative error sum|d| / sum|ref|)."""
    g = gpu_out.double().cpu()
    r = ref.double().cpu()
    d = (g - r).abs()
    return d.max().item(), 2e-2 * r.abs().max().item() + 1e-3, (d.sum() / r.abs().sum().clamp_min(1e-300)).item()


def assert_moe_close(gpu_out, ref):
    dmax, bound, mre = moe_error(gpu_out, ref)
    assert dmax <= bound, f"max |gpu-ref| = {dmax:.3e} > {bound:.3e}"
    assert mre <= 5e-3, f"mean relative error {mre:.3e} > 5e-3"
    return dmax, mre


def oracle_moe_rows(cfg, act, tokens, device="cuda", expert_mask=None):
    """Oracle routing on all tokens, then the MoE output of the listed tokens (fp64, unrounded).
    expert_mask (CPU int32 [E]): only the kept experts' pairs contribute."""
    w, ids = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    a8, asc = O.quant_1x128(act.x[tokens] if tokens is not None else act.x)
    sub_ids = ids[tokens] if tokens is not None else ids
    sub_w = w[tokens] if tokens is not None else w
    out = O.moe_layer(a8, asc, sub_ids, sub_w, lambda e: oracle_expert(cfg, e, device), round_bf16=False,
                      expert_mask=expert_mask)
    return out, w, ids


def tokens_of_expert(ids_ref, e):
    """Tokens (ascending) that the oracle's routing sends to expert e."""
    return torch.nonzero((ids_ref == e).any(dim=1)).flatten()


def m64_tail_expert(ids_ref, E, block_m=128, expert_mask=None):
    """An expert whose last row block holds at most block_m/2 pairs (the GEMMs run that
    block as an M=64 tile): the least-loaded one that also fills a whole block before its
    tail, else the least-loaded one with such a tail; taken from the oracle's routing.
    None if there is none."""
    counts = torch.bincount(ids_ref.flatten().long(), minlength=E)
    best = None
    for e in range(E):
        c = int(counts[e])
        if expert_mask is not None and int(expert_mask[e]) == 0:
            continue
        if 0 < c % block_m <= block_m // 2:
            key = (c < block_m, c)                       # multi-block experts first, then fewest pairs
            if best is None or key < best[0]:
                best = (key, e)
    return None if best is None else best[1]


def full_size_tokens(cfg, ids_ref, n_random, seed, most_loaded=True, m64_tail=True, expert_mask=None):
    """The token selection of a full-size comparison, chosen from the oracle's routing:
    n_random seeded tokens, the first and last token, every token of the most-loaded expert
    and every token of an M=64-tail expert. Returns (tokens, {role: expert})."""
    g = torch.Generator().manual_seed(seed)
    parts = [torch.randperm(cfg.T, generator=g)[: min(n_random, cfg.T)], torch.tensor([0, cfg.T - 1])]
    roles = {}
    flat = ids_ref.flatten().long()
    if expert_mask is not None:
        flat = flat[expert_mask.bool()[flat]]
    counts = torch.bincount(flat, minlength=cfg.E)
    if most_loaded:
        roles["most_loaded"] = int(counts.argmax())
        parts.append(tokens_of_expert(ids_ref, roles["most_loaded"]))
    if m64_tail:
        e = m64_tail_expert(ids_ref, cfg.E, expert_mask=expert_mask)
        if e is not None:
            roles["m64_tail"] = e
            parts.append(tokens_of_expert(ids_ref, e))
    return torch.unique(torch.cat(parts)), roles


def blocks_covered(ids_ref, tokens, E, block_m=128, expert_mask=None):
    """(row blocks holding at least one pair of the listed tokens, row blocks in all), for the
    sorted layout of the oracle's routing."""
    sid, _, _, nv = O.align_sort(ids_ref, torch.ones_like(ids_ref, dtype=torch.float32), E, block_m,
                                 expert_mask=expert_mask)
    K = ids_ref.shape[1]
    chosen = torch.zeros(ids_ref.shape[0] * K + 1, dtype=torch.bool)
    chosen[(tokens[:, None] * K + torch.arange(K)[None, :]).flatten()] = True
    hit = chosen[sid.long()].view(-1, block_m).any(dim=1)
    return int(hit.sum()), nv // block_m


def fused_workspace_intermediate(workspace, capacity, T, topk, H, I):
    """Views of the re-quantised intermediate in a fused MoE call's workspace, by the layout
    include/fp8moe.h states: (a2 fp8 codes as uint8 [capacity, I], scales fp32 [I/128, capacity])."""
    off = 0

    def take(nbytes):
        nonlocal off
        at = off
        off = (off + nbytes + 255) // 256 * 256
        return at

    take(capacity * H)                                  # slot-ordered activations
    take(H // 128 * capacity * 4)                       # their scales
    a2 = take(capacity * I)
    s2 = take(I // 128 * capacity * 4)
    ws = workspace.view(torch.uint8)
    return (ws[a2:a2 + capacity * I].view(capacity, I),
            ws[s2:s2 + I // 128 * capacity * 4].view(torch.float32).view(I // 128, capacity))


def e4m3_ordinal(codes):
    """E4M3 codes as signed ordinals (+-0 -> 0, adjacent values differ by 1), to count steps."""
    c = codes.to(torch.int32)
    return torch.where(c >= 128, -(c - 128), c)
