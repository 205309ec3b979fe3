"""Shared pieces of the GPU parity tests: oracle-side expert weights and the
output criterion. The oracle always quantises raw weights itself; raw weights
drawn on the device by the input generator are copied to the host for it."""
import torch

from oracle import fp8moe_oracle as O
from fp8_block_scaled_biased_b200 import inputs as I


def oracle_expert(cfg, e, device="cuda"):
    """Oracle-quantised weights of expert e from the same raw numbers the device layer used."""
    w1 = I.expert_weight_raw(cfg, "w1", e, device).cpu()
    w2 = I.expert_weight_raw(cfg, "w2", e, device).cpu()
    q1, s1 = O.quant_128x128(w1)
    q2, s2 = O.quant_128x128(w2)
    return q1, s1, q2, s2


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
    cache = {}

    def get(e):
        if e not in cache:
            cache[e] = oracle_expert(cfg, e, device)
        return cache.pop(e)

    out = O.moe_layer(a8, asc, sub_ids, sub_w, get, round_bf16=False, expert_mask=expert_mask)
    return out, w, ids
