"""Write tests/golden/tiny_oracle.json from the oracle alone (no CUDA code involved).

Run from the repository root:  python tests/golden/make_golden.py
The fixture freezes the oracle's results on the tiny workload (T=16, H=256,
E=16 in 4 groups, topk_group=2, topk=4, I=128, renorm, factor 2.5, seed 0) so
that an accidental change to the oracle's arithmetic shows up as a test failure.
"""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from oracle import fp8moe_oracle as O  # noqa: E402
from fp8_block_scaled_biased_b200 import inputs as I  # noqa: E402

BLOCK_M = 4


def sha(t: torch.Tensor) -> str:
    return hashlib.sha256(t.contiguous().numpy().tobytes()).hexdigest()


def compute():
    cfg = I.TINY
    act = I.moe_activations(cfg)
    w, ids = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    sid, sw, se, nv = O.align_sort(ids, w, cfg.E, BLOCK_M)
    a8, asc = O.quant_1x128(act.x)
    ex = {}
    for e in range(cfg.E):
        w1q, w1s = O.quant_128x128(I.expert_weight_raw(cfg, "w1", e))
        w2q, w2s = O.quant_128x128(I.expert_weight_raw(cfg, "w2", e))
        ex[e] = (w1q, w1s, w2q, w2s)
    out = O.moe_layer(a8, asc, ids, w, lambda e: ex[e]).to(torch.float32)
    return {
        "workload": cfg.name,
        "block_m": BLOCK_M,
        "topk_ids": ids.tolist(),
        "topk_weights_f32_bits": w.view(torch.int32).tolist(),
        "sorted_ids": sid.tolist(),
        "sorted_expert_ids": se.tolist(),
        "num_valid_ids": nv,
        "a8_scale_f32_bits": asc.view(torch.int32).tolist(),
        "a8_sha256": sha(a8),
        "w1_expert0_sha256": sha(ex[0][0]),
        "out_bf16_sha256": sha(out.to(torch.bfloat16).view(torch.int16)),
        "out_first_row": out[0, :8].tolist(),
    }


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as f:
        json.dump(compute(), f, indent=1)
    print("wrote", path)
