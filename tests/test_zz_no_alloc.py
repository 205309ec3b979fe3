"""The no-allocation fused MoE entry point against the workspace entry point and the oracle.

fused_moe_fp8_blockscale_g1u1_noalloc exists for callers that cannot allocate
device memory where they call the layer (their memory manager owns the device
after start-up, or the path cannot take cudaMalloc's device-wide sync). It runs
the same kernels on scratch built into the library. These tests call it through
the C ABI twice in a row, with its scratch keeping the previous call's contents,
and require each output to equal fused_moe_fp8_blockscale_g1u1's (which uses a
caller-provided workspace) bit for bit: the kernels are deterministic, so the
scratch's origin must not change a single bit. One output is also held to the
oracle under the MoE output tolerance. A problem too large for the built-in
scratch, and weights whose shapes do not match, are refused before any launch.
This file is collected last so that a run stopping at its first failure has run
every other test before it.
"""
import ctypes

import pytest
import torch

from fp8_block_scaled_biased_b200 import binding as B
from fp8_block_scaled_biased_b200 import inputs as I
from fp8_block_scaled_biased_b200.layer import MoELayer
from tests.gpu_helpers import assert_moe_close, oracle_moe_rows

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

# one row block per expert (about 32 pairs each), and few experts holding several
# row blocks each (about 256 pairs: full 128-row tiles and M=64 tails)
ONE_BLOCK = I.MoEConfig("noalloc_t256_h1024_e32", T=256, H=1024, E=32, G=4, TG=2, K=4, I=512, seed=5)
MULTI_BLOCK = I.MoEConfig("noalloc_t1024_h1024_e8", T=1024, H=1024, E=8, G=2, TG=1, K=2, I=512, seed=6)


@pytest.mark.parametrize("cfg", [ONE_BLOCK, MULTI_BLOCK], ids=lambda c: c.name)
def test_noalloc_equals_workspace_entry_point_on_two_calls(cfg):
    layer = MoELayer(cfg, "cuda", tiled=False).load_synthetic_weights()       # the call takes row-major weights
    act = I.moe_activations(cfg)
    ref = layer.forward(act.logits.cuda(), act.bias.cuda(), act.x.cuda()).clone()
    need = B.load_library().fused_moe_fp8_blockscale_g1u1_workspace(cfg.T, cfg.K, cfg.E, cfg.H, cfg.I,
                                                                    layer.block_m)
    assert need <= B.NOALLOC_SCRATCH_BYTES
    outs = []
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        B.fused_moe_fp8_blockscale_g1u1_noalloc(out, layer.a8, layer.w1, layer.w2, layer.sorted, cfg.K,
                                                layer.a8_scale, layer.w1_scale, layer.w2_scale)
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"call {call}: differs from the workspace entry point"
        outs.append(out)
    assert B.device_status() == 0
    if cfg is MULTI_BLOCK:
        blocks = layer.sorted.sorted_expert_ids[: int(layer.sorted.num_valid_ids.item()) // layer.block_m].cpu()
        assert int(torch.bincount(blocks).max()) >= 2          # some expert spans several row blocks
    oracle, _, ids_ref = oracle_moe_rows(cfg, act, None)
    assert torch.equal(layer.topk_ids.cpu(), ids_ref)
    assert_moe_close(outs[-1], oracle)


def test_noalloc_refuses_problems_beyond_its_scratch():
    lib = B.load_library()
    T, K, E, H, Im = 64, 8, 256, 7168, 2048                  # the DeepSeek-V3 decode layer
    cap = lib.moe_align_sort_capacity(T, K, E, 128)
    assert lib.fused_moe_fp8_blockscale_g1u1_workspace(T, K, E, H, Im, 128) > B.NOALLOC_SCRATCH_BYTES
    p = ctypes.c_void_p(16)                                    # never dereferenced: refused first
    rc = lib.fused_moe_fp8_blockscale_g1u1_noalloc(p, p, p, p, p, p, p, p, T, H, Im, E, K, 128, cap, p, p, p,
                                                   128, 128, None, None)
    assert rc == 2
    assert b"built-in" in lib.fp8moe_last_error()


def test_noalloc_binding_refuses_mismatched_or_strided_weights():
    """The binding checks the no-allocation call's tensors as it checks the workspace call's:
    the library sizes its tensor maps from these shapes, so a mismatch must never reach it."""
    cfg = ONE_BLOCK
    layer = MoELayer(cfg, "cuda", tiled=False)
    act = I.moe_activations(cfg)
    a8, a1 = B.fp8_per_token_group_quant(act.x.cuda(), 128, column_major_scales=True)
    sp = B.alloc_sorted(cfg.T, cfg.K, cfg.E, layer.block_m, "cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    bad_w1 = torch.empty(cfg.E, 2 * cfg.I + 128, cfg.H, dtype=B.FP8, device="cuda")
    strided_w2 = torch.empty(cfg.E, cfg.H, 2 * cfg.I, dtype=B.FP8, device="cuda")[:, :, : cfg.I]
    wrong_dtype_w2 = torch.empty(cfg.E, cfg.H, cfg.I, dtype=torch.uint8, device="cuda")
    for w1, w2 in ((bad_w1, layer.w2), (layer.w1, strided_w2)):
        with pytest.raises(ValueError):
            B.fused_moe_fp8_blockscale_g1u1_noalloc(out, a8, w1, w2, sp, cfg.K, a1, layer.w1_scale, layer.w2_scale)
    with pytest.raises(TypeError):
        B.fused_moe_fp8_blockscale_g1u1_noalloc(out, a8, layer.w1, wrong_dtype_w2, sp, cfg.K, a1, layer.w1_scale,
                                                layer.w2_scale)
