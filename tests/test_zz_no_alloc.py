"""The no-allocation fused MoE entry point against the workspace entry point.

fused_moe_fp8_blockscale_g1u1_noalloc exists for callers that cannot allocate
device memory where they call the layer (their memory manager owns the device
after start-up, or the path cannot take cudaMalloc's device-wide sync). It runs
the same computation on scratch built into the library. These tests call it
through the C ABI twice in a row, with its scratch keeping the previous call's
contents, and compare each output with fused_moe_fp8_blockscale_g1u1 (which
uses a caller-provided workspace) under the MoE output tolerance. They also
check that a problem too large for the built-in scratch is refused up front.
This file is collected last so that a run stopping at its first failure has
run every other test before it.
"""
import ctypes

import pytest
import torch

from fp8_block_scaled_biased_b200 import binding as B
from fp8_block_scaled_biased_b200 import inputs as I
from fp8_block_scaled_biased_b200.layer import MoELayer
from tests.gpu_helpers import moe_error

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CFG = I.MoEConfig("noalloc_t256_h1024_e32", T=256, H=1024, E=32, G=4, TG=2, K=4, I=512, seed=5)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    layer = MoELayer(CFG, "cuda").load_synthetic_weights()
    act = I.moe_activations(CFG)
    ref = layer.forward(act.logits.cuda(), act.bias.cuda(), act.x.cuda()).clone()
    need = B.load_library().fused_moe_fp8_blockscale_g1u1_workspace(CFG.T, CFG.K, CFG.E, CFG.H, CFG.I,
                                                                    layer.block_m)
    assert need <= B.NOALLOC_SCRATCH_BYTES
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        B.fused_moe_fp8_blockscale_g1u1_noalloc(out, layer.a8, layer.w1, layer.w2, layer.sorted, CFG.K,
                                                layer.a8_scale, layer.w1_scale, layer.w2_scale)
        torch.cuda.synchronize()
        dmax, bound, mre = moe_error(out, ref)
        assert dmax <= bound, f"call {call}: max |d| {dmax:.3e} > {bound:.3e}"
        assert mre <= 5e-3, f"call {call}: mean relative error {mre:.3e}"
    assert B.device_status() == 0


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
