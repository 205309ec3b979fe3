"""Host-side checks of the C ABI: the library loads, exports every declared entry
point, sizes its buffers by the stated formulas and rejects bad arguments with a
status code before touching a GPU."""
import ctypes
import os
import re

import pytest

from fp8_block_scaled_biased_b200 import binding as B
from fp8_block_scaled_biased_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return B.load_library()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "fp8moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", src, flags=re.M))


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert names == set(B.EXPORTED)


def test_capacity_and_workspace_formulas(lib):
    assert lib.moe_align_sort_capacity(64, 8, 256, 128) == 64 * 8 + 256 * 127
    assert lib.moe_align_sort_capacity(16, 4, 16, 1) == 64
    cap = 64 * 8 + 256 * 127
    need = lib.fused_moe_fp8_blockscale_g1u1_workspace(64, 8, 256, 7168, 2048, 128)
    assert need >= cap * 7168 + 56 * cap * 4 + cap * 2048 + 16 * cap * 4 + 64 * 8 * 7168 * 2
    assert lib.fp8moe_moe_block_m() == 128


def _rc(lib, name, *args):
    return getattr(lib, name)(*args), lib.fp8moe_last_error().decode()


# A non-null pointer that is never dereferenced: every call below fails validation
# before any CUDA call, so nothing is launched (these tests must never reach a device).
P = ctypes.c_void_p(16)


def test_routing_rejects_bad_arguments(lib):
    rc, msg = _rc(lib, "moe_biased_grouped_topk", P, 16, P, P, P, 3, 16, 16, 4, 4, 2, 1, 2.5, None)
    assert rc == 1 and "ld_out" in msg                                    # strided outputs too narrow
    rc, msg = _rc(lib, "moe_biased_grouped_topk", P, 16, P, P, P, 4, 16, 15, 4, 4, 2, 1, 2.5, None)
    assert rc == 1                                                        # E % groups != 0
    rc, _ = _rc(lib, "moe_biased_grouped_topk", P, 16, P, P, P, 4, 16, 16, 4, 4, 5, 1, 2.5, None)
    assert rc == 1                                                        # topk_group > groups
    rc, _ = _rc(lib, "moe_biased_grouped_topk", P, 16, P, P, P, 9, 16, 16, 9, 4, 2, 1, 2.5, None)
    assert rc == 1                                                        # topk > candidates
    rc, _ = _rc(lib, "moe_biased_grouped_topk", P, 1024, P, P, P, 8, 16, 1024, 8, 8, 4, 1, 2.5, None)
    assert rc == 2                                                        # E above the kernel's limit
    rc, _ = _rc(lib, "moe_biased_grouped_topk", P, 16, P, P, P, 4, 0, 16, 4, 4, 2, 1, 2.5, None)
    assert rc == 0                                                        # T == 0: nothing to do


def test_sort_rejects_bad_arguments(lib):
    cap = lib.moe_align_sort_capacity(16, 4, 16, 4)
    rc, msg = _rc(lib, "moe_align_sort", P, P, 4, 16, 4, 16, 4, P, P, P, P, cap - 1, None, 0, None)
    assert rc == 1 and "capacity" in msg
    rc, _ = _rc(lib, "moe_align_sort", P, P, 3, 16, 4, 16, 4, P, P, P, P, cap, None, 0, None)
    assert rc == 1
    rc, _ = _rc(lib, "moe_align_sort", P, P, 4, 16, 4, 2000, 4, P, P, P, P, 10 ** 6, None, 0, None)
    assert rc == 2
    ws = lib.moe_align_sort_workspace(16, 4, 16, 4)
    assert ws >= 16 * 4                                   # per-chunk histograms
    rc, msg = _rc(lib, "moe_align_sort", P, P, 4, 16, 4, 16, 4, P, P, P, P, cap, P, ws - 1, None)
    assert rc == 3 and "workspace" in msg


def test_quant_and_gemm_reject_bad_arguments(lib):
    rc, _ = _rc(lib, "fp8_per_token_group_quant", P, 256, 4, 256, 64, P, P, 0, None)
    assert rc == 2                                                        # group != 128
    rc, _ = _rc(lib, "fp8_per_token_group_quant", P, 256, 4, 250, 128, P, P, 0, None)
    assert rc == 2                                                        # K % 8 != 0
    rc, _ = _rc(lib, "fp8_per_token_group_quant", P, 256, 4, 256, 128, P, P, 7, None)
    assert rc == 1                                                        # unknown layout
    rc, _ = _rc(lib, "fp8_per_block_quant", P, 256, 256, 256, 64, P, P, None)
    assert rc == 2
    rc, _ = _rc(lib, "fp8_blockscale_gemm", P, P, P, P, P, 64, 64, 64, 100, None)
    assert rc == 2                                                        # K % 16 != 0
    rc, _ = _rc(lib, "fp8_blockscale_gemm", P, P, P, P, P, 32, 64, 64, 128, None)
    assert rc == 1                                                        # ldc < N
    rc, _ = _rc(lib, "fp8_blockscale_gemm", None, P, P, P, P, 64, 64, 64, 128, None)
    assert rc == 1


def test_fused_moe_rejects_bad_arguments(lib):
    T, K, E, H, I = 16, 4, 16, 256, 128
    cap = lib.moe_align_sort_capacity(T, K, E, 128)
    ws = lib.fused_moe_fp8_blockscale_g1u1_workspace(T, K, E, H, I, 128)
    args = [P] * 8 + [T, H, I, E, K, 128, cap, P, P, P, 128, 128, None, ctypes.c_void_p(256), ws, None]

    def call(**over):
        a = list(args)
        idx = {"scale_blk_n": 18, "scale_blk_k": 19, "smooth": 20, "ws_bytes": 22, "block_m": 13, "H": 9,
               "cap": 14, "ws": 21}
        for k, v in over.items():
            a[idx[k]] = v
        return _rc(lib, "fused_moe_fp8_blockscale_g1u1", *a)

    assert call(scale_blk_n=64)[0] == 2
    assert call(scale_blk_k=256)[0] == 2
    assert call(smooth=P)[0] == 2
    assert call(block_m=64)[0] == 2
    assert call(H=200)[0] == 2
    assert call(cap=cap - 1)[0] == 1
    assert call(ws_bytes=ws - 1)[0] == 3
    assert call(ws=None)[0] == 3


def test_binding_fails_loudly_without_library(tmp_path):
    saved = B._lib
    B._lib = None
    try:
        with pytest.raises(RuntimeError):
            B.load_library(str(tmp_path / "missing.so"))
    finally:
        B._lib = saved


def test_bf16_routing_and_masked_sort_reject_bad_arguments(lib):
    rc, msg = _rc(lib, "moe_biased_grouped_topk_bf16", P, 16, P, P, P, 3, 16, 16, 4, 4, 2, 1, 2.5, None)
    assert rc == 1 and "ld_out" in msg
    rc, _ = _rc(lib, "moe_biased_grouped_topk_bf16", P, 1024, P, P, P, 8, 16, 1024, 8, 8, 4, 1, 2.5, None)
    assert rc == 2
    rc, _ = _rc(lib, "moe_biased_grouped_topk_bf16", P, 16, P, P, P, 4, 0, 16, 4, 4, 2, 1, 2.5, None)
    assert rc == 0
    cap = lib.moe_align_sort_capacity(16, 4, 16, 4)
    rc, msg = _rc(lib, "moe_align_sort_masked", P, P, 4, 16, 4, 16, 4, P, P, P, P, P, cap - 1, None, 0, None)
    assert rc == 1 and "capacity" in msg
    ws = lib.moe_align_sort_workspace(16, 4, 16, 4)
    rc, msg = _rc(lib, "moe_align_sort_masked", P, P, 4, 16, 4, 16, 4, P, P, P, P, P, cap, P, ws - 1, None)
    assert rc == 3 and "workspace" in msg


def test_selftest_stall_rejects_a_k_block_out_of_range(lib):
    rc, msg = _rc(lib, "fp8moe_selftest_gemm_stall", P, P, P, P, P, 256, 128, 256, 256, 2, None)
    assert rc == 1 and "stall_kb" in msg


def test_workspace_bytes_cover_a_sorted_list_over_more_experts(lib):
    """A list sorted over E+1 experts (a masked-out sentinel expert, as the expert-parallel
    owner sorts) has a larger capacity than the weights' E implies: the binding sizes the
    fused call's workspace for that capacity."""
    T, K, E, H, I, bm = 256, 4, 8, 1024, 512, 128
    cap = lib.moe_align_sort_capacity(T, K, E + 1, bm)
    assert B.fused_moe_workspace_bytes(T, K, E, H, I, bm, capacity=cap) == \
        lib.fused_moe_fp8_blockscale_g1u1_workspace(T, K, E + 1, H, I, bm)
    assert B.fused_moe_workspace_bytes(T, K, E, H, I, bm) < B.fused_moe_workspace_bytes(T, K, E, H, I, bm, capacity=cap)


def test_tile_weights_and_tiled_fused_call_reject_bad_arguments(lib):
    rc, msg = _rc(lib, "fp8_tile_weights", P, 2, 200, 128, ctypes.c_void_p(1 << 20), None)
    assert rc == 2 and "multiples of 128" in msg                       # N not a multiple of 128
    rc, _ = _rc(lib, "fp8_tile_weights", P, 0, 128, 128, ctypes.c_void_p(1 << 20), None)
    assert rc == 1                                                     # no experts
    rc, msg = _rc(lib, "fp8_tile_weights", P, 1, 128, 128, P, None)
    assert rc == 1 and "overlap" in msg                                # in place is refused
    rc, _ = _rc(lib, "fp8_tile_weights", ctypes.c_void_p(24), 1, 128, 128, ctypes.c_void_p(1 << 20), None)
    assert rc == 1                                                     # w not 16-byte aligned
    T, K, E, H, I = 16, 4, 16, 256, 128
    cap = lib.moe_align_sort_capacity(T, K, E, 128)
    ws = lib.fused_moe_fp8_blockscale_g1u1_workspace(T, K, E, H, I, 128)
    args = [P] * 8 + [T, H, I, E, K, 128, cap, P, P, P, 128, 128, None, ctypes.c_void_p(256), ws, None]
    a = list(args)
    a[18] = 64                                                         # scale_blk_n
    assert _rc(lib, "fused_moe_fp8_blockscale_g1u1_tiled", *a)[0] == 2
    a = list(args)
    a[22] = ws - 1                                                     # workspace too small
    assert _rc(lib, "fused_moe_fp8_blockscale_g1u1_tiled", *a)[0] == 3


def test_multi_gpu_entry_points_reject_bad_arguments(lib):
    """The tensor- and expert-parallel entry points check ranks, sizes and pointers on the
    host and return a status before touching a GPU."""
    p = ctypes.c_void_p(16)
    one = (ctypes.c_void_p * 1)(16)
    nine = (ctypes.c_void_p * 9)(*([16] * 9))
    Ts = -(-300 // 8)
    assert lib.moe_tp_recv_bytes(300, 1024, 8) == 8 * Ts * 1024 * 2
    assert lib.moe_tp_recv_bytes(300, 1024, 9) == 0 and lib.moe_tp_recv_bytes(300, 1024, 0) == 0
    # combine + all-reduce: nranks, rank, sizes, pointers
    assert lib.moe_combine_allreduce(p, 1 << 20, 300, 4, 1024, 512, 0, 0, one, one, one, p, None) == 1
    assert lib.moe_combine_allreduce(p, 1 << 20, 300, 4, 1024, 512, 1, 1, one, one, one, p, None) == 1
    assert lib.moe_combine_allreduce(p, 1 << 20, 300, 4, 1000, 512, 1, 0, one, one, one, p, None) == 2   # H % 128
    assert lib.moe_combine_allreduce(p, 1 << 20, 300, 4, 1024, 512, 1, 0, None, one, one, p, None) == 1
    assert lib.moe_combine_allreduce_emulated(None, 1 << 20, 300, 4, 1024, 512, 1, one, one, one, one, None) == 1
    assert lib.moe_combine_allreduce_emulated(nine, 1 << 20, 300, 4, 1024, 512, 9, nine, nine, nine, nine,
                                              None) == 1
    # expert parallelism: ranks, expert ranges, sizes
    assert lib.moe_ep_routing(one, one, 0, 10, 4, 16, 0, 4, p, p, None) == 1
    assert lib.moe_ep_routing(one, one, 1, 10, 4, 16, 14, 4, p, p, None) == 1     # e0 + ne > E
    assert lib.moe_ep_barrier(2, 2, one, None) == 1
    assert lib.moe_ep_barrier(9, 0, nine, None) == 1
    assert lib.moe_ep_barrier(1, 0, None, None) == 1
    assert lib.moe_ep_return(p, 1 << 20, 9, 10, 4, 1024, 512, p, p, nine, nine, None) == 1
    assert lib.moe_combine_pairs(p, p, 10, 0, 1024, p, None) == 1
    assert lib.moe_combine_pairs(p, p, 10, 4, 1004, p, None) == 1          # H % 8 != 0
    assert lib.fused_moe_fp8_blockscale_g1u1_multi(one, one, 9, 10, p, p, p, p, p, p, 1024, 512, 4, 4, 128, 1 << 20,
                                                   p, p, 128, 128, None, 1, None, None, p, 1 << 30, None) == 1
    assert lib.fused_moe_fp8_blockscale_g1u1_multi(one, one, 1, 10, p, p, p, p, p, p, 1024, 512, 4, 4, 128, 1 << 20,
                                                   p, p, 128, 128, None, 1, p, None, p, 1 << 30, None) == 1


def test_mla_decode_rejects_bad_arguments_and_sizes_its_workspace(lib):
    """The MLA decode entry point checks heads, sizes, scales, pointers, alignment and the
    workspace on the host, and sizes the split partials by the stated formula."""
    p = ctypes.c_void_p(16)
    odd = ctypes.c_void_p(18)
    assert lib.mla_decode_num_splits(64, 16) == 296 // 64
    assert lib.mla_decode_num_splits(64, 128) == 1 and lib.mla_decode_num_splits(1, 16) == 64
    assert lib.mla_decode_workspace(64, 16, 4) == 64 * 16 * 4 * 513 * 4
    assert lib.mla_decode_workspace(64, 16, 1) == 0 and lib.mla_decode_workspace(64, 128, 0) == 0

    def call(q=p, kv=p, o=p, ip=p, ix=p, ll=p, B=2, H=16, pages=4, ps=1, ni=4, scale=0.04, cap=0.0, splits=1,
             ws=None, wsb=0):
        return lib.mla_decode_fwd(q, kv, o, ip, ix, ll, None, B, H, pages, ps, ni, scale, cap, splits, ws, wsb, None)

    assert call(H=8) == 2 and call(H=24) == 2 and call(H=144) == 2        # heads: 16, 32, ..., 128
    assert call(ps=0) == 1 and call(B=-1) == 1 and call(ni=-1) == 1
    assert call(scale=0.0) == 1 and call(scale=float("nan")) == 1 and call(cap=-1.0) == 1
    assert call(splits=65) == 2
    assert call(q=None) == 1 and call(ip=None) == 1 and call(kv=None) == 1
    assert call(q=odd) == 1 and call(kv=odd) == 1
    assert call(splits=2) == 3                                             # partials need a workspace
    assert call(splits=2, ws=p, wsb=lib.mla_decode_workspace(2, 16, 2) - 1) == 3
    assert call(ni=1 << 20, ps=4096) == 2                                  # token positions past int32
    assert call(B=70000) == 2
    assert call(B=0) == 0                                                  # nothing to do
