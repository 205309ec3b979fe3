"""ctypes binding of libfp8moe.so: the C ABI in include/fp8moe.h, called with torch tensors.

Argument marshalling only: every function checks dtypes/devices, passes raw
device pointers and sizes to the library, and raises on a non-zero status.
All arithmetic happens in the library's CUDA kernels. There is no fallback:
if the library cannot be loaded, every call raises.

PyTorch is used for device memory and streams only; each call runs on the
current torch CUDA stream.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfp8moe.so")

_c_int, _c_float, _c_size, _p = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p

_SIGNATURES = {
    "fp8moe_last_error": (ctypes.c_char_p, []),
    "fp8moe_device_status": (_c_int, [_p]),
    "fp8moe_moe_block_m": (_c_int, []),
    "fp8moe_timing_enable": (_c_int, [_c_int]),
    "fp8moe_timing_last": (_c_int, [ctypes.POINTER(ctypes.c_float)]),
    "moe_biased_grouped_topk": (_c_int, [_p, _c_int, _p, _p, _p, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                         _c_int, _c_float, _p]),
    "moe_biased_grouped_topk_bf16": (_c_int, [_p, _c_int, _p, _p, _p, _c_int, _c_int, _c_int, _c_int, _c_int,
                                              _c_int, _c_int, _c_float, _p]),
    "moe_align_sort_capacity": (_c_size, [_c_int, _c_int, _c_int, _c_int]),
    "moe_align_sort_workspace": (_c_size, [_c_int, _c_int, _c_int, _c_int]),
    "moe_align_sort": (_c_int, [_p, _p, _c_int, _c_int, _c_int, _c_int, _c_int, _p, _p, _p, _p, _c_size, _p,
                                _c_size, _p]),
    "moe_align_sort_masked": (_c_int, [_p, _p, _c_int, _c_int, _c_int, _c_int, _c_int, _p, _p, _p, _p, _p, _c_size,
                                       _p, _c_size, _p]),
    "fp8_per_token_group_quant": (_c_int, [_p, _c_int, _c_int, _c_int, _c_int, _p, _p, _c_int, _p]),
    "fp8_per_block_quant": (_c_int, [_p, _c_int, _c_int, _c_int, _c_int, _p, _p, _p]),
    "fp8_blockscale_gemm": (_c_int, [_p, _p, _p, _p, _p, _c_int, _c_int, _c_int, _c_int, _p]),
    "fp8moe_selftest_gemm_stall": (_c_int, [_p, _p, _p, _p, _p, _c_int, _c_int, _c_int, _c_int, _c_int, _p]),
    "fused_moe_fp8_blockscale_g1u1_workspace": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int]),
    "fused_moe_fp8_blockscale_g1u1": (_c_int, [_p, _p, _p, _p, _p, _p, _p, _p, _c_int, _c_int, _c_int, _c_int,
                                               _c_int, _c_int, _c_size, _p, _p, _p, _c_int, _c_int, _p, _p,
                                               _c_size, _p]),
    "fused_moe_fp8_blockscale_g1u1_noalloc": (_c_int, [_p, _p, _p, _p, _p, _p, _p, _p, _c_int, _c_int, _c_int,
                                                       _c_int, _c_int, _c_int, _c_size, _p, _p, _p, _c_int, _c_int,
                                                       _p, _p]),
    "fused_moe_fp8_blockscale_g1u1_tiled": (_c_int, [_p, _p, _p, _p, _p, _p, _p, _p, _c_int, _c_int, _c_int, _c_int,
                                                     _c_int, _c_int, _c_size, _p, _p, _p, _c_int, _c_int, _p, _p,
                                                     _c_size, _p]),
    "fp8_tile_weights": (_c_int, [_p, _c_int, _c_int, _c_int, _p, _p]),
    "fused_moe_fp8_blockscale_g1u1_pairs": (_c_int, [_p, _p, _p, _p, _p, _p, _p, _c_int, _c_int, _c_int, _c_int,
                                                     _c_int, _c_int, _c_size, _p, _p, _p, _c_int, _c_int, _p,
                                                     _c_int, _p, _c_size, _p]),
    "moe_tp_recv_bytes": (_c_size, [_c_int, _c_int, _c_int]),
    "moe_combine_allreduce": (_c_int, [_p, _c_size, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _p, _p, _p, _p,
                                       _p]),
    "moe_combine_allreduce_emulated": (_c_int, [_p, _c_size, _c_int, _c_int, _c_int, _c_int, _c_int, _p, _p, _p, _p,
                                                _p]),
    "moe_ep_routing": (_c_int, [_p, _p, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _p, _p, _p]),
    "fused_moe_fp8_blockscale_g1u1_multi": (_c_int, [_p, _p, _c_int, _c_int, _p, _p, _p, _p, _p, _p, _c_int, _c_int,
                                                     _c_int, _c_int, _c_int, _c_size, _p, _p, _c_int, _c_int, _p,
                                                     _c_int, _p, _p, _p, _c_size, _p]),
    "moe_ep_return": (_c_int, [_p, _c_size, _c_int, _c_int, _c_int, _c_int, _c_int, _p, _p, _p, _p, _p]),
    "moe_ep_barrier": (_c_int, [_c_int, _c_int, _p, _p]),
    "moe_ep_barrier_emulated": (_c_int, [_c_int, _p, _p]),
    "moe_combine_pairs": (_c_int, [_p, _p, _c_int, _c_int, _c_int, _p, _p]),
    "mla_decode_num_splits": (_c_int, [_c_int, _c_int]),
    "mla_decode_workspace": (_c_size, [_c_int, _c_int, _c_int]),
    "mla_decode_fwd": (_c_int, [_p, _p, _p, _p, _p, _p, _p, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                                _c_float, _c_int, _p, _c_size, _p]),
}
EXPORTED = tuple(_SIGNATURES)

NOALLOC_SCRATCH_BYTES = 64 << 20   # FP8MOE_NOALLOC_SCRATCH_BYTES in include/fp8moe.h
TP_MAX_RANKS = 8                   # FP8MOE_TP_MAX_RANKS
TP_FLAG_WORDS = 16                 # FP8MOE_TP_FLAG_WORDS (64-bit words per rank)
TP_BARRIER_WORDS = 3               # FP8MOE_TP_BARRIER_WORDS (arrivals, generation, calls)
EP_MAX_RANKS = 8                   # FP8MOE_EP_MAX_RANKS
EP_BARRIER_WORDS = 9               # FP8MOE_EP_BARRIER_WORDS (one per rank, then the calls)
MLA_QK_HEAD_DIM = 576              # query/key width of the MLA decode call (512 latent + 64 rotary)
MLA_V_HEAD_DIM = 512               # its value width
SCALE_ROW_MAJOR = 0
SCALE_COL_MAJOR = 1
FP8 = torch.float8_e4m3fn

_lib = None


class Fp8MoeError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load (once) and type the library; raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} not found: build it with `python -m fp8_block_scaled_biased_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(name, rc):
    if rc != 0:
        raise Fp8MoeError(name, rc, load_library().fp8moe_last_error().decode())


def _cuda(t, dtype, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def _row_major(t, name):
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D tensor with unit column stride")
    return t.stride(0)


def device_status() -> int:
    """Synchronise the current stream; return and clear the device error word."""
    rc = load_library().fp8moe_device_status(_stream())
    if rc < 0:
        raise Fp8MoeError("fp8moe_device_status", rc, load_library().fp8moe_last_error().decode())
    return rc


def timing_enable(on: bool = True):
    """Record per-kernel events inside each fused MoE call (calling thread only)."""
    _check("fp8moe_timing_enable", load_library().fp8moe_timing_enable(int(bool(on))))


def timing_last():
    """(gather ms, gate/up GEMM ms, down GEMM ms, combine ms) of the most recent fused MoE call; waits for it."""
    ms = (ctypes.c_float * 4)()
    _check("fp8moe_timing_last", load_library().fp8moe_timing_last(ms))
    return tuple(ms)


def moe_block_m() -> int:
    return load_library().fp8moe_moe_block_m()


def moe_biased_grouped_topk(gating_output, correction_bias, topk_weights, topk_ids, num_expert_group, topk_group,
                            need_renorm, routed_scaling_factor=1.0):
    """Writes topk_weights fp32 [T, topk] and topk_ids int32 [T, topk] (row stride may exceed topk).

    gating_output is fp32 or bf16 [T, E]; bf16 logits take moe_biased_grouped_topk_bf16."""
    if gating_output.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"gating_output must be torch.float32 or torch.bfloat16, got {gating_output.dtype}")
    _cuda(gating_output, gating_output.dtype, "gating_output")
    _cuda(correction_bias, torch.float32, "correction_bias")
    _cuda(topk_weights, torch.float32, "topk_weights")
    _cuda(topk_ids, torch.int32, "topk_ids")
    T, E = gating_output.shape
    topk = topk_weights.shape[1]
    ld_out = _row_major(topk_weights, "topk_weights")
    if _row_major(topk_ids, "topk_ids") != ld_out:
        raise ValueError("topk_weights and topk_ids must share a row stride")
    lib = load_library()
    fn = lib.moe_biased_grouped_topk_bf16 if gating_output.dtype == torch.bfloat16 else lib.moe_biased_grouped_topk
    rc = fn(
        _ptr(gating_output), _row_major(gating_output, "gating_output"), _ptr(correction_bias.contiguous()),
        _ptr(topk_weights), _ptr(topk_ids), ld_out, T, E, topk, num_expert_group, topk_group, int(bool(need_renorm)),
        float(routed_scaling_factor), _stream())
    _check(fn.__name__, rc)


def moe_align_sort_capacity(T, topk, E, block_m):
    return load_library().moe_align_sort_capacity(T, topk, E, block_m)


@dataclass
class SortedPairs:
    sorted_ids: torch.Tensor          # int32 [capacity]
    sorted_weights: torch.Tensor      # fp32 [capacity]
    sorted_expert_ids: torch.Tensor   # int32 [capacity // block_m + 1]
    num_valid_ids: torch.Tensor       # int32 [1] (device)
    block_m: int

    @property
    def capacity(self) -> int:
        return self.sorted_ids.numel()


def alloc_sorted(T, topk, E, block_m, device) -> SortedPairs:
    cap = moe_align_sort_capacity(T, topk, E, block_m)
    return SortedPairs(
        sorted_ids=torch.empty(cap, dtype=torch.int32, device=device),
        sorted_weights=torch.empty(cap, dtype=torch.float32, device=device),
        sorted_expert_ids=torch.empty(cap // block_m + 1, dtype=torch.int32, device=device),
        num_valid_ids=torch.empty(1, dtype=torch.int32, device=device),
        block_m=block_m)


def moe_align_sort_workspace_bytes(T, topk, E, block_m):
    return load_library().moe_align_sort_workspace(T, topk, E, block_m)


def moe_align_sort(topk_ids, topk_weights, num_experts, block_m, out: SortedPairs | None = None,
                   workspace=None, expert_mask=None) -> SortedPairs:
    """Sorted, block-padded pair list. expert_mask (int32 [E] on the device, nonzero = keep)
    drops the pairs of masked-out experts (moe_align_sort_masked)."""
    _cuda(topk_ids, torch.int32, "topk_ids")
    if expert_mask is not None:
        _cuda(expert_mask, torch.int32, "expert_mask")
        if expert_mask.numel() != num_experts or not expert_mask.is_contiguous():
            raise ValueError("expert_mask must be a contiguous int32 tensor of num_experts entries")
    _cuda(topk_weights, torch.float32, "topk_weights")
    T, topk = topk_ids.shape
    ld = _row_major(topk_ids, "topk_ids")
    if _row_major(topk_weights, "topk_weights") != ld:
        raise ValueError("topk_ids and topk_weights must share a row stride")
    if out is None:
        out = alloc_sorted(T, topk, num_experts, block_m, topk_ids.device)
    lib = load_library()
    if workspace is None:
        workspace = torch.empty(lib.moe_align_sort_workspace(T, topk, num_experts, block_m), dtype=torch.uint8,
                                device=topk_ids.device)
    if expert_mask is None:
        rc = lib.moe_align_sort(_ptr(topk_ids), _ptr(topk_weights), ld, T, topk, num_experts, block_m,
                                _ptr(out.sorted_ids), _ptr(out.sorted_weights), _ptr(out.sorted_expert_ids),
                                _ptr(out.num_valid_ids), out.capacity, _ptr(workspace), workspace.numel(), _stream())
        _check("moe_align_sort", rc)
    else:
        rc = lib.moe_align_sort_masked(_ptr(topk_ids), _ptr(topk_weights), ld, T, topk, num_experts, block_m,
                                       _ptr(expert_mask), _ptr(out.sorted_ids), _ptr(out.sorted_weights),
                                       _ptr(out.sorted_expert_ids), _ptr(out.num_valid_ids), out.capacity,
                                       _ptr(workspace), workspace.numel(), _stream())
        _check("moe_align_sort_masked", rc)
    return out


def fp8_per_token_group_quant(x, group=128, column_major_scales=False, q=None, scales=None):
    """1 x group FP8 quantisation of bf16 x [M, K] -> (q fp8 [M, K], scales fp32)."""
    _cuda(x, torch.bfloat16, "x")
    M, K = x.shape
    KB = (K + group - 1) // group
    if q is None:
        q = torch.empty(M, K, dtype=FP8, device=x.device)
    if scales is None:
        scales = torch.empty((KB, M) if column_major_scales else (M, KB), dtype=torch.float32, device=x.device)
    rc = load_library().fp8_per_token_group_quant(
        _ptr(x), _row_major(x, "x"), M, K, group, _ptr(q), _ptr(scales),
        SCALE_COL_MAJOR if column_major_scales else SCALE_ROW_MAJOR, _stream())
    _check("fp8_per_token_group_quant", rc)
    return q, scales


def fp8_per_block_quant(w, block=128, q=None, scales=None):
    """128 x 128 FP8 quantisation of fp32 w [N, K] -> (q fp8 [N, K], scales fp32 [N/128, K/128])."""
    _cuda(w, torch.float32, "w")
    N, K = w.shape
    if q is None:
        q = torch.empty(N, K, dtype=FP8, device=w.device)
    if scales is None:
        scales = torch.empty((N + block - 1) // block, (K + block - 1) // block, dtype=torch.float32, device=w.device)
    rc = load_library().fp8_per_block_quant(_ptr(w), _row_major(w, "w"), N, K, block, _ptr(q), _ptr(scales),
                                            _stream())
    _check("fp8_per_block_quant", rc)
    return q, scales


def fp8_tile_weights(w, out=None):
    """Re-pack fp8 expert matrices w [E, N, K] (or one matrix [N, K]) into the tiled layout
    [E, N/128, K/128, 128, 128]: every 128 x 128 block 16 KB of consecutive bytes."""
    _cuda(w, FP8, "w")
    if not w.is_contiguous():
        raise ValueError("w must be contiguous")
    w3 = w if w.dim() == 3 else w.unsqueeze(0)
    E, N, K = w3.shape
    if N % 128 or K % 128:
        raise ValueError(f"N and K must be multiples of 128 (N={N}, K={K})")
    if out is None:
        out = torch.empty(E, N // 128, K // 128, 128, 128, dtype=FP8, device=w.device)
    _cuda(out, FP8, "out")
    if out.numel() != w.numel() or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor with as many elements as w")
    rc = load_library().fp8_tile_weights(_ptr(w), E, N, K, _ptr(out), _stream())
    _check("fp8_tile_weights", rc)
    return out


def is_tiled(w) -> bool:
    """True for expert weights in the tiled layout ([E, N/128, K/128, 128, 128])."""
    return w.dim() == 5 and tuple(w.shape[3:]) == (128, 128)


def _expert_matrix_shape(w):
    """(E, N, K) of expert weights, row-major [E, N, K] or tiled [E, N/128, K/128, 128, 128]."""
    if is_tiled(w):
        return w.shape[0], w.shape[1] * 128, w.shape[2] * 128
    if w.dim() != 3:
        raise ValueError("expert weights must be [E, N, K] or tiled [E, N/128, K/128, 128, 128]")
    return tuple(w.shape)


def fp8_blockscale_gemm(A, B, a_scale, b_scale, out=None):
    """C bf16 [M, N] = block-scaled A fp8 [M, K] x B fp8 [N, K]^T."""
    _cuda(A, FP8, "A")
    _cuda(B, FP8, "B")
    _cuda(a_scale, torch.float32, "a_scale")
    _cuda(b_scale, torch.float32, "b_scale")
    M, K = A.shape
    N = B.shape[0]
    if not (A.is_contiguous() and B.is_contiguous() and a_scale.is_contiguous() and b_scale.is_contiguous()):
        raise ValueError("A, B and the scales must be contiguous")
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=A.device)
    rc = load_library().fp8_blockscale_gemm(_ptr(A), _ptr(B), _ptr(a_scale), _ptr(b_scale), _ptr(out),
                                            _row_major(out, "out"), M, N, K, _stream())
    _check("fp8_blockscale_gemm", rc)
    return out


def selftest_gemm_stall(A, B, a_scale, b_scale, out, stall_kb):
    """Failure-handling test hook: the block-scale GEMM with K block stall_kb's scales withheld,
    so its bounded wait runs out; the caller reads the timeout bit with device_status()."""
    M, K = A.shape
    N = B.shape[0]
    rc = load_library().fp8moe_selftest_gemm_stall(_ptr(A), _ptr(B), _ptr(a_scale), _ptr(b_scale), _ptr(out),
                                                   _row_major(out, "out"), M, N, K, stall_kb, _stream())
    _check("fp8moe_selftest_gemm_stall", rc)


def fused_moe_workspace_bytes(T, topk, E, H, I, block_m, capacity=None):
    """Workspace bytes of the fused call. capacity: the sorted list's capacity when it is larger
    than moe_align_sort_capacity(T, topk, E, block_m) (a list sorted over more experts than
    the weights hold, e.g. with a masked-out sentinel expert); the query is then made for the
    expert count whose capacity covers it."""
    if capacity is not None and block_m > 1:
        E = max(E, -(-(int(capacity) - T * topk) // (block_m - 1)))
    return load_library().fused_moe_fp8_blockscale_g1u1_workspace(T, topk, E, H, I, block_m)


def _fused_moe_shapes(out, a8, w1, w2, sorted_pairs, topk, a1_scale, fc1_scale, fc2_scale):
    """Checks shared by the fused MoE entry points; returns (T, H, I, E). out is None for
    the call without a combine.

    The library builds its TMA maps from these sizes (w1 as E*2I rows of H, w2 as
    E*H rows of I), so every tensor must have exactly the shape and dtype the sizes
    imply and be contiguous; anything else is refused before the call."""
    if out is not None:
        _cuda(out, torch.bfloat16, "out")
    _cuda(a8, FP8, "a8")
    _cuda(w1, FP8, "w1")
    _cuda(w2, FP8, "w2")
    for name, t in (("a1_scale", a1_scale), ("fc1_scale", fc1_scale), ("fc2_scale", fc2_scale)):
        _cuda(t, torch.float32, name)
    if a8.dim() != 2:
        raise ValueError("a8 must be [T, H]")
    if is_tiled(w1) != is_tiled(w2):
        raise ValueError("w1 and w2 must both be row-major or both tiled")
    T, H = a8.shape
    E, twoI, H1 = _expert_matrix_shape(w1)
    E2, H2, I = _expert_matrix_shape(w2)
    if twoI != 2 * I:
        raise ValueError("g1u1 requires 2I rows of w1 for I columns of w2")
    if H1 != H or (E2, H2) != (E, H):
        raise ValueError(f"w1 {tuple(w1.shape)} and w2 {tuple(w2.shape)} do not match a8's H={H}")
    if out is not None and tuple(out.shape) != (T, H):
        raise ValueError(f"out must be [{T}, {H}], got {tuple(out.shape)}")
    if H % 128 or I % 128:
        raise ValueError(f"H and I must be multiples of 128 (H={H}, I={I})")
    expect = {"a1_scale": (H // 128, T), "fc1_scale": (E, 2 * I // 128, H // 128),
              "fc2_scale": (E, H // 128, I // 128)}
    for name, t in (("a1_scale", a1_scale), ("fc1_scale", fc1_scale), ("fc2_scale", fc2_scale)):
        if tuple(t.shape) != expect[name]:
            raise ValueError(f"{name} must be {expect[name]}, got {tuple(t.shape)}")
    for name, t in (("out", out), ("a8", a8), ("w1", w1), ("w2", w2), ("a1_scale", a1_scale),
                    ("fc1_scale", fc1_scale), ("fc2_scale", fc2_scale)):
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    sp = sorted_pairs
    for name, t, dt in (("sorted_ids", sp.sorted_ids, torch.int32), ("sorted_weights", sp.sorted_weights, torch.float32),
                        ("sorted_expert_ids", sp.sorted_expert_ids, torch.int32),
                        ("num_valid_ids", sp.num_valid_ids, torch.int32)):
        _cuda(t, dt, name)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if sp.sorted_weights.numel() < sp.capacity or sp.sorted_expert_ids.numel() < sp.capacity // sp.block_m:
        raise ValueError("sorted_weights / sorted_expert_ids shorter than the sorted list's capacity")
    return T, H, I, E


def fused_moe_fp8_blockscale_g1u1(out, a8, w1, w2, sorted_pairs: SortedPairs, topk, a1_scale, fc1_scale, fc2_scale,
                                  scale_blk_n=128, scale_blk_k=128, fc2_smooth_scale=None, workspace=None):
    """out bf16 [T, H] = fused g1u1 MoE (GEMM1 + SiLU*up + requant + GEMM2 + weighted combine).
    w1, w2 row-major ([E, 2I, H], [E, H, I]) or both tiled (fp8_tile_weights): the tiled
    ones take fused_moe_fp8_blockscale_g1u1_tiled."""
    T, H, I, E = _fused_moe_shapes(out, a8, w1, w2, sorted_pairs, topk, a1_scale, fc1_scale, fc2_scale)
    sp = sorted_pairs
    lib = load_library()
    if workspace is None:
        need = fused_moe_workspace_bytes(T, topk, E, H, I, sp.block_m, capacity=sp.capacity)
        workspace = torch.empty(need, dtype=torch.uint8, device=a8.device)
    name = "fused_moe_fp8_blockscale_g1u1_tiled" if is_tiled(w1) else "fused_moe_fp8_blockscale_g1u1"
    rc = getattr(lib, name)(
        _ptr(out), _ptr(a8), _ptr(w1), _ptr(w2), _ptr(sp.sorted_ids), _ptr(sp.sorted_weights),
        _ptr(sp.sorted_expert_ids), _ptr(sp.num_valid_ids), T, H, I, E, topk, sp.block_m, sp.capacity,
        _ptr(a1_scale), _ptr(fc1_scale), _ptr(fc2_scale), scale_blk_n, scale_blk_k, _ptr(fc2_smooth_scale),
        _ptr(workspace), workspace.numel(), _stream())
    _check(name, rc)
    return out


def fused_moe_fp8_blockscale_g1u1_noalloc(out, a8, w1, w2, sorted_pairs: SortedPairs, topk, a1_scale, fc1_scale,
                                          fc2_scale, scale_blk_n=128, scale_blk_k=128, fc2_smooth_scale=None):
    """fused_moe_fp8_blockscale_g1u1 using the library's built-in scratch (no workspace argument).

    For callers that cannot allocate device memory. Problems needing more than
    NOALLOC_SCRATCH_BYTES of scratch are rejected; calls share the scratch, so
    they must not overlap on the GPU. The arguments are checked exactly as for
    fused_moe_fp8_blockscale_g1u1.
    """
    T, H, I, E = _fused_moe_shapes(out, a8, w1, w2, sorted_pairs, topk, a1_scale, fc1_scale, fc2_scale)
    if is_tiled(w1):
        raise ValueError("the no-allocation entry point takes row-major weights")
    sp = sorted_pairs
    rc = load_library().fused_moe_fp8_blockscale_g1u1_noalloc(
        _ptr(out), _ptr(a8), _ptr(w1), _ptr(w2), _ptr(sp.sorted_ids), _ptr(sp.sorted_weights),
        _ptr(sp.sorted_expert_ids), _ptr(sp.num_valid_ids), T, H, I, E, topk, sp.block_m, sp.capacity,
        _ptr(a1_scale), _ptr(fc1_scale), _ptr(fc2_scale), scale_blk_n, scale_blk_k, _ptr(fc2_smooth_scale),
        _stream())
    _check("fused_moe_fp8_blockscale_g1u1_noalloc", rc)
    return out


# ---------------------------------------------------------------- tensor-parallel combine + all-reduce
def fused_moe_fp8_blockscale_g1u1_pairs(a8, w1, w2, sorted_pairs: SortedPairs, topk, a1_scale, fc1_scale, fc2_scale,
                                        workspace=None, scale_blk_n=128, scale_blk_k=128, fc2_smooth_scale=None):
    """The fused call without its combine (one tensor-parallel rank's share of I): the
    weighted pair rows and pair flags are left in the returned workspace for
    moe_combine_allreduce. Arguments and checks as fused_moe_fp8_blockscale_g1u1, minus out."""
    T, H, I, E = _fused_moe_shapes(None, a8, w1, w2, sorted_pairs, topk, a1_scale, fc1_scale, fc2_scale)
    sp = sorted_pairs
    if workspace is None:
        need = fused_moe_workspace_bytes(T, topk, E, H, I, sp.block_m, capacity=sp.capacity)
        workspace = torch.empty(need, dtype=torch.uint8, device=a8.device)
    rc = load_library().fused_moe_fp8_blockscale_g1u1_pairs(
        _ptr(a8), _ptr(w1), _ptr(w2), _ptr(sp.sorted_ids), _ptr(sp.sorted_weights), _ptr(sp.sorted_expert_ids),
        _ptr(sp.num_valid_ids), T, H, I, E, topk, sp.block_m, sp.capacity, _ptr(a1_scale), _ptr(fc1_scale),
        _ptr(fc2_scale), scale_blk_n, scale_blk_k, _ptr(fc2_smooth_scale), 1 if is_tiled(w1) else 0,
        _ptr(workspace), workspace.numel(), _stream())
    _check("fused_moe_fp8_blockscale_g1u1_pairs", rc)
    return workspace


def moe_tp_recv_bytes(T, H, nranks):
    """Bytes of one rank's receive buffer for moe_combine_allreduce."""
    return load_library().moe_tp_recv_bytes(T, H, nranks)


def _addresses(items, name):
    """A ctypes array of device addresses from tensors or plain integer addresses."""
    addrs = [t if isinstance(t, int) else t.data_ptr() for t in items]
    if any(a == 0 for a in addrs):
        raise ValueError(f"{name}: null address")
    return (ctypes.c_void_p * len(addrs))(*addrs)


def moe_combine_allreduce(workspace, capacity, T, topk, H, I, rank, recv, out, flags, barrier):
    """One tensor-parallel rank's fused combine + all-reduce (include/fp8moe.h). recv, out,
    flags: one device address (or tensor) per rank, as this GPU addresses that rank's buffer;
    barrier: int64 [TP_BARRIER_WORDS] on this GPU (it also counts the rank's calls)."""
    _cuda(workspace, torch.uint8, "workspace")
    _cuda(barrier, torch.int64, "barrier")
    n = len(recv)
    if not (len(out) == len(flags) == n) or not 1 <= n <= TP_MAX_RANKS:
        raise ValueError("recv, out and flags need one entry per rank (at most TP_MAX_RANKS)")
    if barrier.numel() < TP_BARRIER_WORDS:
        raise ValueError("barrier too small")
    rc = load_library().moe_combine_allreduce(
        _ptr(workspace), capacity, T, topk, H, I, n, rank, _addresses(recv, "recv"), _addresses(out, "out"),
        _addresses(flags, "flags"), _ptr(barrier), _stream())
    _check("moe_combine_allreduce", rc)


def moe_combine_allreduce_emulated(workspaces, capacity, T, topk, H, I, recv, out, flags, barriers):
    """Every rank of moe_combine_allreduce on this GPU in one launch (the rank protocol on one
    device). Per rank r: workspaces[r] (its pairs call's workspace), recv[r] bf16 [n, Ts, H],
    out[r] bf16 [T, H], flags[r] int64 [TP_FLAG_WORDS], barriers[r] int64 [TP_BARRIER_WORDS]."""
    n = len(workspaces)
    if not (len(recv) == len(out) == len(flags) == len(barriers) == n) or not 1 <= n <= TP_MAX_RANKS:
        raise ValueError("one workspace, recv, out, flags and barrier per rank (at most TP_MAX_RANKS)")
    Ts = -(-T // n)
    for r in range(n):
        _cuda(workspaces[r], torch.uint8, "workspaces")
        _cuda(recv[r], torch.bfloat16, "recv")
        _cuda(out[r], torch.bfloat16, "out")
        _cuda(flags[r], torch.int64, "flags")
        _cuda(barriers[r], torch.int64, "barriers")
        if recv[r].numel() < n * Ts * H or out[r].numel() < T * H or flags[r].numel() < TP_FLAG_WORDS \
                or barriers[r].numel() < TP_BARRIER_WORDS:
            raise ValueError(f"rank {r}: a buffer is smaller than the call needs")
    rc = load_library().moe_combine_allreduce_emulated(
        _addresses(workspaces, "workspaces"), capacity, T, topk, H, I, n, _addresses(recv, "recv"),
        _addresses(out, "out"), _addresses(flags, "flags"), _addresses(barriers, "barriers"), _stream())
    _check("moe_combine_allreduce_emulated", rc)


# ---------------------------------------------------------------- expert parallelism over peer memory
def moe_ep_routing(ids, w, Tq, topk, E, e0, ne, ids_out, w_out):
    """Every rank's routing as this owner's local ids (include/fp8moe.h). ids, w: one device
    address (or tensor) per rank; ids_out int32 / w_out fp32 [n*Tq, topk] on this GPU."""
    n = len(ids)
    if len(w) != n or not 1 <= n <= EP_MAX_RANKS:
        raise ValueError("one ids and one weights buffer per rank (at most EP_MAX_RANKS)")
    _cuda(ids_out, torch.int32, "ids_out")
    _cuda(w_out, torch.float32, "w_out")
    if ids_out.numel() < n * Tq * topk or w_out.numel() < n * Tq * topk:
        raise ValueError("ids_out / w_out smaller than n*Tq*topk")
    rc = load_library().moe_ep_routing(_addresses(ids, "ids"), _addresses(w, "w"), n, Tq, topk, E, e0, ne,
                                       _ptr(ids_out), _ptr(w_out), _stream())
    _check("moe_ep_routing", rc)


def fused_moe_fp8_blockscale_g1u1_multi(a8, a1_scale, Tq, H, w1, w2, sorted_pairs: SortedPairs, topk, fc1_scale,
                                        fc2_scale, workspace=None, return_rows=None, return_flags=None):
    """The owner's fused MoE over every rank's tokens (without the combine): a8[q] fp8 [Tq, H]
    and a1_scale[q] fp32 [H/128, Tq] of rank q, as addresses or tensors; the owner's weights;
    the sort over n*Tq tokens. return_rows / return_flags: int64 [n] device tensors holding
    every rank's return rows and pair-flag addresses, for the down GEMM to store each pair's
    row into its origin's buffer; without them the rows stay in the returned workspace."""
    n = len(a8)
    if (return_rows is None) != (return_flags is None):
        raise ValueError("return_rows and return_flags go together")
    if return_rows is not None:
        for name, t in (("return_rows", return_rows), ("return_flags", return_flags)):
            _cuda(t, torch.int64, name)
            if t.numel() != n or not t.is_contiguous():
                raise ValueError(f"{name} must hold one address per rank")
    if len(a1_scale) != n or not 1 <= n <= EP_MAX_RANKS:
        raise ValueError("one activation and one scale buffer per rank (at most EP_MAX_RANKS)")
    for name, t in (("w1", w1), ("w2", w2)):
        _cuda(t, FP8, name)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    E, twoI, H1 = _expert_matrix_shape(w1)
    E2, H2, I = _expert_matrix_shape(w2)
    if is_tiled(w1) != is_tiled(w2) or twoI != 2 * I or H1 != H or (E2, H2) != (E, H) or H % 128 or I % 128:
        raise ValueError(f"w1 {tuple(w1.shape)} and w2 {tuple(w2.shape)} do not form a g1u1 pair for H={H}")
    for name, t, shape in (("fc1_scale", fc1_scale, (E, 2 * I // 128, H // 128)),
                           ("fc2_scale", fc2_scale, (E, H // 128, I // 128))):
        _cuda(t, torch.float32, name)
        if tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {shape}")
    sp = sorted_pairs
    for name, t, dt in (("sorted_ids", sp.sorted_ids, torch.int32), ("sorted_weights", sp.sorted_weights, torch.float32),
                        ("sorted_expert_ids", sp.sorted_expert_ids, torch.int32),
                        ("num_valid_ids", sp.num_valid_ids, torch.int32)):
        _cuda(t, dt, name)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if workspace is None:
        need = fused_moe_workspace_bytes(n * Tq, topk, E, H, I, sp.block_m, capacity=sp.capacity)
        workspace = torch.empty(need, dtype=torch.uint8, device=w1.device)
    rc = load_library().fused_moe_fp8_blockscale_g1u1_multi(
        _addresses(a8, "a8"), _addresses(a1_scale, "a1_scale"), n, Tq, _ptr(w1), _ptr(w2), _ptr(sp.sorted_ids),
        _ptr(sp.sorted_weights), _ptr(sp.sorted_expert_ids), _ptr(sp.num_valid_ids), H, I, E, topk, sp.block_m,
        sp.capacity, _ptr(fc1_scale), _ptr(fc2_scale), 128, 128, None, 1 if is_tiled(w1) else 0, _ptr(return_rows),
        _ptr(return_flags), _ptr(workspace), workspace.numel(), _stream())
    _check("fused_moe_fp8_blockscale_g1u1_multi", rc)
    return workspace


def moe_ep_return(workspace, capacity, Tq, topk, H, I, sorted_pairs: SortedPairs, rows, pair_flags):
    """Each listed pair's weighted row into its origin's return rows, its flag set. rows,
    pair_flags: one address (or tensor) per rank."""
    n = len(rows)
    if len(pair_flags) != n or not 1 <= n <= EP_MAX_RANKS:
        raise ValueError("one rows and one flags buffer per rank (at most EP_MAX_RANKS)")
    _cuda(workspace, torch.uint8, "workspace")
    sp = sorted_pairs
    rc = load_library().moe_ep_return(_ptr(workspace), capacity, n, Tq, topk, H, I, _ptr(sp.sorted_ids),
                                      _ptr(sp.num_valid_ids), _addresses(rows, "rows"),
                                      _addresses(pair_flags, "pair_flags"), _stream())
    _check("moe_ep_return", rc)


def moe_ep_barrier(rank, words):
    """Flag barrier of len(words) ranks (include/fp8moe.h); words: one address (or int64
    tensor of EP_BARRIER_WORDS) per rank."""
    rc = load_library().moe_ep_barrier(len(words), rank, _addresses(words, "words"), _stream())
    _check("moe_ep_barrier", rc)


def moe_ep_barrier_emulated(words):
    rc = load_library().moe_ep_barrier_emulated(len(words), _addresses(words, "words"), _stream())
    _check("moe_ep_barrier_emulated", rc)


def moe_combine_pairs(rows, flag_region, T, topk, out):
    """out bf16 [T, H] = the combine over pair rows bf16 [T*topk, H] and their flag region
    (16-byte count, then one flag byte per pair)."""
    _cuda(rows, torch.bfloat16, "rows")
    _cuda(flag_region, torch.uint8, "flag_region")
    _cuda(out, torch.bfloat16, "out")
    H = out.shape[-1]
    if rows.numel() < T * topk * H or flag_region.numel() < 16 + T * topk or out.numel() < T * H:
        raise ValueError("rows, flag_region or out smaller than the call needs")
    rc = load_library().moe_combine_pairs(_ptr(rows), _ptr(flag_region), T, topk, H, _ptr(out), _stream())
    _check("moe_combine_pairs", rc)
    return out


def mla_decode_num_splits(batch, num_heads):
    """The split count mla_decode_fwd uses when num_kv_splits is not given."""
    return load_library().mla_decode_num_splits(batch, num_heads)


def mla_decode_workspace_bytes(batch, num_heads, num_kv_splits=0):
    return load_library().mla_decode_workspace(batch, num_heads, num_kv_splits)


def mla_decode_fwd(q, kv_buffer, o, kv_indptr, kv_indices, kv_last_page_lens, sm_scale=None, logit_cap=0.0,
                   num_kv_splits=0, lse=None, workspace=None):
    """MLA decode: o bf16 [B, Hq, 512] from q bf16 [B, Hq, 576] and the paged latent KV
    buffer bf16 [pages, page_size, 1, 576] (kv_indptr int32 [B+1], kv_indices int32,
    kv_last_page_lens int32 [B]). sm_scale defaults to 1/sqrt(576); lse (fp32 [B, Hq],
    optional) receives the log-sum-exp of the scores. Returns o."""
    _cuda(q, torch.bfloat16, "q")
    _cuda(kv_buffer, torch.bfloat16, "kv_buffer")
    _cuda(o, torch.bfloat16, "o")
    for t, name in ((kv_indptr, "kv_indptr"), (kv_indices, "kv_indices"), (kv_last_page_lens, "kv_last_page_lens")):
        _cuda(t, torch.int32, name)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if q.dim() != 3 or q.shape[2] != MLA_QK_HEAD_DIM or not q.is_contiguous():
        raise ValueError(f"q must be a contiguous [B, Hq, {MLA_QK_HEAD_DIM}] tensor")
    B, Hq = q.shape[0], q.shape[1]
    if kv_buffer.dim() != 4 or kv_buffer.shape[2] != 1 or kv_buffer.shape[3] != MLA_QK_HEAD_DIM \
            or not kv_buffer.is_contiguous():
        raise ValueError(f"kv_buffer must be a contiguous [pages, page_size, 1, {MLA_QK_HEAD_DIM}] tensor")
    if o.shape != (B, Hq, MLA_V_HEAD_DIM) or not o.is_contiguous():
        raise ValueError(f"o must be a contiguous [{B}, {Hq}, {MLA_V_HEAD_DIM}] tensor")
    if kv_indptr.numel() != B + 1 or kv_last_page_lens.numel() != B:
        raise ValueError("kv_indptr must hold B+1 entries and kv_last_page_lens B")
    if lse is not None:
        _cuda(lse, torch.float32, "lse")
        if lse.shape != (B, Hq) or not lse.is_contiguous():
            raise ValueError(f"lse must be a contiguous [{B}, {Hq}] tensor")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(MLA_QK_HEAD_DIM)
    need = mla_decode_workspace_bytes(B, Hq, num_kv_splits)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace is not None:
        _cuda(workspace, torch.uint8, "workspace")
    rc = load_library().mla_decode_fwd(
        _ptr(q), _ptr(kv_buffer), _ptr(o), _ptr(kv_indptr), _ptr(kv_indices), _ptr(kv_last_page_lens), _ptr(lse),
        B, Hq, kv_buffer.shape[0], kv_buffer.shape[1], kv_indices.numel(), float(sm_scale), float(logit_cap),
        int(num_kv_splits), _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream())
    _check("mla_decode_fwd", rc)
    return o
