// The MoE layer's memory-bound steps around the two grouped GEMMs.
//
// "Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang", section
// "Blockscale FP8 MoE Computation": the fused MoE reads the sorted token-expert
// slots (moe_sorting) and writes the top-k weighted sum per token (moe_buf).
// moe_gather_kernel and moe_gather_rows_kernel put each slot's FP8 activation
// row and scales into slot order for the gate/up GEMM's TMA loads;
// moe_combine_kernel sums a token's topk weighted down-projection rows in a
// fixed order.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace fp8moe {

constexpr int kMoeBlockRows = 128;            // rows per sorted block (the GEMM tile's M)

constexpr int kGatherWarps = 8;

// The activations of several GPUs' tokens, read where they lie (expert parallelism:
// the GPU that owns an expert gathers the rows of every GPU's tokens routed to it).
// Global token g is token g % Tq of source g / Tq; the pointers are as this GPU
// addresses each source's memory (peer memory over NVLink, or local).
constexpr int kMaxSources = 8;
struct GatherSources {
  const uint8_t* a8[kMaxSources];        // fp8 [Tq, H]
  const float* a1_scale[kMaxSources];    // fp32 [H/128, Tq]
  int n, Tq;
};
// Slot-ordered pass over the sorted list: sets pair_flag[p] = 1 for every listed
// pair p and adds the number of distinct listed pairs to *n_present (the caller
// zeroes both first; pair_flag is 4-byte aligned; a pair id listed twice, which
// moe_align_sort never produces, is counted once, so *n_present == T*topk means
// every pair is present), writes the pair -> slot map inv[p] (valid where the
// flag is set) and copies each slot's H/128 scales from a1_scale [H/128, T] into
// slot order. Padding slots are skipped: the GEMMs treat rows independently and
// never store padding rows.
// MULTI: the scales of token t come from its source (src), not from a1_scale.
template <bool MULTI = false>
__global__ void __launch_bounds__(32 * kGatherWarps)
moe_gather_kernel(const float* __restrict__ a1_scale, const int32_t* __restrict__ sorted_ids,
                  const int32_t* __restrict__ sorted_expert_ids, const int32_t* __restrict__ num_valid_ids, int T,
                  int topk, int H, int cap, float* __restrict__ s1s, uint8_t* __restrict__ pair_flag,
                  int* __restrict__ n_present, int* __restrict__ inv,
                  const __grid_constant__ GatherSources src = {}) {
  __shared__ int cta_present;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) cta_present = 0;
  __syncthreads();
  int present = 0;
  const int P = T * topk;
  const int nv = min(max(*num_valid_ids, 0), cap);
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b + 1 < nv / kMoeBlockRows; b += gridDim.x * blockDim.x)
    if (sorted_expert_ids[b] > sorted_expert_ids[b + 1]) raise_device_error(FP8MOE_DEVERR_BLOCK_ORDER);
  const int KB = H / 128;
  for (int slot = blockIdx.x * blockDim.x + threadIdx.x; slot < nv; slot += gridDim.x * blockDim.x) {
    const int sid = sorted_ids[slot];
    if (sid < 0 || sid >= P) continue;
    const unsigned bit = 1u << (8 * (sid & 3));
    if ((atomicOr(reinterpret_cast<unsigned*>(pair_flag) + (sid >> 2), bit) & bit) == 0) ++present;
    inv[sid] = slot;
  }
  present = __reduce_add_sync(0xffffffffu, present);
  if (lane == 0 && present) atomicAdd(&cta_present, present);
  __syncthreads();
  if (threadIdx.x == 0 && cta_present) atomicAdd(n_present, cta_present);
  const int nwarps = gridDim.x * kGatherWarps;
  for (int s0 = (blockIdx.x * kGatherWarps + (threadIdx.x >> 5)) * 32; s0 < nv; s0 += nwarps * 32) {
    const int slot = s0 + lane;
    const int sid = slot < nv ? sorted_ids[slot] : -1;
    if (sid < 0 || sid >= P) continue;
    const int t = sid / topk;
    if constexpr (MULTI) {
      const int q = t / src.Tq, lt = t - q * src.Tq;
      const float* sc = src.a1_scale[q];
      for (int kb = 0; kb < KB; ++kb)
        __stcs(&s1s[static_cast<size_t>(kb) * cap + slot], __ldcg(sc + static_cast<size_t>(kb) * src.Tq + lt));
    } else {
      for (int kb = 0; kb < KB; ++kb)
        __stcs(&s1s[static_cast<size_t>(kb) * cap + slot], __ldg(a1_scale + static_cast<size_t>(kb) * T + t));
    }
  }
}

// Token-ordered pass: each token's FP8 row of a8 [T, H] is read once and written
// to the slot of each of its listed pairs. Going by token rather than by slot
// keeps a8 from being re-read topk times from memory once the slot-ordered
// writes have pushed it out of L2. A warp takes one 2 KB chunk of one token's row
// (so that a small batch still spreads over the GPU); stores are marked
// evict-first.
constexpr int kRowChunkVec = 4;               // 16-byte vectors per lane per chunk
// MULTI: token t's row comes from its source (src), not from a8.
template <bool MULTI = false>
__global__ void __launch_bounds__(32 * kGatherWarps)
moe_gather_rows_kernel(const uint8_t* __restrict__ a8, int T, int topk, int H,
                       const uint8_t* __restrict__ pair_flag, const int* __restrict__ inv,
                       uint8_t* __restrict__ a8s,
                       const __grid_constant__ GatherSources src = {}) {
  const int lane = threadIdx.x & 31;
  const int vec_per_row = H / 16;
  const int chunks = (vec_per_row + 32 * kRowChunkVec - 1) / (32 * kRowChunkVec);
  const long long units = static_cast<long long>(T) * chunks;
  for (long long u = static_cast<long long>(blockIdx.x) * kGatherWarps + (threadIdx.x >> 5); u < units;
       u += static_cast<long long>(gridDim.x) * kGatherWarps) {
    const int t = static_cast<int>(u / chunks);
    const int v0 = static_cast<int>(u % chunks) * 32 * kRowChunkVec;
    int slot_k = -1;
    if (lane < topk) {
      const int p = t * topk + lane;
      if (pair_flag[p]) slot_k = inv[p];
    }
    if (__ballot_sync(0xffffffffu, slot_k >= 0) == 0) continue;   // no listed pair: the row is not read
    uint4 buf[kRowChunkVec];
    if constexpr (MULTI) {
      const int q = t / src.Tq;
      const uint4* row = reinterpret_cast<const uint4*>(src.a8[q] + static_cast<size_t>(t - q * src.Tq) * H);
#pragma unroll
      for (int i = 0; i < kRowChunkVec; ++i) {
        const int v = v0 + i * 32 + lane;
        if (v < vec_per_row) buf[i] = __ldcg(row + v);
      }
    } else {
      const uint4* row = reinterpret_cast<const uint4*>(a8 + static_cast<size_t>(t) * H);
#pragma unroll
      for (int i = 0; i < kRowChunkVec; ++i) {
        const int v = v0 + i * 32 + lane;
        if (v < vec_per_row) buf[i] = __ldg(row + v);
      }
    }
    for (int k = 0; k < topk; ++k) {
      const int slot = __shfl_sync(0xffffffffu, slot_k, k);
      if (slot < 0) continue;
      uint4* dst = reinterpret_cast<uint4*>(a8s + static_cast<size_t>(slot) * H);
#pragma unroll
      for (int i = 0; i < kRowChunkVec; ++i) {
        const int v = v0 + i * 32 + lane;
        if (v < vec_per_row) __stcs(dst + v, buf[i]);
      }
    }
  }
}

// out[t, :] = bf16( y[t*K + 0] + y[t*K + 1] + ... + y[t*K + K-1] ), fp32 adds in
// slot order k over the pairs whose flag is set (the routing weight is already
// in y; a pair absent from the sorted list has no row). When every pair is
// listed (*n_present, the count of distinct listed pairs, equals T*K: one cached
// load) the flags are not read. One thread per 8 columns; the rows are read once,
// with evict-first loads.
__global__ void __launch_bounds__(256)
moe_combine_kernel(const __nv_bfloat16* __restrict__ ystage, const uint8_t* __restrict__ pair_flag,
                   const int* __restrict__ n_present, int T, int K, int H, __nv_bfloat16* __restrict__ out) {
  const int cpr = H / 8;
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<size_t>(T) * cpr) return;
  const int t = static_cast<int>(idx / cpr);
  const int c = static_cast<int>(idx % cpr) * 8;
  const __nv_bfloat16* y = ystage + static_cast<size_t>(t) * K * H + c;
  float sum[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) sum[i] = 0.0f;
  // fp32 sum in k order (0.0f + y0 == y0 exactly, so the order is fixed from the first term)
  auto add_row = [&](int k) {
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(y + static_cast<size_t>(k) * H));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[u]));
      sum[2 * u] += f.x;
      sum[2 * u + 1] += f.y;
    }
  };
  if (*n_present == T * K) {
    for (int k = 0; k < K; ++k) add_row(k);
  } else {
    for (int k = 0; k < K; ++k)
      if (pair_flag[static_cast<size_t>(t) * K + k]) add_row(k);
  }
  __align__(16) __nv_bfloat162 pk[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) pk[u] = __floats2bfloat162_rn(sum[2 * u], sum[2 * u + 1]);
  *reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H + c) = *reinterpret_cast<const uint4*>(pk);
}

}  // namespace fp8moe
