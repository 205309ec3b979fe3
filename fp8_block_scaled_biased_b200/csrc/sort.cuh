// MoE align/sort of token-expert pairs into block_m-padded per-expert segments.
//
// "Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang", section
// "MoE Sorting" (moe_sorting -> sorted_token_ids, sorted_weight_buf,
// sorted_expert_ids, num_valid_ids). Layout: pair (t, k) is the flat id
// p = t*topk + k; experts ascending, pairs ascending inside an expert, each
// segment padded to a multiple of block_m with id T*topk and weight 0; one
// expert id per block; experts without pairs get no block.
//
// One CTA does it all: a shared-memory histogram, a scan over experts, then a
// stable scatter in chunks of 1024 pairs (one per thread) in which a pair's
// slot is its expert's running base + the count of same-expert pairs in lower
// warps of the chunk + its rank among same-expert lanes of its warp.
#pragma once

#include "common.cuh"

namespace fp8moe {

constexpr int kSortThreads = 1024;
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kSortMaxExperts = 1024;

__device__ __forceinline__ int read_pair_expert(const int32_t* ids, int ld, int K, int p, int E) {
  const int t = p / K, k = p - t * K;
  const int e = ids[static_cast<size_t>(t) * ld + k];
  return (e >= 0 && e < E) ? e : -1;
}

// dynamic shared memory: cnt[E] | base[E] | warp_cnt[kSortWarps][E]
__global__ void __launch_bounds__(kSortThreads, 1)
align_sort_kernel(const int32_t* __restrict__ ids, const float* __restrict__ w, int ld, int T, int K, int E,
                  int block_m, int32_t* __restrict__ sorted_ids, float* __restrict__ sorted_w,
                  int32_t* __restrict__ sorted_e, int32_t* __restrict__ num_valid) {
  extern __shared__ int sm_sort[];
  int* cnt = sm_sort;
  int* base = cnt + E;
  int* warp_cnt = base + E;
  __shared__ int s_bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int P = T * K;

  for (int e = tid; e < E; e += kSortThreads) cnt[e] = 0;
  if (tid == 0) s_bad = 0;
  __syncthreads();

  // 1. histogram
  for (int p = tid; p < P; p += kSortThreads) {
    const int e = read_pair_expert(ids, ld, K, p, E);
    if (e >= 0)
      atomicAdd(&cnt[e], 1);
    else
      s_bad = 1;
  }
  __syncthreads();

  // 2. padded segment starts (exclusive scan of ceil(cnt/bm)*bm over experts, by warp 0)
  if (warp == 0) {
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int c = (e < E) ? cnt[e] : 0;
      const int len = (c + block_m - 1) / block_m * block_m;
      int incl = len;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (e < E) base[e] = carry + incl - len;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      *num_valid = carry;
      if (s_bad) raise_device_error(FP8MOE_DEVERR_EXPERT_ID);
    }
  }
  __syncthreads();

  // 3. block expert ids and padding slots
  for (int e = warp; e < E; e += kSortWarps) {
    const int c = cnt[e];
    const int start = base[e];
    const int len = (c + block_m - 1) / block_m * block_m;
    for (int j = lane; j < len / block_m; j += 32) sorted_e[start / block_m + j] = e;
    for (int s = start + c + lane; s < start + len; s += 32) {
      sorted_ids[s] = P;
      sorted_w[s] = 0.0f;
    }
  }

  // 4. stable scatter, 1024 pairs per round
  for (int c0 = 0; c0 < P; c0 += kSortThreads) {
    const int p = c0 + tid;
    const int e = (p < P) ? read_pair_expert(ids, ld, K, p, E) : -1;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(same & ((1u << lane) - 1u));
    for (int i = tid; i < kSortWarps * E; i += kSortThreads) warp_cnt[i] = 0;
    __syncthreads();
    if (e >= 0 && rank == 0) warp_cnt[warp * E + e] = __popc(same);
    __syncthreads();
    // per expert: exclusive prefix over warps, from the expert's running base
    for (int ex = tid; ex < E; ex += kSortThreads) {
      int run = base[ex];
      for (int wi = 0; wi < kSortWarps; ++wi) {
        const int v = warp_cnt[wi * E + ex];
        warp_cnt[wi * E + ex] = run;
        run += v;
      }
      base[ex] = run;
    }
    __syncthreads();
    if (e >= 0) {
      const int slot = warp_cnt[warp * E + e] + rank;
      const int t = p / K, k = p - t * K;
      sorted_ids[slot] = p;
      sorted_w[slot] = w[static_cast<size_t>(t) * ld + k];
    }
    __syncthreads();
  }
}

}  // namespace fp8moe
