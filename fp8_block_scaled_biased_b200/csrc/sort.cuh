// MoE align/sort of token-expert pairs into block_m-padded per-expert segments.
//
// "Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang", section
// "MoE Sorting" (moe_sorting -> sorted_token_ids, sorted_weight_buf,
// sorted_expert_ids, num_valid_ids). Layout: pair (t, k) is the flat id
// p = t*topk + k; experts ascending, pairs ascending inside an expert, each
// segment padded to a multiple of block_m with id T*topk and weight 0; one
// expert id per block; experts without pairs get no block. An optional expert
// mask (the expert_mask argument of the page's asm_moe call: the experts this
// GPU holds under expert parallelism) drops the pairs of masked-out experts.
//
// Two kernels over chunks of kSortChunk consecutive pairs (one CTA each):
//   1. sort_count_kernel: per-chunk expert histogram -> counts[chunk][E];
//   2. sort_scatter_kernel: each CTA reads all chunks' counts and derives, for
//      every expert, the pairs in earlier chunks and the padded segment start
//      (a block-wide scan); it writes the block expert ids and padding of a
//      share of the experts (CTA 0 also num_valid_ids), then the stable rank of
//      each of its pairs (count of same-expert pairs in lower warps + rank among
//      same-expert lanes of its warp) added to its expert's first slot for the
//      chunk.
// Stable by construction: no atomics decide an order.
#pragma once

#include "common.cuh"

namespace fp8moe {

constexpr int kSortChunk = 1024;                 // pairs per CTA = threads per CTA
constexpr int kSortWarps = kSortChunk / 32;
constexpr int kSortMaxExperts = 1024;
static_assert(kSortMaxExperts <= kSortChunk, "the segment-start scan takes one expert per thread");
static_assert(kSortWarps == 32, "block_exclusive_scan combines one partial per lane of warp 0");

// Expert of pair p: kDropInvalid for an id outside [0, E) (flagged by the
// caller), kDropMasked for an expert that mask (if any) excludes.
constexpr int kDropInvalid = -1;
constexpr int kDropMasked = -2;
__device__ __forceinline__ int read_pair_expert(const int32_t* ids, int ld, int K, int p, int E,
                                                const int32_t* mask) {
  const int t = p / K, k = p - t * K;
  const int e = ids[static_cast<size_t>(t) * ld + k];
  if (e < 0 || e >= E) return kDropInvalid;
  return (mask && mask[e] == 0) ? kDropMasked : e;
}

// 1. counts[c][e] = pairs of chunk c routed to expert e.
__global__ void __launch_bounds__(kSortChunk)
sort_count_kernel(const int32_t* __restrict__ ids, int ld, int T, int K, int E, const int32_t* __restrict__ mask,
                  int32_t* __restrict__ counts) {
  extern __shared__ int sm_cnt[];
  const int P = T * K;
  for (int e = threadIdx.x; e < E; e += kSortChunk) sm_cnt[e] = 0;
  __syncthreads();
  const int p = blockIdx.x * kSortChunk + threadIdx.x;
  if (p < P) {
    const int e = read_pair_expert(ids, ld, K, p, E, mask);
    if (e >= 0)
      atomicAdd(&sm_cnt[e], 1);
    else if (e == kDropInvalid)
      raise_device_error(FP8MOE_DEVERR_EXPERT_ID);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kSortChunk) counts[static_cast<size_t>(blockIdx.x) * E + e] = sm_cnt[e];
}

// Exclusive scan over a block of kSortChunk threads (one value each); returns
// the exclusive prefix of v and writes the total to *total_out (shared). Uses
// warp_sums[kSortWarps] of shared memory.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total_out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int ws = warp_sums[lane];          // kSortWarps == 32
    int wincl = ws;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, wincl, off);
      if (lane >= off) wincl += o;
    }
    warp_sums[lane] = wincl - ws;
    if (lane == 31) *total_out = wincl;
  }
  __syncthreads();
  return warp_sums[warp] + incl - v;
}

// Dynamic shared memory of sort_scatter_kernel for E experts.
__host__ __device__ constexpr size_t sort_scatter_smem(int E) {
  return (static_cast<size_t>(kSortWarps + 3) * E + kSortWarps + 1) * sizeof(int);
}

// 2. Offsets and stable scatter of chunk blockIdx.x.
// Shared memory: warp_cnt[kSortWarps][E], total[E], start[E], before[E], 33 ints.
__global__ void __launch_bounds__(kSortChunk)
sort_scatter_kernel(const int32_t* __restrict__ ids, const float* __restrict__ w, int ld, int T, int K, int E,
                    const int32_t* __restrict__ mask, int block_m, const int32_t* __restrict__ counts, int nchunks,
                    int32_t* __restrict__ sorted_ids, float* __restrict__ sorted_w, int32_t* __restrict__ sorted_e,
                    int32_t* __restrict__ num_valid) {
  extern __shared__ int sm_scatter[];
  int* warp_cnt = sm_scatter;                       // [kSortWarps][E]
  int* total = warp_cnt + kSortWarps * E;           // [E] pairs per expert
  int* start = total + E;                           // [E] padded segment start
  int* before = start + E;                          // [E] expert's pairs in earlier chunks
  int* scan_tmp = before + E;                       // [kSortWarps + 1]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int P = T * K;
  const int chunk = blockIdx.x;
  // per expert: pairs in chunks before this one and in all chunks (eight loads in flight)
  for (int e = tid; e < E; e += kSortChunk) {
    int run = 0, mine = 0;
    for (int c0 = 0; c0 < nchunks; c0 += 8) {
      int v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = (c0 + i < nchunks) ? counts[static_cast<size_t>(c0 + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (c0 + i == chunk) mine = run;
        run += v[i];
      }
    }
    total[e] = run;
    before[e] = mine;
  }
  __syncthreads();
  // padded segment starts: exclusive scan of ceil(total/bm)*bm over experts (E <= kSortChunk)
  {
    const int len = (tid < E) ? (total[tid] + block_m - 1) / block_m * block_m : 0;
    const int ex = block_exclusive_scan(len, scan_tmp, &scan_tmp[kSortWarps]);
    if (tid < E) start[tid] = ex;
    __syncthreads();
  }
  if (chunk == 0 && tid == 0) *num_valid = scan_tmp[kSortWarps];
  // block expert ids and padding slots of this CTA's share of the experts
  for (int ex = chunk + warp * nchunks; ex < E; ex += kSortWarps * nchunks) {
    const int c = total[ex];
    const int s0 = start[ex];
    const int len = (c + block_m - 1) / block_m * block_m;
    for (int j = lane; j < len / block_m; j += 32) sorted_e[s0 / block_m + j] = ex;
    for (int sl = s0 + c + lane; sl < s0 + len; sl += 32) {
      sorted_ids[sl] = P;
      sorted_w[sl] = 0.0f;
    }
  }
  // stable scatter of this chunk's pairs
  const int p = chunk * kSortChunk + tid;
  const int e = (p < P) ? read_pair_expert(ids, ld, K, p, E, mask) : kDropInvalid;
  float wv = 0.0f;
  if (e >= 0) {
    const int t = p / K, k = p - t * K;
    wv = w[static_cast<size_t>(t) * ld + k];
  }
  const unsigned same = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(same & ((1u << lane) - 1u));
  for (int i = tid; i < kSortWarps * E; i += kSortChunk) warp_cnt[i] = 0;
  __syncthreads();
  if (e >= 0 && rank == 0) warp_cnt[warp * E + e] = __popc(same);
  __syncthreads();
  // per expert: exclusive prefix over the warps of this chunk, from the chunk's first slot
  for (int ex = tid; ex < E; ex += kSortChunk) {
    int run = start[ex] + before[ex];
    for (int wi = 0; wi < kSortWarps; ++wi) {
      const int v = warp_cnt[wi * E + ex];
      warp_cnt[wi * E + ex] = run;
      run += v;
    }
  }
  __syncthreads();
  if (e >= 0) {
    const int slot = warp_cnt[warp * E + e] + rank;
    sorted_ids[slot] = p;
    sorted_w[slot] = wv;
  }
}

// Both steps in one CTA when the pairs fit one chunk (P <= kSortChunk, a
// decode-sized batch): the chunk histogram is the per-warp counts summed, the
// segment starts come from it directly, and there are no earlier chunks.
// Shared memory: total[E], start[E], warp_cnt[kSortWarps][E].
__global__ void __launch_bounds__(kSortChunk)
sort_small_kernel(const int32_t* __restrict__ ids, const float* __restrict__ w, int ld, int T, int K, int E,
                  const int32_t* __restrict__ mask, int block_m, int32_t* __restrict__ sorted_ids, float* __restrict__ sorted_w,
                  int32_t* __restrict__ sorted_e, int32_t* __restrict__ num_valid) {
  extern __shared__ int sm_small[];
  int* total = sm_small;
  int* start = sm_small + E;
  int* warp_cnt = sm_small + 2 * E;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int P = T * K;
  for (int i = tid; i < E; i += kSortChunk) total[i] = 0;
  for (int i = tid; i < kSortWarps * E; i += kSortChunk) warp_cnt[i] = 0;
  __syncthreads();
  const int p = tid;
  int e = kDropInvalid;
  float wv = 0.0f;
  if (p < P) {
    e = read_pair_expert(ids, ld, K, p, E, mask);
    if (e >= 0) {
      const int t = p / K, k = p - t * K;
      wv = w[static_cast<size_t>(t) * ld + k];
    } else if (e == kDropInvalid) {
      raise_device_error(FP8MOE_DEVERR_EXPERT_ID);
    }
  }
  const unsigned same = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(same & ((1u << lane) - 1u));
  if (e >= 0 && rank == 0) {
    warp_cnt[warp * E + e] = __popc(same);
    atomicAdd(&total[e], __popc(same));
  }
  __syncthreads();
  // padded segment starts: exclusive scan of ceil(total/bm)*bm over experts (warp 0)
  if (warp == 0) {
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int ex = e0 + lane;
      const int len = (ex < E) ? (total[ex] + block_m - 1) / block_m * block_m : 0;
      int incl = len;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (ex < E) start[ex] = carry + incl - len;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) *num_valid = carry;
  }
  __syncthreads();
  // per expert: each warp's first slot (exclusive prefix over warps from the segment start)
  for (int ex = tid; ex < E; ex += kSortChunk) {
    int run = start[ex];
    for (int wi = 0; wi < kSortWarps; ++wi) {
      const int v = warp_cnt[wi * E + ex];
      warp_cnt[wi * E + ex] = run;
      run += v;
    }
  }
  // block expert ids and padding slots
  for (int ex = warp; ex < E; ex += kSortWarps) {
    const int c = total[ex];
    const int s0 = start[ex];
    const int len = (c + block_m - 1) / block_m * block_m;
    for (int j = lane; j < len / block_m; j += 32) sorted_e[s0 / block_m + j] = ex;
    for (int sl = s0 + c + lane; sl < s0 + len; sl += 32) {
      sorted_ids[sl] = P;
      sorted_w[sl] = 0.0f;
    }
  }
  __syncthreads();
  if (e >= 0) {
    const int slot = warp_cnt[warp * E + e] + rank;
    sorted_ids[slot] = p;
    sorted_w[slot] = wv;
  }
}

}  // namespace fp8moe
