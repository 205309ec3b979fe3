// Expert-parallel dispatch and return over peer memory.
//
// "Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang", section
// "Blockscale FP8 MoE Computation": asm_moe takes an expert_mask, the hook of
// expert parallelism (each GPU computes the pairs of the experts it holds).
//
// Rank r of n holds experts [e0, e0 + ne) and its own Tq tokens. Every rank first
// publishes, in memory the other GPUs can address, its routing (top-k ids and
// weights), its FP8 activations and their scales, and zeroes the pair flags of
// its return buffer; a flag barrier follows. Then each rank, as an owner:
//   1. ep_routing_kernel reads every rank's routing (global token g = q*Tq + t)
//      and maps each id to the owner's local id (another rank's expert becomes
//      the sentinel ne, which the owner's masked sort drops);
//   2. the owner's sort and fused MoE run over the n*Tq global tokens; its gather
//      reads each listed pair's activation row and scales where they lie
//      (moe_gather_*_kernel with GatherSources), the GEMMs read the local weights,
//      and the weighted pair rows land in the owner's workspace by global pair id;
//   3. ep_return_kernel stores each listed pair's row into the return buffer of
//      the pair's origin, at the origin's own pair id, and sets its flag byte.
// After a second barrier every rank's return buffer holds all its pairs' rows, and
// the ordinary combine (moe_combine_kernel, flags read) gives exactly the
// one-GPU layer's output for that rank's tokens.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "moe_aux.cuh"
#include "tp_reduce.cuh"

namespace fp8moe {

struct EpRouting {
  const int32_t* ids[kMaxSources];   // [Tq, K] top-k expert ids of rank q
  const float* w[kMaxSources];       // [Tq, K] routing weights of rank q
};

// ids_out / w_out [n*Tq, K]: the owner's view of every rank's pairs. An id of the
// owner's experts becomes id - e0, another valid id the sentinel ne, an invalid
// one stays out of range (the sort drops and flags it).
__global__ void __launch_bounds__(256)
ep_routing_kernel(const __grid_constant__ EpRouting src, int n, int Tq, int K, int E, int e0, int ne, int32_t* __restrict__ ids_out,
                  float* __restrict__ w_out) {
  const long long per = static_cast<long long>(Tq) * K;
  const long long total = per * n;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int q = static_cast<int>(i / per);
    const long long li = i - q * per;
    const int id = __ldcg(src.ids[q] + li);
    int local;
    if (id < 0 || id >= E)
      local = -1;
    else if (id >= e0 && id < e0 + ne)
      local = id - e0;
    else
      local = ne;
    ids_out[i] = local;
    w_out[i] = __ldcg(src.w[q] + li);
  }
}

struct EpReturn {
  __nv_bfloat16* rows[kMaxSources];   // rank q's return rows [Tq*K, H]
  uint8_t* flags[kMaxSources];         // rank q's pair flags [Tq*K]
};

// One warp per sorted slot: a listed pair p = q*Tq*K + lp has its weighted row
// ystage[p] stored into rank q's return row lp, and its flag set.
__global__ void __launch_bounds__(256)
ep_return_kernel(const int32_t* __restrict__ sorted_ids, const int32_t* __restrict__ num_valid_ids, int cap,
                 const __nv_bfloat16* __restrict__ ystage, int n, int Pq, int H,
                 const __grid_constant__ EpReturn dst) {
  const int lane = threadIdx.x & 31;
  const int nv = min(max(*num_valid_ids, 0), cap);
  const int vec = H / 8;
  const long long P = static_cast<long long>(Pq) * n;
  for (int slot = blockIdx.x * 8 + (threadIdx.x >> 5); slot < nv; slot += gridDim.x * 8) {
    const int p = sorted_ids[slot];
    if (p < 0 || p >= P) continue;
    const int q = p / Pq, lp = p - q * Pq;
    const uint4* srow = reinterpret_cast<const uint4*>(ystage + static_cast<size_t>(p) * H);
    uint4* drow = reinterpret_cast<uint4*>(dst.rows[q] + static_cast<size_t>(lp) * H);
    for (int v = lane; v < vec; v += 32) drow[v] = __ldcs(srow + v);
    if (lane == 0) dst.flags[q][lp] = 1;
  }
}

// Flag barrier of n ranks: rank r publishes epoch (its own count of barrier calls
// plus one, kept in word kMaxSources of its words, so a CUDA graph replay advances
// it like a launch) in every rank's word r (release, system scope), then waits
// until its own words q hold >= epoch for every q. The stream order before it makes
// every earlier store of this rank (peer stores included) visible to the ranks
// that pass it. Bounded: on expiry the device error word is set. One CTA (one
// warp) per rank: rank = rank_first + blockIdx.x.
constexpr int kEpBarrierWords = kMaxSources + 1;
struct EpBarrierArgs {
  unsigned long long* flags[kMaxSources];   // rank p's barrier words [kEpBarrierWords]
  int n;
};

__global__ void __launch_bounds__(32) ep_barrier_kernel(const __grid_constant__ EpBarrierArgs a, int rank_first) {
  const int rank = rank_first + static_cast<int>(blockIdx.x);
  unsigned long long epoch = 0;
  if (threadIdx.x == 0) epoch = ld_acquire_gpu_u64(a.flags[rank] + kMaxSources) + 1;
  epoch = __shfl_sync(0xffffffffu, epoch, 0);
  __threadfence_system();
  if (threadIdx.x < a.n) st_release_sys_u64(a.flags[threadIdx.x] + rank, epoch);
  if (threadIdx.x < a.n) tp_wait_ge(a.flags[rank] + threadIdx.x, epoch);
  __syncwarp();
  if (threadIdx.x == 0) atomicExch(a.flags[rank] + kMaxSources, epoch);
  __threadfence_system();
}

}  // namespace fp8moe
