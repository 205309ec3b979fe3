// The MoE combine fused with the tensor-parallel all-reduce, over peer memory.
//
// "Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang": the layer runs
// at TP8 (section "Performance Reproduction for AITER-Optimized in SGLang",
// --tp 8) and the ranks' outputs are summed by a custom all-reduce (section
// "Other Operators"). Under tensor parallelism over I every rank holds, for every
// token, its weighted down-projection rows (one per top-k pair, the fused call's
// pair rows) over its share of I; the layer output is the sum of those rows over
// the pairs and the ranks.
//
// One kernel per rank (rank r of n, token slice s(p) = [p*Ts, (p+1)*Ts), Ts =
// ceil(T/n)):
//   1. combine: for each token t, the fp32 sum of its listed pair rows in k order,
//      rounded to bf16 once, is stored into the receive buffer of the rank p that
//      owns t's slice (recv_p[r][t - p*Ts], a store over NVLink when p != r);
//   2. the rank's CTAs meet at a barrier (in this GPU's memory), then one thread
//      publishes flag_p[0][r] = epoch to every rank p (release, system scope),
//      epoch being the rank's call count plus one (a counter kept in its barrier
//      words, so that no value comes from the host and a CUDA graph replay of the
//      call advances it like a launch does);
//   3. each rank waits for flag_r[0][q] >= epoch from every q (acquire, system
//      scope), then sums its slice's n partial rows in rank order q = 0..n-1 in
//      fp32, rounds to bf16 once and stores the row into every rank's output
//      (the all-gather, again over NVLink);
//   4. a second barrier and flag_p[1][r] = epoch; the kernel ends once every rank
//      has written this rank's output (flag_r[1][q] >= epoch for all q).
// The result is bitwise identical on every rank and deterministic: the reduction
// order is fixed (pairs in k order within a rank, then ranks in order).
//
// Waits are bounded (kWaitLimitNs): on expiry the kernel flags
// FP8MOE_DEVERR_TIMEOUT and carries on without waiting, so a missing rank ends in
// an error status, not a hang. Every CTA of a rank must be resident at once (the
// barrier spins), so the kernel goes out as a cooperative launch. The same kernel
// runs every rank of a group on one GPU (rank_first = 0, grid = n x CTAs per
// rank) with all buffers in that GPU's memory: the emulation the tests use.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace fp8moe {

constexpr int kTpMaxRanks = 8;
constexpr int kTpThreads = 256;
constexpr int kTpFlagWords = 2 * kTpMaxRanks;   // per rank: [phase][source rank]
constexpr int kTpBarrierWords = 3;               // per rank: arrivals, generation, calls
constexpr int kTpBatch = 4;                      // pair rows loaded before they are added

struct TpArgs {
  // per rank, in that rank's GPU memory (only [rank] is read by a one-rank launch)
  const __nv_bfloat16* ystage[kTpMaxRanks];   // weighted pair rows [T*K, H]
  const uint8_t* pair_flag[kTpMaxRanks];       // [T*K]: 1 where the pair is listed
  const int* n_present[kTpMaxRanks];           // distinct listed pairs
  unsigned long long* barrier[kTpMaxRanks];    // {arrivals, generation, calls}
  // per rank p, as this GPU addresses it (peer memory for p != own rank)
  __nv_bfloat16* recv[kTpMaxRanks];            // [n][Ts][H]
  __nv_bfloat16* out[kTpMaxRanks];             // [T][H]
  unsigned long long* flags[kTpMaxRanks];      // [kTpFlagWords]
  int nranks, T, K, H;
};

__device__ __forceinline__ void st_release_sys_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.sys.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_sys_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Waits until *p >= want (bounded); false on expiry (the device error word is set).
__device__ __forceinline__ bool tp_wait_ge(const unsigned long long* p, unsigned long long want) {
  if (ld_acquire_sys_u64(p) >= want) return true;
  const unsigned long long t0 = global_timer_ns();
  while (ld_acquire_sys_u64(p) < want) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      raise_device_error(FP8MOE_DEVERR_TIMEOUT);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

// All `ctas` CTAs of one rank meet; each thread's earlier global stores (peer
// memory included) are visible system-wide when any CTA leaves. A reusable
// generation barrier: the last arrival resets the count, then advances the
// generation. Bounded like every wait.
__device__ __forceinline__ void tp_rank_barrier(unsigned long long* bar, int ctas) {
  __threadfence_system();
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long* count = bar;
    unsigned long long* gen = bar + 1;
    const unsigned long long g = ld_acquire_gpu_u64(gen);   // before arriving: the last arrival moves it
    __threadfence_system();   // cumulative over the stores the CTA made before __syncthreads
    if (atomicAdd(count, 1ull) == static_cast<unsigned long long>(ctas - 1)) {
      atomicExch(count, 0ull);
      __threadfence_system();
      atomicAdd(gen, 1ull);
    } else {
      const unsigned long long t0 = global_timer_ns();
      while (ld_acquire_gpu_u64(gen) == g) {
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          raise_device_error(FP8MOE_DEVERR_TIMEOUT);
          break;
        }
        __nanosleep(32);
      }
    }
    __threadfence_system();
  }
  __syncthreads();
}

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[u]));
    acc[2 * u] += f.x;
    acc[2 * u + 1] += f.y;
  }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float (&acc)[8]) {
  __align__(16) __nv_bfloat162 pk[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) pk[u] = __floats2bfloat162_rn(acc[2 * u], acc[2 * u + 1]);
  return *reinterpret_cast<const uint4*>(pk);
}

__global__ void __launch_bounds__(kTpThreads)
tp_combine_allreduce_kernel(const __grid_constant__ TpArgs a, int rank_first, int ctas_per_rank) {
  const int rank = rank_first + static_cast<int>(blockIdx.x) / ctas_per_rank;
  const int cta = static_cast<int>(blockIdx.x) % ctas_per_rank;
  const int n = a.nranks, T = a.T, K = a.K, H = a.H;
  const int cpr = H / 8;                            // 8-column (16-byte) units per row
  const int Ts = (T + n - 1) / n;
  const long long stride = static_cast<long long>(ctas_per_rank) * kTpThreads;
  const long long first = static_cast<long long>(cta) * kTpThreads + threadIdx.x;
  // this call's epoch: read by every CTA before the first barrier, advanced by CTA 0
  // after it (when no CTA of this launch reads the counter any more)
  __shared__ unsigned long long s_epoch;
  if (threadIdx.x == 0) s_epoch = ld_acquire_gpu_u64(a.barrier[rank] + 2) + 1;
  __syncthreads();
  const unsigned long long epoch = s_epoch;

  // 1. combine this rank's pair rows per token; the bf16 partial goes to the slice owner
  const __nv_bfloat16* y = a.ystage[rank];
  const uint8_t* flag = a.pair_flag[rank];
  const bool all_present = *a.n_present[rank] == T * K;
  for (long long i = first; i < static_cast<long long>(T) * cpr; i += stride) {
    const int t = static_cast<int>(i / cpr);
    const int c = static_cast<int>(i % cpr) * 8;
    float acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = 0.0f;
    const __nv_bfloat16* row = y + static_cast<size_t>(t) * K * H + c;
    if (all_present) {
      // up to kTpBatch rows in flight per thread, then added in k order
      for (int k0 = 0; k0 < K; k0 += kTpBatch) {
        uint4 v[kTpBatch];
#pragma unroll
        for (int j = 0; j < kTpBatch; ++j)
          if (k0 + j < K) v[j] = __ldcs(reinterpret_cast<const uint4*>(row + static_cast<size_t>(k0 + j) * H));
#pragma unroll
        for (int j = 0; j < kTpBatch; ++j)
          if (k0 + j < K) add_bf16x8(acc, v[j]);
      }
    } else {
      for (int k = 0; k < K; ++k)
        if (flag[static_cast<size_t>(t) * K + k])
          add_bf16x8(acc, __ldcs(reinterpret_cast<const uint4*>(row + static_cast<size_t>(k) * H)));
    }
    const int p = t / Ts;
    __nv_bfloat16* dst = a.recv[p] + (static_cast<size_t>(rank) * Ts + (t - p * Ts)) * H + c;
    *reinterpret_cast<uint4*>(dst) = pack_bf16x8(acc);
  }

  // 2. publish: this rank's partials are in every owner's receive buffer
  tp_rank_barrier(a.barrier[rank], ctas_per_rank);
  if (cta == 0 && threadIdx.x < n) st_release_sys_u64(a.flags[threadIdx.x] + rank, epoch);

  // 3. reduce this rank's slice in rank order and write it into every rank's output
  if (threadIdx.x < n) tp_wait_ge(a.flags[rank] + threadIdx.x, epoch);
  __syncthreads();
  __threadfence_system();
  const int t0 = rank * Ts;
  const int rows = max(0, min(T, t0 + Ts) - t0);
  const __nv_bfloat16* mine = a.recv[rank];
  for (long long i = first; i < static_cast<long long>(rows) * cpr; i += stride) {
    const int r = static_cast<int>(i / cpr);
    const int c = static_cast<int>(i % cpr) * 8;
    float acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = 0.0f;
    // the n partials in flight together, read at L2 (other ranks wrote them during this
    // kernel), then added in rank order
    uint4 part[kTpMaxRanks];
#pragma unroll
    for (int q = 0; q < kTpMaxRanks; ++q)
      if (q < n) part[q] = __ldcg(reinterpret_cast<const uint4*>(mine + (static_cast<size_t>(q) * Ts + r) * H + c));
#pragma unroll
    for (int q = 0; q < kTpMaxRanks; ++q)
      if (q < n) add_bf16x8(acc, part[q]);
    const uint4 v = pack_bf16x8(acc);
    for (int p = 0; p < n; ++p)
      *reinterpret_cast<uint4*>(a.out[p] + static_cast<size_t>(t0 + r) * H + c) = v;
  }

  // 4. publish the slice; leave once every rank has written this rank's output
  tp_rank_barrier(a.barrier[rank], ctas_per_rank);
  if (cta == 0 && threadIdx.x < n) st_release_sys_u64(a.flags[threadIdx.x] + kTpMaxRanks + rank, epoch);
  if (cta == 0) {
    if (threadIdx.x < n) tp_wait_ge(a.flags[rank] + kTpMaxRanks + threadIdx.x, epoch);
    if (threadIdx.x == 0) atomicExch(a.barrier[rank] + 2, epoch);   // the next call's base
    __syncthreads();
    __threadfence_system();
  }
}

}  // namespace fp8moe
