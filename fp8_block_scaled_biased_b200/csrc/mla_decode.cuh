// Multi-head latent attention (MLA) at decode over a paged latent KV buffer.
//
// "Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang", section
// "Attention Mechanisms", subsection "MLA For Decode": queries q [B, Hq, 576]
// (512 latent + 64 rotary entries, weights absorbed), one latent KV head shared
// by every query head in a buffer viewed as [pages, page_size, 1, 576], the page
// table (kv_indptr, kv_indices, kv_last_page_lens), sm_scale and logit_cap; the
// output o [B, Hq, 512] is the softmax-weighted sum of the rows' first 512
// entries, the score of row j being sm_scale * <q, row_j> (soft-capped as
// logit_cap * tanh(s / logit_cap) when logit_cap > 0).
//
// Layout of the work. A CTA owns 16 query heads (the M of one warp-level MMA) of
// one sequence and one contiguous split of its tokens, walked in chunks of 32
// rows. Per chunk:
//   - warp 0 issues one bulk asynchronous copy (cp.async.bulk, 1152 bytes) per
//     row from wherever its page lies into a shared-memory stage, completing on
//     the stage's mbarrier; two stages, so the next chunk's rows stream in while
//     this one is computed, and a stage is refilled (chunk c + 2) as soon as every
//     warp is past chunk c's P V. Rows past the split's end copy the chunk's first
//     row instead (a finite value that gets weight 0);
//   - S = Q K^T: warp w scores rows 8w..8w+7 for all 16 heads (36 MMAs over the
//     576 entries, Q and K read from shared memory with ldmatrix);
//   - online softmax in base 2: per-head maxima and sums meet across the warps in
//     shared memory; the weights, rounded to bf16, go to shared memory as the A
//     operand of the second product, and the running sum adds the same rounded
//     weights, so the output is a true weighted mean of the rows;
//   - O += P V: warp w owns value columns 128w..128w+127 (64 fp32 accumulators per
//     thread), the V operand read transposed from the same stage (ldmatrix.trans).
// Scores and accumulators are fp32 and every product is exact (bf16 x bf16).
// With one split the CTA writes o (bf16) and lse; with several, each split writes
// its normalised partial and log-sum-exp, and mla_combine_kernel merges them in
// split order (deterministic).
//
// Why warp-level MMAs and not tcgen05: the decode batch of the pages' TP8 run
// gives a GPU 16 query heads, and the smallest tcgen05 tile is M=64, which would
// run 75% padding; the kernel moves 30 FLOP per KV byte and is bound by HBM, so
// the MMA instruction's rate is not what limits it.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace fp8moe {

constexpr int kMlaDk = 576;                         // query/key head width
constexpr int kMlaDv = 512;                         // value width (the latent part)
constexpr int kMlaHeads = 16;                       // query heads per CTA
constexpr int kMlaRows = 32;                        // KV rows per chunk
constexpr int kMlaStages = 2;
constexpr int kMlaWarps = 4;
constexpr int kMlaThreads = kMlaWarps * 32;
constexpr int kMlaRowBytes = kMlaDk * 2;            // 1152: one bulk copy per row
constexpr int kMlaPitch = kMlaRowBytes + 16;        // shared-memory row pitch: rows 4 banks apart
constexpr int kMlaPPitch = (kMlaRows + 8) * 2;      // 80 bytes per head of P
constexpr int kMlaStageBytes = kMlaRows * kMlaPitch;
constexpr int kMlaOffQ = kMlaStages * kMlaStageBytes;
constexpr int kMlaOffP = kMlaOffQ + kMlaHeads * kMlaPitch;
constexpr int kMlaOffRed = kMlaOffP + kMlaHeads * kMlaPPitch;
constexpr int kMlaOffBar = kMlaOffRed + 2 * kMlaWarps * kMlaHeads * 4;
constexpr int kMlaSmemBytes = kMlaOffBar + kMlaStages * 8;
constexpr int kMlaMaxSplits = 64;
static_assert(kMlaStageBytes % 16 == 0 && kMlaOffQ % 16 == 0 && kMlaOffP % 16 == 0 && kMlaOffBar % 8 == 0,
              "shared-memory regions must keep 16-byte rows");
static_assert(kMlaSmemBytes <= 113 * 1024, "two CTAs per SM");

struct MlaArgs {
  const __nv_bfloat16* q;        // [B, Hq, 576]
  const __nv_bfloat16* kv;       // [pages, page_size, 576]
  __nv_bfloat16* o;              // [B, Hq, 512]
  float* lse;                    // [B, Hq] or null
  const int32_t* indptr;         // [B + 1]
  const int32_t* indices;        // [num_indices]
  const int32_t* last_lens;      // [B]
  float* part_o;                 // [B, Hq, splits, 512] (splits > 1)
  float* part_lse;               // [B, Hq, splits]
  int B, Hq, num_pages, page_size, num_indices, splits;
  float sm_scale, logit_cap;
};

__device__ __forceinline__ void bulk_copy_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Bounded wait for one phase of a stage barrier (false once the time limit passes).
__device__ __forceinline__ bool mla_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// Warp 0: the bulk copies of chunk `c` (rows row0 + 32c + lane of the sequence) into
// its stage. Every lane copies one row; a lane past the split's end copies the
// chunk's first row, so the stage always receives 32 rows.
__device__ __forceinline__ void mla_issue_chunk(const MlaArgs& a, unsigned char* smem, int c, int row0, int row1,
                                                int page0) {
  const int lane = threadIdx.x & 31;
  const int stage = c % kMlaStages;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kMlaOffBar) + stage;
  if (lane == 0) mbar_arrive_expect_tx(bar, kMlaRows * kMlaRowBytes);
  __syncwarp();
  int r = row0 + c * kMlaRows + lane;
  if (r >= row1) r = row0 + c * kMlaRows;
  const int ps = a.page_size;
  int page = __ldg(a.indices + page0 + r / ps);
  int slot = r % ps;
  if (page < 0 || page >= a.num_pages) {
    raise_device_error(FP8MOE_DEVERR_PAGE);
    page = 0;
  }
  const __nv_bfloat16* src = a.kv + (static_cast<size_t>(page) * ps + slot) * kMlaDk;
  fence_proxy_async_smem();   // the stage's earlier generic reads come before the async writes
  bulk_copy_g2s(smem + stage * kMlaStageBytes + lane * kMlaPitch, src, kMlaRowBytes, bar);
}

__global__ void __launch_bounds__(kMlaThreads, 2) mla_decode_kernel(const __grid_constant__ MlaArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int hg = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kMlaOffBar);
  float* red_max = reinterpret_cast<float*>(smem + kMlaOffRed);      // [warp][head]
  float* red_sum = red_max + kMlaWarps * kMlaHeads;

  // the sequence's extent from the page table (checked; a bad table gives an empty sequence)
  int page0 = 0, L = 0;
  {
    const int lo = __ldg(a.indptr + b), hi = __ldg(a.indptr + b + 1);
    if (lo < 0 || hi < lo || hi > a.num_indices) {
      if (threadIdx.x == 0) raise_device_error(FP8MOE_DEVERR_PAGE);
    } else if (hi > lo) {
      int last = __ldg(a.last_lens + b);
      if (last < 1 || last > a.page_size) {
        if (threadIdx.x == 0) raise_device_error(FP8MOE_DEVERR_PAGE);
        last = min(max(last, 1), a.page_size);
      }
      page0 = lo;
      L = (hi - lo - 1) * a.page_size + last;
    }
  }
  // this split's rows: equal shares rounded up to whole chunks
  const int per = ((L + a.splits - 1) / a.splits + kMlaRows - 1) / kMlaRows * kMlaRows;
  const int row0 = min(L, split * per), row1 = min(L, row0 + per);
  const int nchunks = (row1 - row0 + kMlaRows - 1) / kMlaRows;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMlaStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  // the 16 query rows of this head group
  {
    const uint4* qsrc = reinterpret_cast<const uint4*>(a.q + (static_cast<size_t>(b) * a.Hq + hg * kMlaHeads) * kMlaDk);
    constexpr int kVec = kMlaDk / 8;   // 72 16-byte pieces per row
    for (int i = threadIdx.x; i < kMlaHeads * kVec; i += kMlaThreads) {
      const int h = i / kVec, v = i % kVec;
      *reinterpret_cast<uint4*>(smem + kMlaOffQ + h * kMlaPitch + v * 16) = __ldg(qsrc + i);
    }
  }
  __syncthreads();
  if (warp == 0) {
    for (int c = 0; c < min(nchunks, kMlaStages); ++c) mla_issue_chunk(a, smem, c, row0, row1, page0);
  }

  const float kLog2e = 1.4426950408889634f;
  const float scale2 = a.sm_scale * kLog2e;
  const bool capped = a.logit_cap > 0.0f;
  float m2[2] = {-INFINITY, -INFINITY};   // running maxima (base-2 units) of heads g, g+8
  float l[2] = {0.0f, 0.0f};              // running sums of the rounded weights
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;

  const uint32_t q_base = smem_u32(smem + kMlaOffQ);
  const uint32_t p_base = smem_u32(smem + kMlaOffP);
  bool failed = false;
  int issued = min(nchunks, kMlaStages);   // chunks whose copies have been issued (same on every thread)
  for (int c = 0; c < nchunks; ++c) {
    const int stage = c % kMlaStages;
    if (!mla_wait(&full[stage], (c / kMlaStages) & 1)) failed = true;
    const uint32_t kv_base = smem_u32(smem + stage * kMlaStageBytes);

    // S = Q K^T for this warp's 8 rows
    float s[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    {
      const uint32_t qa = q_base + (lane & 15) * kMlaPitch + (lane >> 4) * 16;
      const uint32_t ka = kv_base + (warp * 8 + (lane & 7)) * kMlaPitch + (lane >> 3) * 16;
#pragma unroll 6
      for (int kk = 0; kk < kMlaDk / 16; kk += 2) {
        uint32_t kb[4], a0[4], a1[4];
        ldsm_x4(ka + kk * 32, kb);
        ldsm_x4(qa + kk * 32, a0);
        ldsm_x4(qa + (kk + 1) * 32, a1);
        mma_bf16_16816(s, a0, kb[0], kb[1]);
        mma_bf16_16816(s, a1, kb[2], kb[3]);
      }
    }
    // scores in base-2 units, masked past the split's end
    const int rbase = row0 + c * kMlaRows + warp * 8 + 2 * tig;
    float t[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float x = s[i];
      if (capped) x = a.logit_cap * tanhf(x * a.sm_scale / a.logit_cap) * kLog2e;
      else x *= scale2;
      t[i] = (rbase + (i & 1) < row1) ? x : -INFINITY;
    }
    float mx0 = fmaxf(t[0], t[1]), mx1 = fmaxf(t[2], t[3]);
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    if (tig == 0) {
      red_max[warp * kMlaHeads + g] = mx0;
      red_max[warp * kMlaHeads + g + 8] = mx1;
    }
    if (__syncthreads_or(failed)) {
      failed = true;
      break;
    }

    float mnew[2], alpha[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int h = g + 8 * j;
      float cm = red_max[h];
#pragma unroll
      for (int w = 1; w < kMlaWarps; ++w) cm = fmaxf(cm, red_max[w * kMlaHeads + h]);
      mnew[j] = fmaxf(m2[j], cm);   // finite: every chunk holds at least one row of the split
      alpha[j] = (m2[j] == -INFINITY) ? 0.0f : exp2f(m2[j] - mnew[j]);
    }
    // weights rounded to bf16: the A operand of P V, and the terms of the running sum
    const __nv_bfloat162 p01 = __floats2bfloat162_rn(exp2f(t[0] - mnew[0]), exp2f(t[1] - mnew[0]));
    const __nv_bfloat162 p23 = __floats2bfloat162_rn(exp2f(t[2] - mnew[1]), exp2f(t[3] - mnew[1]));
    *reinterpret_cast<__nv_bfloat162*>(smem + kMlaOffP + g * kMlaPPitch + (warp * 8 + 2 * tig) * 2) = p01;
    *reinterpret_cast<__nv_bfloat162*>(smem + kMlaOffP + (g + 8) * kMlaPPitch + (warp * 8 + 2 * tig) * 2) = p23;
    const float2 f01 = __bfloat1622float2(p01), f23 = __bfloat1622float2(p23);
    float sm0 = f01.x + f01.y, sm1 = f23.x + f23.y;
    sm0 += __shfl_xor_sync(0xffffffffu, sm0, 1);
    sm0 += __shfl_xor_sync(0xffffffffu, sm0, 2);
    sm1 += __shfl_xor_sync(0xffffffffu, sm1, 1);
    sm1 += __shfl_xor_sync(0xffffffffu, sm1, 2);
    if (tig == 0) {
      red_sum[warp * kMlaHeads + g] = sm0;
      red_sum[warp * kMlaHeads + g + 8] = sm1;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int h = g + 8 * j;
      float cs = red_sum[h];
#pragma unroll
      for (int w = 1; w < kMlaWarps; ++w) cs += red_sum[w * kMlaHeads + h];
      l[j] = l[j] * alpha[j] + cs;
      m2[j] = mnew[j];
    }
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      o[n][0] *= alpha[0];
      o[n][1] *= alpha[0];
      o[n][2] *= alpha[1];
      o[n][3] *= alpha[1];
    }
    // O += P V over this warp's 128 value columns
#pragma unroll
    for (int ks = 0; ks < kMlaRows / 16; ++ks) {
      uint32_t pa[4];
      ldsm_x4(p_base + (lane & 15) * kMlaPPitch + (ks * 16 + (lane >> 4) * 8) * 2, pa);
      const uint32_t va = kv_base + (ks * 16 + (lane & 15)) * kMlaPitch + (warp * 128 + (lane >> 4) * 8) * 2;
#pragma unroll
      for (int n = 0; n < 16; n += 2) {
        uint32_t vb[4];
        ldsm_x4_t(va + n * 16, vb);
        mma_bf16_16816(o[n], pa, vb[0], vb[1]);
        mma_bf16_16816(o[n + 1], pa, vb[2], vb[3]);
      }
    }
    // this chunk's stage is free once every warp is past P V: stream in chunk c + 2
    if (c + kMlaStages < nchunks) {
      __syncthreads();
      if (warp == 0) mla_issue_chunk(a, smem, c + kMlaStages, row0, row1, page0);
      issued = c + kMlaStages + 1;
    }
  }

  if (failed) {
    raise_device_error(FP8MOE_DEVERR_TIMEOUT);
    // let the copies already issued land (bounded) before the CTA's shared memory goes away
    if (threadIdx.x == 0)
      for (int c = max(0, issued - kMlaStages); c < issued; ++c) (void)mla_wait(&full[c % kMlaStages], (c / kMlaStages) & 1);
    return;
  }

  // o = O / l, lse = ln(sum of exp(score))
  const float inv[2] = {l[0] > 0.0f ? 1.0f / l[0] : 0.0f, l[1] > 0.0f ? 1.0f / l[1] : 0.0f};
  const float kLn2 = 0.6931471805599453f;
  const size_t head0 = static_cast<size_t>(b) * a.Hq + hg * kMlaHeads;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const size_t head = head0 + g + 8 * j;
    const float lse = l[j] > 0.0f ? (m2[j] + log2f(l[j])) * kLn2 : -INFINITY;
    if (a.splits == 1) {
      __nv_bfloat16* dst = a.o + head * kMlaDv + warp * 128 + 2 * tig;
#pragma unroll
      for (int n = 0; n < 16; ++n)
        *reinterpret_cast<__nv_bfloat162*>(dst + n * 8) =
            __floats2bfloat162_rn(o[n][2 * j] * inv[j], o[n][2 * j + 1] * inv[j]);
      if (a.lse && warp == 0 && tig == 0) a.lse[head] = lse;
    } else {
      float* dst = a.part_o + (head * a.splits + split) * kMlaDv + warp * 128 + 2 * tig;
#pragma unroll
      for (int n = 0; n < 16; ++n)
        *reinterpret_cast<float2*>(dst + n * 8) = make_float2(o[n][2 * j] * inv[j], o[n][2 * j + 1] * inv[j]);
      if (warp == 0 && tig == 0) a.part_lse[head * a.splits + split] = lse;
    }
  }
}

// Merges the splits of each (sequence, head): weights exp(lse_s - max), summed in
// split order. One warp per (sequence, head); a lane owns 16 value columns.
__global__ void __launch_bounds__(256) mla_combine_kernel(const float* __restrict__ part_o,
                                                          const float* __restrict__ part_lse, int BH, int splits,
                                                          __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
  const int bh = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (bh >= BH) return;
  const float* pl = part_lse + static_cast<size_t>(bh) * splits;
  float mx = -INFINITY;
  for (int s = 0; s < splits; ++s) mx = fmaxf(mx, pl[s]);
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
  float wsum = 0.0f;
  if (mx != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const float ls = pl[s];
      if (ls == -INFINITY) continue;
      const float w = expf(ls - mx);
      wsum += w;
      const float4* src = reinterpret_cast<const float4*>(part_o + (static_cast<size_t>(bh) * splits + s) * kMlaDv);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 v = src[j * 32 + lane];
        acc[4 * j] += w * v.x;
        acc[4 * j + 1] += w * v.y;
        acc[4 * j + 2] += w * v.z;
        acc[4 * j + 3] += w * v.w;
      }
    }
  }
  const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
  __nv_bfloat16* dst = o + static_cast<size_t>(bh) * kMlaDv;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __align__(8) __nv_bfloat162 pk[2] = {__floats2bfloat162_rn(acc[4 * j] * inv, acc[4 * j + 1] * inv),
                                         __floats2bfloat162_rn(acc[4 * j + 2] * inv, acc[4 * j + 3] * inv)};
    *reinterpret_cast<uint2*>(dst + (j * 32 + lane) * 4) = *reinterpret_cast<const uint2*>(pk);
  }
  if (lse && lane == 0) lse[bh] = wsum > 0.0f ? mx + logf(wsum) : -INFINITY;
}

}  // namespace fp8moe
