// Biased grouped top-k routing: one warp per token.
//
// "Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang", section
// "Top-K routing": each token keeps topk_group of num_expert_group expert
// groups and picks its top-k experts inside them; weights are scaled by
// routed_scaling_factor. Scoring (DeepSeek-V3 style): s = sigmoid(logit),
// b = s + correction_bias; group score = sum of the group's two largest b;
// ties go to the lower group / expert index; weights are the unbiased s.
// The logits are fp32 or bf16 (the page's routing test runs over a dtype);
// bf16 values widen to fp32 exactly, so both take the same fp32 sequence.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace fp8moe {

constexpr int kRouteMaxPerLane = 16;   // E <= 32 * 16 = 512
constexpr int kRouteWarps = 8;

// e^y as a fixed sequence of IEEE fp32 operations (Cody & Waite reduction,
// degree-7 Taylor polynomial in Horner form, no fused multiply-add), so that
// the host-side reference and this kernel produce identical bits.
__device__ __forceinline__ float exp_f32_recipe(float y) {
  y = fminf(fmaxf(y, -87.0f), 88.0f);
  const float n = rintf(__fmul_rn(y, 0x1.715476p+0f));            // log2(e) rounded to fp32
  float r = __fsub_rn(y, __fmul_rn(n, 0.693359375f));           // exact product (355/512)
  r = __fsub_rn(r, __fmul_rn(n, -0x1.bd0106p-13f));              // ln2 - 355/512
  // 1/k!, k = 7..0, rounded to fp32 (hex literals: exact values)
  float p = 0x1.a01a02p-13f;
  p = __fadd_rn(__fmul_rn(p, r), 0x1.6c16c2p-10f);
  p = __fadd_rn(__fmul_rn(p, r), 0x1.111112p-7f);
  p = __fadd_rn(__fmul_rn(p, r), 0x1.555556p-5f);
  p = __fadd_rn(__fmul_rn(p, r), 0x1.555556p-3f);
  p = __fadd_rn(__fmul_rn(p, r), 0.5f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  const float two_n = __int_as_float((static_cast<int>(n) + 127) << 23);
  return __fmul_rn(p, two_n);
}

__device__ __forceinline__ float sigmoid_f32_recipe(float x) {
  return __fdiv_rn(1.0f, __fadd_rn(1.0f, exp_f32_recipe(-x)));
}

__device__ __forceinline__ float logit_f32(float v) { return v; }
__device__ __forceinline__ float logit_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
// four consecutive logits: 16-byte aligned for fp32, 8-byte aligned for bf16
__device__ __forceinline__ float4 load_logits4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ float4 load_logits4(const __nv_bfloat16* p) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// (value desc, index asc) ordering: does (v1, i1) rank before (v0, i0)?
__device__ __forceinline__ bool ranks_before(float v1, int i1, float v0, int i0) {
  return v1 > v0 || (v1 == v0 && i1 < i0);
}

// Each lane owns `per_lane` consecutive experts; a lane's experts never span two
// groups (per_lane divides the group size), so a group is lanes_per_group
// consecutive lanes. PL > 0 fixes per_lane at compile time (the usual 1, 2, 4,
// 8, 16); PL == 0 takes it from the argument. vec4: rows and bias allow vector
// loads of four of a lane's experts (PL % 4 == 0 only). LT: fp32 or bf16 logits.
template <int PL, typename LT>
__global__ void __launch_bounds__(32 * kRouteWarps)
route_kernel(const LT* __restrict__ logits, int ld_in, const float* __restrict__ bias,
             float* __restrict__ topk_w, int32_t* __restrict__ topk_ids, int ld_out, int T, int E, int K,
             int G, int TG, int renorm, float factor, int per_lane_arg, int vec4) {
  constexpr int kPL = PL > 0 ? PL : kRouteMaxPerLane;
  const int per_lane = PL > 0 ? PL : per_lane_arg;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const int per_group = E / G;
  const int lanes_per_group = per_group / per_lane;
  const int e0 = lane * per_lane;

  float s[kPL], b[kPL];
  const LT* row = logits + static_cast<size_t>(t) * ld_in;
  float x[kPL], bs[kPL];
  if (PL % 4 == 0 && PL > 0 && vec4 && e0 < E) {
#pragma unroll
    for (int j = 0; j < kPL; j += 4) {
      const float4 xv = load_logits4(row + e0 + j);
      const float4 bv = __ldg(reinterpret_cast<const float4*>(bias + e0 + j));
      x[j] = xv.x; x[j + 1] = xv.y; x[j + 2] = xv.z; x[j + 3] = xv.w;
      bs[j] = bv.x; bs[j + 1] = bv.y; bs[j + 2] = bv.z; bs[j + 3] = bv.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < kPL; ++j) {
      const int e = e0 + j;
      const bool in = j < per_lane && e < E;
      x[j] = in ? logit_f32(__ldg(row + e)) : 0.0f;
      bs[j] = in ? __ldg(bias + e) : 0.0f;
    }
  }
#pragma unroll
  for (int j = 0; j < kPL; ++j) {
    if (j < per_lane && e0 + j < E) {
      s[j] = sigmoid_f32_recipe(x[j]);
      b[j] = __fadd_rn(s[j], bs[j]);
    } else {
      s[j] = 0.0f;
      b[j] = -INFINITY;
    }
  }

  // Two largest b among this lane's experts (values only: the group score does
  // not depend on which index holds a tied value).
  float t1 = -INFINITY, t2 = -INFINITY;
#pragma unroll
  for (int j = 0; j < kPL; ++j) {
    if (j < per_lane) {
      if (b[j] > t1) {
        t2 = t1;
        t1 = b[j];
      } else if (b[j] > t2) {
        t2 = b[j];
      }
    }
  }
  // Merge with the other lanes of the group into the group's first lane.
  float g1 = t1, g2 = t2;
  for (int d = 1; d < lanes_per_group; ++d) {
    const int src = min(lane + d, 31);
    const float o1 = __shfl_sync(0xffffffffu, t1, src);
    const float o2 = __shfl_sync(0xffffffffu, t2, src);
    if (o1 > g1) {
      g2 = fmaxf(g1, o2);
      g1 = o1;
    } else {
      g2 = fmaxf(g2, o1);
    }
  }
  const float my_gscore = (per_group >= 2) ? __fadd_rn(g1, g2) : g1;

  // Group scores to lanes 0..G-1, then rank them.
  const int gsrc = min(lane * lanes_per_group, 31);
  const float gs = __shfl_sync(0xffffffffu, my_gscore, gsrc);
  int grank = 0;
  for (int h = 0; h < G; ++h) {
    const float o = __shfl_sync(0xffffffffu, gs, h);
    if (lane < G && ranks_before(o, h, gs, lane)) ++grank;
  }
  const bool gsel_lane = (lane < G) && (grank < TG);
  const unsigned gmask = __ballot_sync(0xffffffffu, gsel_lane);   // bit g: group g kept

  // Experts outside kept groups leave the race.
  const int my_group = (e0 < E) ? e0 / per_group : 0;
  const bool my_group_kept = (e0 < E) && ((gmask >> my_group) & 1u);
#pragma unroll
  for (int j = 0; j < kPL; ++j)
    if (!my_group_kept) b[j] = -INFINITY;

  // Top-k by repeated warp argmax over (b desc, index asc).
  float my_w = 0.0f;
  int my_id = 0;
  for (int k = 0; k < K; ++k) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < kPL; ++j) {
      if (j < per_lane && (e0 + j) < E && ranks_before(b[j], e0 + j, bv, bi)) {
        bv = b[j];
        bi = e0 + j;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (ranks_before(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    // the owner removes the winner and publishes its unbiased score
    const int owner = bi / per_lane;
    float sw = 0.0f;
#pragma unroll
    for (int j = 0; j < kPL; ++j) {
      if (lane == owner && e0 + j == bi) {
        sw = s[j];
        b[j] = -INFINITY;
      }
    }
    sw = __shfl_sync(0xffffffffu, sw, owner);
    if (lane == k) {
      my_w = sw;
      my_id = bi;
    }
  }

  if (renorm) {
    float denom = 0.0f;
    for (int k = 0; k < K; ++k) {
      const float wk = __shfl_sync(0xffffffffu, my_w, k);
      denom = (k == 0) ? wk : __fadd_rn(denom, wk);
    }
    if (denom != 0.0f) my_w = __fdiv_rn(my_w, denom);
  }
  my_w = __fmul_rn(my_w, factor);
  if (lane < K) {
    topk_w[static_cast<size_t>(t) * ld_out + lane] = my_w;
    topk_ids[static_cast<size_t>(t) * ld_out + lane] = my_id;
  }
}

}  // namespace fp8moe
