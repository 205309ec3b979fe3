// Dynamic FP8 (OCP E4M3fn) quantisation: 1x128 activation groups and 128x128
// weight blocks.
//
// "Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang": section
// "Blockscale FP8 MoE Computation" (hidden states viewed as [M*H/128, 128],
// one fp32 scale per 128 values, dynamic_per_token_scaled_fp8_quant; the MoE
// kernel takes the scales transposed) and section "General Linear Layer" (one
// scale per 1x128 activation block and per 128x128 weight block). Recipe:
// scale = amax / 448 (fp32 division), q = E4M3fn(x / scale) rounded to nearest
// even and saturated (hardware cvt); an all-zero group gives scale 0, codes 0.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace fp8moe {

constexpr float kFp8Max = 448.0f;
constexpr int kQuantWarps = 8;

// Eight quantised codes of v[0..7] with one scale, packed little-endian.
__device__ __forceinline__ uint2 quant8(const float (&v)[8], float scale) {
  uint32_t lo = 0, hi = 0;
  if (scale != 0.0f) {
    lo = static_cast<uint32_t>(cvt_e4m3x2(__fdiv_rn(v[0], scale), __fdiv_rn(v[1], scale))) |
         (static_cast<uint32_t>(cvt_e4m3x2(__fdiv_rn(v[2], scale), __fdiv_rn(v[3], scale))) << 16);
    hi = static_cast<uint32_t>(cvt_e4m3x2(__fdiv_rn(v[4], scale), __fdiv_rn(v[5], scale))) |
         (static_cast<uint32_t>(cvt_e4m3x2(__fdiv_rn(v[6], scale), __fdiv_rn(v[7], scale))) << 16);
  }
  return make_uint2(lo, hi);
}

// One warp per (row, span of 2 * kQuantUnroll groups); each half-warp (16 lanes
// x 8 bf16) covers one 128-wide group. K % 8 == 0; a last group shorter than
// 128 uses its valid elements. Each lane issues the loads of its kQuantUnroll
// groups before using them, so a warp costs one memory round trip.
constexpr int kQuantUnroll = 4;
constexpr int kQuantSpan = 2 * kQuantUnroll;     // groups per warp
__global__ void __launch_bounds__(32 * kQuantWarps)
quant_1x128_kernel(const __nv_bfloat16* __restrict__ x, int ld_x, int M, int K, uint8_t* __restrict__ q,
                   float* __restrict__ scales, int col_major) {
  const int lane = threadIdx.x & 31;
  const int KB = (K + 127) / 128;
  const int spans = (KB + kQuantSpan - 1) / kQuantSpan;
  const long long w = static_cast<long long>(blockIdx.x) * kQuantWarps + (threadIdx.x >> 5);
  if (w >= static_cast<long long>(M) * spans) return;
  const int m = static_cast<int>(w / spans);
  const int half = lane >> 4, hl = lane & 15;
  const __nv_bfloat16* row = x + static_cast<size_t>(m) * ld_x;
  {
    const int g0 = static_cast<int>(w % spans) * kQuantSpan;
    uint4 raw[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int g = g0 + 2 * u + half;
      const int col = g * 128 + hl * 8;
      raw[u] = (g < KB && col < K) ? __ldg(reinterpret_cast<const uint4*>(row + col)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int g = g0 + 2 * u + half;
      const int col = g * 128 + hl * 8;
      const bool in = (g < KB) && (col < K);
      float v[8];
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h2[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
      }
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const float scale = __fdiv_rn(amax, kFp8Max);
      if (in) *reinterpret_cast<uint2*>(q + static_cast<size_t>(m) * K + col) = quant8(v, scale);
      if (g < KB && hl == 0) {
        if (col_major)
          scales[static_cast<size_t>(g) * M + m] = scale;
        else
          scales[static_cast<size_t>(m) * KB + g] = scale;
      }
    }
  }
}

// One CTA per 128x128 block of an fp32 matrix; 256 threads, each a 1x64 strip.
__global__ void __launch_bounds__(256)
quant_128x128_kernel(const float* __restrict__ w, int ld_w, int N, int K, uint8_t* __restrict__ q,
                     float* __restrict__ scales) {
  const int nb = blockIdx.y, kb = blockIdx.x;
  const int KB = gridDim.x;
  const int r = nb * 128 + (threadIdx.x >> 1);
  const int c0 = kb * 128 + (threadIdx.x & 1) * 64;
  float v[64];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const int c = c0 + i;
    v[i] = (r < N && c < K) ? w[static_cast<size_t>(r) * ld_w + c] : 0.0f;
    amax = fmaxf(amax, fabsf(v[i]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  __shared__ float s_amax[8];
  if ((threadIdx.x & 31) == 0) s_amax[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = s_amax[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, s_amax[i]);
  const float scale = __fdiv_rn(amax, kFp8Max);
  if (threadIdx.x == 0) scales[static_cast<size_t>(nb) * KB + kb] = scale;
  if (r >= N) return;
#pragma unroll
  for (int i = 0; i < 64; i += 8) {
    float e8[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) e8[j] = v[i + j];
    const uint2 packed = quant8(e8, scale);
    const uint8_t* b = reinterpret_cast<const uint8_t*>(&packed);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (c0 + i + j < K) q[static_cast<size_t>(r) * K + c0 + i + j] = b[j];
  }
}

// Weight re-pack into the tiled layout the MoE GEMMs can read with one contiguous
// 16 KB box per 128 x 128 block: w [E, N, K] row-major -> out [E, N/128, K/128,
// 128, 128] (block (e, nb, kb) holds rows nb*128.. and columns kb*128.. of expert
// e's matrix, row-major inside the block). One CTA per block, 16-byte copies.
__global__ void __launch_bounds__(256)
tile_weights_kernel(const uint8_t* __restrict__ w, int N, int K, uint8_t* __restrict__ out) {
  const int kb = blockIdx.x, nb = blockIdx.y, e = blockIdx.z;
  const int NB = gridDim.y, KB = gridDim.x;
  const uint8_t* src = w + (static_cast<size_t>(e) * N + static_cast<size_t>(nb) * 128) * K + static_cast<size_t>(kb) * 128;
  uint8_t* dst = out + ((static_cast<size_t>(e) * NB + nb) * KB + kb) * (128 * 128);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = i * 256 + threadIdx.x;   // 16-byte piece: row idx / 8, column piece idx % 8
    const int r = idx >> 3, c = (idx & 7) * 16;
    *reinterpret_cast<uint4*>(dst + r * 128 + c) =
        __ldg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(r) * K + c));
  }
}

}  // namespace fp8moe
