// C ABI of the FP8 block-scaled biased MoE layer (declarations and contracts in
// include/fp8moe.h). Host code: argument checks, TMA tensor maps, launches.
// All kernels live in this one translation unit so they share the device error word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include "common.cuh"
#include "gemm_sm100.cuh"
#include "moe_aux.cuh"
#include "quant.cuh"
#include "route.cuh"
#include "sort.cuh"
#include "tp_reduce.cuh"
#include "ep_peer.cuh"
#include "mla_decode.cuh"

static_assert(fp8moe::kMoeBlockRows == fp8moe::kBM, "sorted blocks are GEMM tiles");

using namespace fp8moe;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FP8MOE_ECUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
  g_last_error.clear();
  return FP8MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch check for the GEMM kernels: on failure the message carries the kernel's
// resource attributes next to what the launch asked for.
template <typename Kernel>
int check_gemm_launch(const char* what, Kernel kernel, int threads, size_t smem) {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    g_last_error.clear();
    return FP8MOE_OK;
  }
  cudaFuncAttributes fa{};
  cudaFuncGetAttributes(&fa, kernel);
  return fail(FP8MOE_ECUDA,
              "%s: launch failed: %s (kernel: %d regs, max %d threads, %zu B static smem, %d B max dynamic smem, "
              "%zu B local; launch: %d threads, %zu B dynamic smem)",
              what, cudaGetErrorString(e), fa.numRegs, fa.maxThreadsPerBlock, fa.sharedSizeBytes,
              fa.maxDynamicSharedSizeBytes, fa.localSizeBytes, threads, smem);
}

// ---------------------------------------------------------------- per-device state
constexpr int kMaxDevices = 64;

struct DeviceInfo {
  std::once_flag once;
  int sm_count = 0;
  int err = 0;
};
DeviceInfo g_dev[kMaxDevices];

template <int MODE, bool TILED_B = false, bool ROUTED = false>
cudaError_t enable_gemm_smem() {
  return cudaFuncSetAttribute(blockscale_gemm_kernel<MODE, TILED_B, ROUTED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kGemmSmemBytes));
}

// Fetches the current device's SM count and opts every kernel into the shared
// memory it needs, once per device.
int device_setup(int* sm_count) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(FP8MOE_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(FP8MOE_ECUDA, "device ordinal %d unsupported", dev);
  DeviceInfo& d = g_dev[dev];
  std::call_once(d.once, [&] {
    cudaError_t r = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    int major = 0, minor = 0;
    if (r == cudaSuccess) r = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (r == cudaSuccess) r = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (r == cudaSuccess && !(major == 10 && minor == 0)) {
      d.err = -1;
      return;
    }
    if (r == cudaSuccess) r = enable_gemm_smem<kModeDense>();
    if (r == cudaSuccess) r = enable_gemm_smem<kModeMoeUp>();
    if (r == cudaSuccess) r = enable_gemm_smem<kModeMoeDown>();
    if (r == cudaSuccess) r = enable_gemm_smem<kModeMoeUp, true>();
    if (r == cudaSuccess) r = enable_gemm_smem<kModeMoeDown, true>();
    if (r == cudaSuccess) r = enable_gemm_smem<kModeMoeDown, false, true>();
    if (r == cudaSuccess) r = enable_gemm_smem<kModeMoeDown, true, true>();
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(mla_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMlaSmemBytes);
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(sort_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(sort_scatter_smem(kSortMaxExperts)));
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(sort_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (kSortWarps + 2) * kSortMaxExperts * static_cast<int>(sizeof(int)));
    d.err = static_cast<int>(r);
  });
  if (d.err == -1) return fail(FP8MOE_EUNSUPPORTED, "device %d is not sm_100 (B200)", dev);
  if (d.err != 0)
    return fail(FP8MOE_ECUDA, "device setup: %s", cudaGetErrorString(static_cast<cudaError_t>(d.err)));
  *sm_count = d.sm_count;
  return FP8MOE_OK;
}

// ---------------------------------------------------------------- TMA tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 2-D map over a row-major matrix [rows, cols] of `elem_bytes`-byte elements
// (row stride `ld_bytes`), box {box_cols, box_rows}, zero fill outside the matrix.
int make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* base, uint64_t rows,
                uint64_t cols, uint64_t ld_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FP8MOE_ECUDA, "cuTensorMapEncodeTiled unavailable");
  (void)elem_bytes;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(FP8MOE_ECUDA, "cuTensorMapEncodeTiled failed (%d) for [%llu x %llu]", static_cast<int>(r),
                static_cast<unsigned long long>(rows), static_cast<unsigned long long>(cols));
  return FP8MOE_OK;
}

// Operand tile map: FP8 bytes, box {128 bytes of K, 128 rows}, 128-byte swizzle.
int make_operand_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
  return make_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, rows, cols, cols, 128, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

// Map over weights in the tiled layout (fp8_tile_weights): 128 x 128-byte blocks,
// each 16 KB of consecutive bytes, ordered (row block, K block). Viewed as a 3-D
// tensor {128 bytes, 128 rows, block}; a box is one block; 128-byte swizzle.
int make_tiled_weight_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FP8MOE_ECUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[3] = {128, 128, (rows / 128) * (cols / 128)};
  const cuuint64_t strides[2] = {128, 128 * 128};
  const cuuint32_t box[3] = {128, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(FP8MOE_ECUDA, "cuTensorMapEncodeTiled failed (%d) for tiled weights [%llu x %llu]", static_cast<int>(r),
                static_cast<unsigned long long>(rows), static_cast<unsigned long long>(cols));
  return FP8MOE_OK;
}

// The same with a 64-row box (the first half of an M=64 tile's A rows).
int make_operand_map_64(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
  return make_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, rows, cols, cols, 128, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Scratch of the fused MoE call: the slot-ordered FP8 activations and their
// scales (capacity rows), the slot-ordered re-quantised intermediate and its
// scales, and the weighted down-projection rows of every pair (by pair id).
struct MoeWorkspace {
  size_t a8s_off, s1s_off, a2_off, s2_off, y_off, flag_off, total;
};

MoeWorkspace moe_workspace_layout(size_t capacity, int T, int topk, int H, int I) {
  MoeWorkspace w;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = round_up(off + bytes, 256);
    return at;
  };
  w.a8s_off = take(capacity * static_cast<size_t>(H));
  w.s1s_off = take(static_cast<size_t>(H / 128) * capacity * sizeof(float));
  w.a2_off = take(capacity * static_cast<size_t>(I));
  w.s2_off = take(static_cast<size_t>(I / 128) * capacity * sizeof(float));
  w.y_off = take(static_cast<size_t>(T) * topk * H * sizeof(__nv_bfloat16));
  w.flag_off = take(16 + static_cast<size_t>(T) * topk);   // listed-pair count, then 1 flag per pair
  w.total = off;
  return w;
}

struct TimingState {
  bool on = false;
  int dev = -1;
  cudaEvent_t ev[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
};
thread_local TimingState g_timing;

void timing_record(int i, cudaStream_t st) {
  if (!g_timing.on || !g_timing.ev[i]) return;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cap);
  // inside a stream capture an external record becomes an event node of the graph
  if (cap == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(g_timing.ev[i], st, cudaEventRecordExternal);
  else
    cudaEventRecord(g_timing.ev[i], st);
}

int choose_group_m(int n_tiles) {
  // Visit a few consecutive row blocks per column tile so blocks of the same
  // expert share each weight tile while it is in L2.
  return n_tiles >= 8 ? 4 : 16;
}

}  // namespace

// Routing for fp32 or bf16 logits (the two C entry points below).
template <typename LT>
static int route_impl(const char* name, const LT* gating_output, int ld_in, const float* correction_bias,
                      float* topk_weights, int32_t* topk_ids, int ld_out, int T, int E, int topk,
                      int num_expert_group, int topk_group, int need_renorm, float routed_scaling_factor,
                      void* stream) {
  if (T < 0) return fail(FP8MOE_EINVAL, "T must be >= 0 (got %d)", T);
  if (E < 1 || E > 32 * kRouteMaxPerLane) return fail(FP8MOE_EUNSUPPORTED, "E must be in [1, 512] (got %d)", E);
  if (num_expert_group < 1 || num_expert_group > 32 || E % num_expert_group != 0)
    return fail(FP8MOE_EINVAL, "num_expert_group must divide E and be <= 32 (E=%d, groups=%d)", E,
                num_expert_group);
  if (topk_group < 1 || topk_group > num_expert_group)
    return fail(FP8MOE_EINVAL, "topk_group must be in [1, num_expert_group] (got %d)", topk_group);
  const int per_group = E / num_expert_group;
  if (topk < 1 || topk > 32 || topk > topk_group * per_group)
    return fail(FP8MOE_EINVAL, "topk must be in [1, min(32, topk_group*E/groups)] (got %d)", topk);
  if (ld_in < E) return fail(FP8MOE_EINVAL, "ld_in (%d) < E (%d)", ld_in, E);
  if (ld_out < topk) return fail(FP8MOE_EINVAL, "ld_out (%d) < topk (%d)", ld_out, topk);
  if (T == 0) return FP8MOE_OK;
  if (!gating_output || !correction_bias || !topk_weights || !topk_ids)
    return fail(FP8MOE_EINVAL, "null pointer argument");
  // experts per lane: the smallest divisor of the group size that covers E with 32 lanes
  const int need = (E + 31) / 32;
  int per_lane = 0;
  for (int d = need; d <= per_group; ++d)
    if (per_group % d == 0) {
      per_lane = d;
      break;
    }
  if (per_lane == 0 || per_lane > kRouteMaxPerLane)
    return fail(FP8MOE_EUNSUPPORTED, "group size %d cannot be split over 32 lanes", per_group);
  int sms = 0;
  if (int rc = device_setup(&sms)) return rc;
  const dim3 grid((T + kRouteWarps - 1) / kRouteWarps);
  const uintptr_t lg = reinterpret_cast<uintptr_t>(gating_output);
  const int vec4 = (ld_in % 4 == 0) && (lg % (4 * sizeof(LT)) == 0) && aligned16(correction_bias);
  auto launch = [&](auto kernel) {
    kernel<<<grid, 32 * kRouteWarps, 0, static_cast<cudaStream_t>(stream)>>>(
        gating_output, ld_in, correction_bias, topk_weights, topk_ids, ld_out, T, E, topk, num_expert_group,
        topk_group, need_renorm ? 1 : 0, routed_scaling_factor, per_lane, vec4);
  };
  switch (per_lane) {
    case 1: launch(route_kernel<1, LT>); break;
    case 2: launch(route_kernel<2, LT>); break;
    case 4: launch(route_kernel<4, LT>); break;
    case 8: launch(route_kernel<8, LT>); break;
    case 16: launch(route_kernel<16, LT>); break;
    default: launch(route_kernel<0, LT>); break;
  }
  return check_launch(name);
}

extern "C" {

const char* fp8moe_last_error(void) { return g_last_error.c_str(); }

int fp8moe_moe_block_m(void) { return kBM; }

int fp8moe_timing_enable(int on) {
  if (!on) {
    g_timing.on = false;
    return FP8MOE_OK;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess && dev != g_timing.dev) {
    for (auto& ev : g_timing.ev) {
      if (ev) cudaEventDestroy(ev);
      ev = nullptr;
    }
    for (auto& ev : g_timing.ev)
      if (e == cudaSuccess) e = cudaEventCreate(&ev);
    g_timing.dev = dev;
  }
  if (e != cudaSuccess) return fail(FP8MOE_ECUDA, "timing events: %s", cudaGetErrorString(e));
  g_timing.on = true;
  return FP8MOE_OK;
}

int fp8moe_timing_last(float* ms) {
  if (!ms) return fail(FP8MOE_EINVAL, "null pointer argument");
  if (!g_timing.ev[4]) return fail(FP8MOE_EINVAL, "timing was never enabled");
  cudaError_t e = cudaEventSynchronize(g_timing.ev[4]);
  for (int i = 0; i < 4 && e == cudaSuccess; ++i) e = cudaEventElapsedTime(&ms[i], g_timing.ev[i], g_timing.ev[i + 1]);
  if (e != cudaSuccess) return fail(FP8MOE_ECUDA, "timing read: %s", cudaGetErrorString(e));
  return FP8MOE_OK;
}

int fp8moe_device_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    fail(FP8MOE_ECUDA, "stream synchronize: %s", cudaGetErrorString(e));
    return -1;
  }
  unsigned int word = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  if (e != cudaSuccess) {
    fail(FP8MOE_ECUDA, "device status: %s", cudaGetErrorString(e));
    return -1;
  }
  return static_cast<int>(word);
}

// ------------------------------------------------------------------ S1 routing
int moe_biased_grouped_topk(const float* gating_output, int ld_in, const float* correction_bias, float* topk_weights,
                            int32_t* topk_ids, int ld_out, int T, int E, int topk, int num_expert_group,
                            int topk_group, int need_renorm, float routed_scaling_factor, void* stream) {
  return route_impl("moe_biased_grouped_topk", gating_output, ld_in, correction_bias, topk_weights, topk_ids,
                    ld_out, T, E, topk, num_expert_group, topk_group, need_renorm, routed_scaling_factor, stream);
}

int moe_biased_grouped_topk_bf16(const uint16_t* gating_output, int ld_in, const float* correction_bias,
                                 float* topk_weights, int32_t* topk_ids, int ld_out, int T, int E, int topk,
                                 int num_expert_group, int topk_group, int need_renorm,
                                 float routed_scaling_factor, void* stream) {
  return route_impl("moe_biased_grouped_topk_bf16", reinterpret_cast<const __nv_bfloat16*>(gating_output), ld_in,
                    correction_bias, topk_weights, topk_ids, ld_out, T, E, topk, num_expert_group, topk_group,
                    need_renorm, routed_scaling_factor, stream);
}

// ------------------------------------------------------------------ S2 align/sort
size_t moe_align_sort_capacity(int T, int topk, int E, int block_m) {
  if (T < 0 || topk < 1 || E < 1 || block_m < 1) return 0;
  return static_cast<size_t>(T) * topk + static_cast<size_t>(E) * (block_m - 1);
}

size_t moe_align_sort_workspace(int T, int topk, int E, int block_m) {
  if (T < 0 || topk < 1 || E < 1 || block_m < 1) return 0;
  const size_t pairs = static_cast<size_t>(T) * topk;
  const size_t nchunks = (pairs + kSortChunk - 1) / kSortChunk;
  return round_up(nchunks * E * sizeof(int32_t), 256);
}

int moe_align_sort_masked(const int32_t* topk_ids, const float* topk_weights, int ld, int T, int topk, int E,
                          int block_m, const int32_t* expert_mask, int32_t* sorted_ids, float* sorted_weights,
                          int32_t* sorted_expert_ids, int32_t* num_valid_ids, size_t capacity, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (T < 0 || topk < 1) return fail(FP8MOE_EINVAL, "T >= 0 and topk >= 1 required");
  if (E < 1 || E > kSortMaxExperts) return fail(FP8MOE_EUNSUPPORTED, "E must be in [1, %d]", kSortMaxExperts);
  if (block_m < 1 || block_m > 1024) return fail(FP8MOE_EINVAL, "block_m must be in [1, 1024]");
  if (ld < topk) return fail(FP8MOE_EINVAL, "ld (%d) < topk (%d)", ld, topk);
  if (static_cast<long long>(T) * topk >= (1ll << 31)) return fail(FP8MOE_EUNSUPPORTED, "T*topk too large");
  if (capacity < moe_align_sort_capacity(T, topk, E, block_m))
    return fail(FP8MOE_EINVAL, "capacity %zu < required %zu", capacity, moe_align_sort_capacity(T, topk, E, block_m));
  if (!sorted_ids || !sorted_weights || !sorted_expert_ids || !num_valid_ids || (T > 0 && (!topk_ids || !topk_weights)))
    return fail(FP8MOE_EINVAL, "null pointer argument");
  const size_t need = moe_align_sort_workspace(T, topk, E, block_m);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(FP8MOE_EWORKSPACE, "workspace of %zu bytes needed (got %zu)", need, workspace_bytes);
  int sms = 0;
  if (int rc = device_setup(&sms)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int pairs = T * topk;
  const int nchunks = (pairs + kSortChunk - 1) / kSortChunk;
  if (nchunks <= 1) {                   // one chunk: count, offsets and scatter in a single CTA
    sort_small_kernel<<<1, kSortChunk, static_cast<size_t>(kSortWarps + 2) * E * sizeof(int), st>>>(
        topk_ids, topk_weights, ld, T, topk, E, expert_mask, block_m, sorted_ids, sorted_weights, sorted_expert_ids,
        num_valid_ids);
    return check_launch("moe_align_sort (single chunk)");
  }
  int32_t* counts = static_cast<int32_t*>(workspace);                       // [nchunks][E]
  sort_count_kernel<<<nchunks, kSortChunk, E * sizeof(int), st>>>(topk_ids, ld, T, topk, E, expert_mask, counts);
  if (int rc = check_launch("moe_align_sort (count)")) return rc;
  sort_scatter_kernel<<<nchunks, kSortChunk, sort_scatter_smem(E), st>>>(
      topk_ids, topk_weights, ld, T, topk, E, expert_mask, block_m, counts, nchunks, sorted_ids, sorted_weights,
      sorted_expert_ids, num_valid_ids);
  if (int rc = check_launch("moe_align_sort (scatter)")) return rc;
  return FP8MOE_OK;
}

int moe_align_sort(const int32_t* topk_ids, const float* topk_weights, int ld, int T, int topk, int E, int block_m,
                   int32_t* sorted_ids, float* sorted_weights, int32_t* sorted_expert_ids, int32_t* num_valid_ids,
                   size_t capacity, void* workspace, size_t workspace_bytes, void* stream) {
  return moe_align_sort_masked(topk_ids, topk_weights, ld, T, topk, E, block_m, nullptr, sorted_ids, sorted_weights,
                               sorted_expert_ids, num_valid_ids, capacity, workspace, workspace_bytes, stream);
}

// ------------------------------------------------------------------ S3 quant
int fp8_per_token_group_quant(const uint16_t* x, int ld_x, int M, int K, int group, uint8_t* q, float* scales,
                              int scale_layout, void* stream) {
  if (group != 128) return fail(FP8MOE_EUNSUPPORTED, "only group == 128 is supported (got %d)", group);
  if (M < 0 || K < 0) return fail(FP8MOE_EINVAL, "negative size");
  if (K % 8 != 0) return fail(FP8MOE_EUNSUPPORTED, "K must be a multiple of 8 (got %d)", K);
  if (ld_x < K || ld_x % 8 != 0) return fail(FP8MOE_EINVAL, "ld_x must be >= K and a multiple of 8");
  if (scale_layout != FP8MOE_SCALE_ROW_MAJOR && scale_layout != FP8MOE_SCALE_COL_MAJOR)
    return fail(FP8MOE_EINVAL, "unknown scale_layout %d", scale_layout);
  if (M == 0 || K == 0) return FP8MOE_OK;
  if (!x || !q || !scales) return fail(FP8MOE_EINVAL, "null pointer argument");
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(q) & 7u)) return fail(FP8MOE_EINVAL, "x must be 16-byte and q 8-byte aligned");
  int sms = 0;
  if (int rc = device_setup(&sms)) return rc;
  const long long warps = static_cast<long long>(M) * ((K + 128 * kQuantSpan - 1) / (128 * kQuantSpan));
  if ((warps + kQuantWarps - 1) / kQuantWarps >= (1ll << 31)) return fail(FP8MOE_EUNSUPPORTED, "M too large");
  const dim3 grid(static_cast<unsigned>((warps + kQuantWarps - 1) / kQuantWarps));
  quant_1x128_kernel<<<grid, 32 * kQuantWarps, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(x), ld_x, M, K, q, scales, scale_layout == FP8MOE_SCALE_COL_MAJOR);
  return check_launch("fp8_per_token_group_quant");
}

int fp8_per_block_quant(const float* w, int ld_w, int N, int K, int block, uint8_t* q, float* scales, void* stream) {
  if (block != 128) return fail(FP8MOE_EUNSUPPORTED, "only block == 128 is supported (got %d)", block);
  if (N < 0 || K < 0 || ld_w < K) return fail(FP8MOE_EINVAL, "bad size or stride");
  if (N == 0 || K == 0) return FP8MOE_OK;
  if (!w || !q || !scales) return fail(FP8MOE_EINVAL, "null pointer argument");
  if ((N + 127) / 128 > 65535) return fail(FP8MOE_EUNSUPPORTED, "N too large");
  int sms = 0;
  if (int rc = device_setup(&sms)) return rc;
  const dim3 grid((K + 127) / 128, (N + 127) / 128);
  quant_128x128_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(w, ld_w, N, K, q, scales);
  return check_launch("fp8_per_block_quant");
}

// ------------------------------------------------------------------ S0 GEMM
static int blockscale_gemm_impl(const char* name, const uint8_t* A, const uint8_t* B, const float* a_scale,
                                const float* b_scale, uint16_t* C, int ldc, int M, int N, int K, int stall_kb1,
                                void* stream) {
  if (M < 1 || N < 1 || K < 1) return fail(FP8MOE_EINVAL, "M, N, K must be >= 1");
  if (K % 16 != 0) return fail(FP8MOE_EUNSUPPORTED, "K must be a multiple of 16 (got %d)", K);
  if (ldc < N) return fail(FP8MOE_EINVAL, "ldc (%d) < N (%d)", ldc, N);
  if (!A || !B || !a_scale || !b_scale || !C) return fail(FP8MOE_EINVAL, "null pointer argument");
  if (!aligned16(A) || !aligned16(B)) return fail(FP8MOE_EINVAL, "A and B must be 16-byte aligned");
  int sms = 0;
  if (int rc = device_setup(&sms)) return rc;
  CUtensorMap ma, mb;
  if (int rc = make_operand_map(&ma, A, M, K)) return rc;
  if (int rc = make_operand_map(&mb, B, N, K)) return rc;
  GemmArgs a{};
  a.M = M;
  a.N = N;
  a.num_kb = (K + 127) / 128;
  a.n_tiles = (N + kBN - 1) / kBN;
  a.group_m = choose_group_m(a.n_tiles);
  a.a_scale = a_scale;
  a.b_scale = b_scale;
  a.nb_per_expert = (N + 127) / 128;
  a.nb_valid = a.nb_per_expert;
  a.C = reinterpret_cast<__nv_bfloat16*>(C);
  a.ldc = ldc;
  a.c_vec = (ldc % 16 == 0) && (reinterpret_cast<uintptr_t>(C) & 31u) == 0;   // 32-byte row stores
  a.b_rows_per_expert = 0;
  a.stall_kb1 = stall_kb1;
  const long long tiles = static_cast<long long>((M + kBM - 1) / kBM) * a.n_tiles;
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  blockscale_gemm_kernel<kModeDense><<<grid, kGemmThreads, kGemmSmemBytes, static_cast<cudaStream_t>(stream)>>>(
      ma, mb, ma, a);
  return check_gemm_launch(name, blockscale_gemm_kernel<kModeDense>, kGemmThreads, kGemmSmemBytes);
}

int fp8_blockscale_gemm(const uint8_t* A, const uint8_t* B, const float* a_scale, const float* b_scale, uint16_t* C,
                        int ldc, int M, int N, int K, void* stream) {
  return blockscale_gemm_impl("fp8_blockscale_gemm", A, B, a_scale, b_scale, C, ldc, M, N, K, 0, stream);
}

int fp8moe_selftest_gemm_stall(const uint8_t* A, const uint8_t* B, const float* a_scale, const float* b_scale,
                               uint16_t* C, int ldc, int M, int N, int K, int stall_kb, void* stream) {
  if (stall_kb < 0 || stall_kb >= (K + 127) / 128) return fail(FP8MOE_EINVAL, "stall_kb must be a K block index");
  return blockscale_gemm_impl("fp8moe_selftest_gemm_stall", A, B, a_scale, b_scale, C, ldc, M, N, K, stall_kb + 1,
                              stream);
}

// ------------------------------------------------------------------ S4-S7 fused MoE
size_t fused_moe_fp8_blockscale_g1u1_workspace(int T, int topk, int E, int H, int I, int block_m) {
  if (T < 0 || topk < 1 || E < 1 || H < 1 || I < 1 || block_m < 1) return 0;
  return moe_workspace_layout(moe_align_sort_capacity(T, topk, E, block_m), T, topk, H, I).total;
}

}  // extern "C"

// The fused MoE call on row-major (tiled == false) or tiled (fp8_tile_weights) weights;
// with combine == false it stops after the down GEMM (the weighted pair rows and the
// pair flags stay in the workspace) and out is not used. With srcs, the activation
// rows and scales are gathered from several sources (a8 and a1_scale unused; T is the
// sources' tokens together).
static int fused_moe_impl(const char* name, bool tiled, bool combine, uint16_t* out, const uint8_t* a8,
                          const uint8_t* w1,
                          const uint8_t* w2, const int32_t* sorted_ids, const float* sorted_weights,
                          const int32_t* sorted_expert_ids, const int32_t* num_valid_ids, int T, int H, int I, int E,
                          int topk, int block_m, size_t capacity, const float* a1_scale, const float* fc1_scale,
                          const float* fc2_scale, int scale_blk_n, int scale_blk_k, const float* fc2_smooth_scale,
                          void* workspace, size_t workspace_bytes, void* stream,
                          const GatherSources* srcs = nullptr, __nv_bfloat16* const* y_src_rows = nullptr,
                          uint8_t* const* y_src_flags = nullptr, int y_src_pairs = 0) {
  (void)name;
  if (scale_blk_n != 128 || scale_blk_k != 128)
    return fail(FP8MOE_EUNSUPPORTED, "only (128, 128) scale blocks are supported (got %d, %d)", scale_blk_n,
                scale_blk_k);
  if (fc2_smooth_scale) return fail(FP8MOE_EUNSUPPORTED, "fc2_smooth_scale must be NULL");
  if (block_m != kBM) return fail(FP8MOE_EUNSUPPORTED, "block_m must be %d (got %d)", kBM, block_m);
  if (T < 0 || E < 1 || topk < 1) return fail(FP8MOE_EINVAL, "bad T, E or topk");
  if (topk > 32) return fail(FP8MOE_EUNSUPPORTED, "topk must be <= 32 (got %d)", topk);
  if (H < 128 || I < 128 || H % 128 || I % 128)
    return fail(FP8MOE_EUNSUPPORTED, "H and I must be positive multiples of 128 (H=%d, I=%d)", H, I);
  if (static_cast<long long>(T) * topk >= (1ll << 31)) return fail(FP8MOE_EUNSUPPORTED, "T*topk too large");
  if (capacity < moe_align_sort_capacity(T, topk, E, block_m) || capacity >= (1ull << 31))
    return fail(FP8MOE_EINVAL, "capacity %zu below the sort's bound %zu", capacity,
                moe_align_sort_capacity(T, topk, E, block_m));
  if (T == 0) return FP8MOE_OK;
  if ((combine && !out) || (!srcs && (!a8 || !a1_scale)) || !w1 || !w2 || !sorted_ids || !sorted_weights ||
      !sorted_expert_ids || !num_valid_ids || !fc1_scale || !fc2_scale)
    return fail(FP8MOE_EINVAL, "null pointer argument");
  if (!aligned16(a8) || !aligned16(w1) || !aligned16(w2) || !aligned16(sorted_ids) || !aligned16(out))
    return fail(FP8MOE_EINVAL, "a8, w1, w2, sorted_ids and out must be 16-byte aligned");
  const MoeWorkspace lay = moe_workspace_layout(capacity, T, topk, H, I);
  if (!workspace || workspace_bytes < lay.total)
    return fail(FP8MOE_EWORKSPACE, "workspace of %zu bytes needed (got %zu)", lay.total, workspace_bytes);
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return fail(FP8MOE_EINVAL, "workspace must be 256-byte aligned");
  int sms = 0;
  if (int rc = device_setup(&sms)) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* a8s = ws + lay.a8s_off;
  float* s1s = reinterpret_cast<float*>(ws + lay.s1s_off);
  uint8_t* a2 = ws + lay.a2_off;
  float* s2 = reinterpret_cast<float*>(ws + lay.s2_off);
  __nv_bfloat16* ystage = reinterpret_cast<__nv_bfloat16*>(ws + lay.y_off);
  int* n_present = reinterpret_cast<int*>(ws + lay.flag_off);
  uint8_t* pair_flag = ws + lay.flag_off + 16;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  CUtensorMap m_a8s, m_w1, m_a2, m_w2;
  if (int rc = make_operand_map(&m_a8s, a8s, capacity, H)) return rc;
  if (int rc = make_operand_map(&m_a2, a2, capacity, I)) return rc;
  CUtensorMap m_a8s64, m_a264;
  if (int rc = make_operand_map_64(&m_a8s64, a8s, capacity, H)) return rc;
  if (int rc = make_operand_map_64(&m_a264, a2, capacity, I)) return rc;
  if (tiled) {
    if (int rc = make_tiled_weight_map(&m_w1, w1, static_cast<uint64_t>(E) * 2 * I, H)) return rc;
    if (int rc = make_tiled_weight_map(&m_w2, w2, static_cast<uint64_t>(E) * H, I)) return rc;
  } else {
    if (int rc = make_operand_map(&m_w1, w1, static_cast<uint64_t>(E) * 2 * I, H)) return rc;
    if (int rc = make_operand_map(&m_w2, w2, static_cast<uint64_t>(E) * H, I)) return rc;
  }

  // pairs absent from the sorted list (a masked-out expert, a dropped id) keep
  // flag 0 and add nothing in the combine
  if (cudaMemsetAsync(n_present, 0, 16 + static_cast<size_t>(T) * topk, st) != cudaSuccess)
    return check_launch("fused_moe (pair flags)");
  timing_record(0, st);
  // pair -> slot map of the gather, kept in the pair-row region (P * 4 <= P * H * 2
  // bytes) that the down GEMM writes only later
  int* inv = reinterpret_cast<int*>(ystage);
  if (srcs) {
    moe_gather_kernel<true><<<sms * 4, 32 * kGatherWarps, 0, st>>>(
        nullptr, sorted_ids, sorted_expert_ids, num_valid_ids, T, topk, H, static_cast<int>(capacity), s1s,
        pair_flag, n_present, inv, *srcs);
    if (int rc = check_launch("fused_moe (gather)")) return rc;
    moe_gather_rows_kernel<true><<<sms * 4, 32 * kGatherWarps, 0, st>>>(nullptr, T, topk, H, pair_flag, inv, a8s,
                                                                       *srcs);
  } else {
    moe_gather_kernel<<<sms * 4, 32 * kGatherWarps, 0, st>>>(a1_scale, sorted_ids, sorted_expert_ids, num_valid_ids,
                                                              T, topk, H, static_cast<int>(capacity), s1s, pair_flag,
                                                              n_present, inv);
    if (int rc = check_launch("fused_moe (gather)")) return rc;
    moe_gather_rows_kernel<<<sms * 4, 32 * kGatherWarps, 0, st>>>(a8, T, topk, H, pair_flag, inv, a8s);
  }
  if (int rc = check_launch("fused_moe (gather rows)")) return rc;
  timing_record(1, st);

  GemmArgs up{};
  up.M = static_cast<int>(capacity);
  up.N = I;
  up.num_kb = H / 128;
  up.n_tiles = I / 128;
  up.group_m = choose_group_m(up.n_tiles);
  up.a_scale = s1s;
  up.b_scale = fc1_scale;
  up.nb_per_expert = 2 * I / 128;
  up.nb_valid = up.nb_per_expert;
  up.sorted_ids = sorted_ids;
  up.sorted_expert_ids = sorted_expert_ids;
  up.num_valid_ids = num_valid_ids;
  up.sorted_weights = sorted_weights;
  up.T = T;
  up.topk = topk;
  up.E = E;
  up.b_rows_per_expert = 2 * I;
  up.a2 = a2;
  up.s2 = s2;
  up.ystage = ystage;
  if (tiled)
    blockscale_gemm_kernel<kModeMoeUp, true><<<sms, kGemmThreads, kGemmSmemBytes, st>>>(m_a8s, m_w1, m_a8s64, up);
  else
    blockscale_gemm_kernel<kModeMoeUp><<<sms, kGemmThreads, kGemmSmemBytes, st>>>(m_a8s, m_w1, m_a8s64, up);
  if (int rc = check_gemm_launch("fused_moe (gate/up GEMM)", blockscale_gemm_kernel<kModeMoeUp>, kGemmThreads,
                                 kGemmSmemBytes))
    return rc;
  timing_record(2, st);

  GemmArgs dn = up;
  dn.N = H;
  dn.num_kb = I / 128;
  dn.n_tiles = (H + kBN - 1) / kBN;
  dn.group_m = choose_group_m(dn.n_tiles);
  dn.a_scale = s2;
  dn.b_scale = fc2_scale;
  dn.nb_per_expert = H / 128;
  dn.nb_valid = H / 128;
  dn.b_rows_per_expert = H;
  dn.s2 = nullptr;
  dn.y_src_rows = y_src_rows;
  dn.y_src_flags = y_src_flags;
  dn.y_src_pairs = y_src_pairs;
  if (dn.y_src_rows && tiled)
    blockscale_gemm_kernel<kModeMoeDown, true, true><<<sms, kGemmThreads, kGemmSmemBytes, st>>>(m_a2, m_w2, m_a264, dn);
  else if (dn.y_src_rows)
    blockscale_gemm_kernel<kModeMoeDown, false, true><<<sms, kGemmThreads, kGemmSmemBytes, st>>>(m_a2, m_w2, m_a264, dn);
  else if (tiled)
    blockscale_gemm_kernel<kModeMoeDown, true><<<sms, kGemmThreads, kGemmSmemBytes, st>>>(m_a2, m_w2, m_a264, dn);
  else
    blockscale_gemm_kernel<kModeMoeDown><<<sms, kGemmThreads, kGemmSmemBytes, st>>>(m_a2, m_w2, m_a264, dn);
  if (int rc = check_gemm_launch("fused_moe (down GEMM)", blockscale_gemm_kernel<kModeMoeDown>, kGemmThreads,
                                 kGemmSmemBytes))
    return rc;
  timing_record(3, st);
  if (!combine) return FP8MOE_OK;

  const size_t threads = static_cast<size_t>(T) * (H / 8);
  moe_combine_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(
      ystage, pair_flag, n_present, T, topk, H, reinterpret_cast<__nv_bfloat16*>(out));
  if (int rc = check_launch("fused_moe (combine)")) return rc;
  timing_record(4, st);
  return FP8MOE_OK;
}

extern "C" {

int fused_moe_fp8_blockscale_g1u1(uint16_t* out, const uint8_t* a8, const uint8_t* w1, const uint8_t* w2,
                                  const int32_t* sorted_ids, const float* sorted_weights,
                                  const int32_t* sorted_expert_ids, const int32_t* num_valid_ids, int T, int H, int I,
                                  int E, int topk, int block_m, size_t capacity, const float* a1_scale,
                                  const float* fc1_scale, const float* fc2_scale, int scale_blk_n, int scale_blk_k,
                                  const float* fc2_smooth_scale, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  return fused_moe_impl("fused_moe_fp8_blockscale_g1u1", false, true, out, a8, w1, w2, sorted_ids, sorted_weights,
                        sorted_expert_ids, num_valid_ids, T, H, I, E, topk, block_m, capacity, a1_scale, fc1_scale,
                        fc2_scale, scale_blk_n, scale_blk_k, fc2_smooth_scale, workspace, workspace_bytes, stream);
}

int fused_moe_fp8_blockscale_g1u1_tiled(uint16_t* out, const uint8_t* a8, const uint8_t* w1, const uint8_t* w2,
                                        const int32_t* sorted_ids, const float* sorted_weights,
                                        const int32_t* sorted_expert_ids, const int32_t* num_valid_ids, int T, int H,
                                        int I, int E, int topk, int block_m, size_t capacity, const float* a1_scale,
                                        const float* fc1_scale, const float* fc2_scale, int scale_blk_n,
                                        int scale_blk_k, const float* fc2_smooth_scale, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  return fused_moe_impl("fused_moe_fp8_blockscale_g1u1_tiled", true, true, out, a8, w1, w2, sorted_ids, sorted_weights,
                        sorted_expert_ids, num_valid_ids, T, H, I, E, topk, block_m, capacity, a1_scale, fc1_scale,
                        fc2_scale, scale_blk_n, scale_blk_k, fc2_smooth_scale, workspace, workspace_bytes, stream);
}

// ------------------------------------------------------------------ weight re-pack
int fp8_tile_weights(const uint8_t* w, int E, int N, int K, uint8_t* out, void* stream) {
  if (E < 1 || E > 65535) return fail(FP8MOE_EINVAL, "E must be in [1, 65535] (got %d)", E);
  if (N < 128 || K < 128 || N % 128 || K % 128)
    return fail(FP8MOE_EUNSUPPORTED, "N and K must be positive multiples of 128 (N=%d, K=%d)", N, K);
  if (N / 128 > 65535 || K / 128 > 65535) return fail(FP8MOE_EUNSUPPORTED, "N or K too large");
  if (!w || !out) return fail(FP8MOE_EINVAL, "null pointer argument");
  if (!aligned16(w) || !aligned16(out)) return fail(FP8MOE_EINVAL, "w and out must be 16-byte aligned");
  const size_t bytes = static_cast<size_t>(E) * N * K;
  const uintptr_t a = reinterpret_cast<uintptr_t>(w), b = reinterpret_cast<uintptr_t>(out);
  if (a < b + bytes && b < a + bytes) return fail(FP8MOE_EINVAL, "w and out overlap");
  int sms = 0;
  if (int rc = device_setup(&sms)) return rc;
  const dim3 grid(K / 128, N / 128, E);
  tile_weights_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(w, N, K, out);
  return check_launch("fp8_tile_weights");
}

// ------------------------------------------------------------------ no-allocation variant
// The fused call's scratch for callers that cannot allocate device memory: one
// fixed array per device, held for the life of the process. Its name is only a
// host-side handle; the device address comes from cudaGetSymbolAddress, looked
// up on the first successful call on each device (with that device current).
}  // extern "C"

namespace {
static __device__ __align__(256) unsigned char g_noalloc_scratch[FP8MOE_NOALLOC_SCRATCH_BYTES];

// The looked-up address of the scratch array on each device. A failed lookup
// (for example one made while the stream was being captured) is not kept: the
// next call on that device tries again.
struct NoAllocScratch {
  std::mutex mu;
  void* ptr = nullptr;
};
NoAllocScratch g_noalloc[kMaxDevices];
}  // namespace

extern "C" {

int fused_moe_fp8_blockscale_g1u1_noalloc(uint16_t* out, const uint8_t* a8, const uint8_t* w1, const uint8_t* w2,
                                          const int32_t* sorted_ids, const float* sorted_weights,
                                          const int32_t* sorted_expert_ids, const int32_t* num_valid_ids, int T,
                                          int H, int I, int E, int topk, int block_m, size_t capacity,
                                          const float* a1_scale, const float* fc1_scale, const float* fc2_scale,
                                          int scale_blk_n, int scale_blk_k, const float* fc2_smooth_scale,
                                          void* stream) {
  if (T < 0 || topk < 1 || H < 1 || I < 1) return fail(FP8MOE_EINVAL, "bad T, topk, H or I");
  const size_t need = moe_workspace_layout(capacity, T, topk, H, I).total;
  if (need > FP8MOE_NOALLOC_SCRATCH_BYTES)
    return fail(FP8MOE_EUNSUPPORTED,
                "fused_moe_fp8_blockscale_g1u1_noalloc: this problem needs %zu bytes of scratch, more than the "
                "built-in %llu bytes; use fused_moe_fp8_blockscale_g1u1 with a caller-provided workspace",
                need, static_cast<unsigned long long>(FP8MOE_NOALLOC_SCRATCH_BYTES));
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(FP8MOE_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(FP8MOE_ECUDA, "device ordinal %d unsupported", dev);
  NoAllocScratch& sc = g_noalloc[dev];
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(sc.mu);
    if (!sc.ptr) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || !p) {
        cudaGetLastError();   // the failed lookup leaves no sticky error behind; the next call retries
        return fail(FP8MOE_ECUDA, "scratch address lookup: %s", cudaGetErrorString(e));
      }
      sc.ptr = p;
    }
    scratch = sc.ptr;
  }
  return fused_moe_fp8_blockscale_g1u1(out, a8, w1, w2, sorted_ids, sorted_weights, sorted_expert_ids,
                                       num_valid_ids, T, H, I, E, topk, block_m, capacity, a1_scale, fc1_scale,
                                       fc2_scale, scale_blk_n, scale_blk_k, fc2_smooth_scale, scratch,
                                       FP8MOE_NOALLOC_SCRATCH_BYTES, stream);
}

// ------------------------------------------------------------------ tensor-parallel combine + all-reduce
int fused_moe_fp8_blockscale_g1u1_pairs(const uint8_t* a8, const uint8_t* w1, const uint8_t* w2,
                                        const int32_t* sorted_ids, const float* sorted_weights,
                                        const int32_t* sorted_expert_ids, const int32_t* num_valid_ids, int T, int H,
                                        int I, int E, int topk, int block_m, size_t capacity, const float* a1_scale,
                                        const float* fc1_scale, const float* fc2_scale, int scale_blk_n,
                                        int scale_blk_k, const float* fc2_smooth_scale, int weights_tiled,
                                        void* workspace, size_t workspace_bytes, void* stream) {
  return fused_moe_impl("fused_moe_fp8_blockscale_g1u1_pairs", weights_tiled != 0, false, nullptr, a8, w1, w2,
                        sorted_ids, sorted_weights, sorted_expert_ids, num_valid_ids, T, H, I, E, topk, block_m,
                        capacity, a1_scale, fc1_scale, fc2_scale, scale_blk_n, scale_blk_k, fc2_smooth_scale,
                        workspace, workspace_bytes, stream);
}

size_t moe_tp_recv_bytes(int T, int H, int nranks) {
  if (T < 0 || H < 0 || nranks < 1 || nranks > FP8MOE_TP_MAX_RANKS) return 0;
  const size_t Ts = (static_cast<size_t>(T) + nranks - 1) / nranks;
  return static_cast<size_t>(nranks) * Ts * H * sizeof(__nv_bfloat16);
}

}  // extern "C"

static_assert(FP8MOE_TP_MAX_RANKS == kTpMaxRanks && FP8MOE_TP_FLAG_WORDS == kTpFlagWords &&
                  FP8MOE_TP_BARRIER_WORDS == kTpBarrierWords,
              "header and kernel agree");

// Checks shared by the one-rank and the emulated launches: fills `a` (the peer
// buffers, and the workspace buffers of the nlocal ranks launched here) and
// *ctas (CTAs per rank: all of the launch must be resident at once).
static int tp_setup(const char* name, int nranks, int T, int topk, int H, int I, size_t capacity,
                    const void* const* workspaces, const int* ranks, int nlocal, void* const* recv,
                    void* const* out, uint64_t* const* flags, uint64_t* const* barriers, TpArgs* a,
                    int* ctas) {
  if (nranks < 1 || nranks > kTpMaxRanks) return fail(FP8MOE_EINVAL, "%s: nranks must be in [1, %d]", name, kTpMaxRanks);
  if (T < 1 || topk < 1 || topk > 32) return fail(FP8MOE_EINVAL, "%s: T >= 1 and topk in [1, 32] required", name);
  if (H < 128 || H % 128 || I < 128 || I % 128)
    return fail(FP8MOE_EUNSUPPORTED, "%s: H and I must be positive multiples of 128", name);
  if (static_cast<long long>(T) * topk >= (1ll << 31) || static_cast<long long>(T) * (H / 8) >= (1ll << 40))
    return fail(FP8MOE_EUNSUPPORTED, "%s: T too large", name);
  if (!recv || !out || !flags) return fail(FP8MOE_EINVAL, "%s: null pointer argument", name);
  *a = TpArgs{};
  for (int p = 0; p < nranks; ++p) {
    if (!recv[p] || !out[p] || !flags[p]) return fail(FP8MOE_EINVAL, "%s: null buffer of rank %d", name, p);
    if (!aligned16(recv[p]) || !aligned16(out[p]) || (reinterpret_cast<uintptr_t>(flags[p]) & 7u))
      return fail(FP8MOE_EINVAL, "%s: rank %d's buffers must be 16-byte (flags 8-byte) aligned", name, p);
    a->recv[p] = static_cast<__nv_bfloat16*>(recv[p]);
    a->out[p] = static_cast<__nv_bfloat16*>(out[p]);
    a->flags[p] = reinterpret_cast<unsigned long long*>(flags[p]);
  }
  const MoeWorkspace lay = moe_workspace_layout(capacity, T, topk, H, I);
  for (int i = 0; i < nlocal; ++i) {
    const int r = ranks[i];
    if (!workspaces[i] || !barriers[i]) return fail(FP8MOE_EINVAL, "%s: null workspace or barrier", name);
    if (reinterpret_cast<uintptr_t>(workspaces[i]) & 255u)
      return fail(FP8MOE_EINVAL, "%s: workspace must be 256-byte aligned", name);
    if (reinterpret_cast<uintptr_t>(barriers[i]) & 7u) return fail(FP8MOE_EINVAL, "%s: barrier must be 8-byte aligned", name);
    const uint8_t* ws = static_cast<const uint8_t*>(workspaces[i]);
    a->ystage[r] = reinterpret_cast<const __nv_bfloat16*>(ws + lay.y_off);
    a->n_present[r] = reinterpret_cast<const int*>(ws + lay.flag_off);
    a->pair_flag[r] = ws + lay.flag_off + 16;
    a->barrier[r] = reinterpret_cast<unsigned long long*>(barriers[i]);
  }
  a->nranks = nranks;
  a->T = T;
  a->K = topk;
  a->H = H;
  int sms = 0;
  if (int rc = device_setup(&sms)) return rc;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tp_combine_allreduce_kernel, kTpThreads, 0) !=
          cudaSuccess || per_sm < 1)
    return fail(FP8MOE_ECUDA, "%s: occupancy query failed", name);
  const long long resident = static_cast<long long>(per_sm) * sms / nlocal;
  const long long need = (static_cast<long long>(T) * (H / 8) + kTpThreads - 1) / kTpThreads;
  *ctas = static_cast<int>(std::min(resident, need));
  if (*ctas < 1) return fail(FP8MOE_EUNSUPPORTED, "%s: %d ranks do not fit one GPU", name, nlocal);
  return FP8MOE_OK;
}

// A cooperative launch (every CTA resident at once) through cudaLaunchKernelEx, which
// stream capture records as a cooperative kernel node of the graph.
template <typename... KArgs, typename... Args>
static cudaError_t launch_cooperative(void (*kernel)(KArgs...), dim3 grid, dim3 block, cudaStream_t st,
                                      Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

static int tp_launch(const char* name, const TpArgs& a, int rank_first, int ctas, int nlocal, void* stream) {
  const cudaError_t e = launch_cooperative(tp_combine_allreduce_kernel, dim3(ctas * nlocal), dim3(kTpThreads),
                                           static_cast<cudaStream_t>(stream), a, rank_first, ctas);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FP8MOE_ECUDA, "%s: launch failed: %s", name, cudaGetErrorString(e));
  }
  return check_launch(name);
}

extern "C" {

int moe_combine_allreduce(const void* workspace, size_t capacity, int T, int topk, int H, int I, int nranks,
                          int rank, void* const* recv, void* const* out, uint64_t* const* flags, uint64_t* barrier,
                          void* stream) {
  if (nranks < 1 || rank < 0 || rank >= nranks) return fail(FP8MOE_EINVAL, "moe_combine_allreduce: bad rank");
  TpArgs a;
  int ctas = 0;
  const void* ws[1] = {workspace};
  uint64_t* bars[1] = {barrier};
  const int ranks[1] = {rank};
  if (int rc = tp_setup("moe_combine_allreduce", nranks, T, topk, H, I, capacity, ws, ranks, 1, recv, out, flags,
                        bars, &a, &ctas))
    return rc;
  return tp_launch("moe_combine_allreduce", a, rank, ctas, 1, stream);
}

int moe_combine_allreduce_emulated(const void* const* workspaces, size_t capacity, int T, int topk, int H, int I,
                                   int nranks, void* const* recv, void* const* out, uint64_t* const* flags,
                                   uint64_t* const* barriers, void* stream) {
  if (!workspaces || !barriers) return fail(FP8MOE_EINVAL, "moe_combine_allreduce_emulated: null pointer argument");
  if (nranks < 1 || nranks > kTpMaxRanks) return fail(FP8MOE_EINVAL, "moe_combine_allreduce_emulated: bad nranks");
  TpArgs a;
  int ctas = 0;
  int ranks[kTpMaxRanks];
  for (int r = 0; r < nranks; ++r) ranks[r] = r;
  if (int rc = tp_setup("moe_combine_allreduce_emulated", nranks, T, topk, H, I, capacity, workspaces, ranks, nranks,
                        recv, out, flags, barriers, &a, &ctas))
    return rc;
  return tp_launch("moe_combine_allreduce_emulated", a, 0, ctas, nranks, stream);
}

}  // extern "C"

// ------------------------------------------------------------------ expert-parallel dispatch and return
static_assert(FP8MOE_EP_MAX_RANKS == kMaxSources && FP8MOE_EP_BARRIER_WORDS == kEpBarrierWords,
              "header and kernels agree");

extern "C" {

int moe_ep_routing(const int32_t* const* ids, const float* const* w, int n, int Tq, int topk, int E, int e0, int ne,
                   int32_t* ids_out, float* w_out, void* stream) {
  if (n < 1 || n > kMaxSources) return fail(FP8MOE_EINVAL, "moe_ep_routing: n must be in [1, %d]", kMaxSources);
  if (Tq < 0 || topk < 1 || E < 1 || ne < 1 || e0 < 0 || e0 + ne > E)
    return fail(FP8MOE_EINVAL, "moe_ep_routing: bad sizes (Tq=%d, topk=%d, E=%d, e0=%d, ne=%d)", Tq, topk, E, e0, ne);
  if (static_cast<long long>(Tq) * topk * n >= (1ll << 31)) return fail(FP8MOE_EUNSUPPORTED, "moe_ep_routing: too many pairs");
  if (Tq == 0) return FP8MOE_OK;
  if (!ids || !w || !ids_out || !w_out) return fail(FP8MOE_EINVAL, "moe_ep_routing: null pointer argument");
  EpRouting src{};
  for (int q = 0; q < n; ++q) {
    if (!ids[q] || !w[q]) return fail(FP8MOE_EINVAL, "moe_ep_routing: null routing of rank %d", q);
    src.ids[q] = ids[q];
    src.w[q] = w[q];
  }
  int sms = 0;
  if (int rc = device_setup(&sms)) return rc;
  const long long total = static_cast<long long>(Tq) * topk * n;
  const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 4ll * sms));
  ep_routing_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(src, n, Tq, topk, E, e0, ne, ids_out,
                                                                           w_out);
  return check_launch("moe_ep_routing");
}

int fused_moe_fp8_blockscale_g1u1_multi(const uint8_t* const* a8, const float* const* a1_scale, int n, int Tq,
                                        const uint8_t* w1, const uint8_t* w2, const int32_t* sorted_ids,
                                        const float* sorted_weights, const int32_t* sorted_expert_ids,
                                        const int32_t* num_valid_ids, int H, int I, int E, int topk, int block_m,
                                        size_t capacity, const float* fc1_scale, const float* fc2_scale,
                                        int scale_blk_n, int scale_blk_k, const float* fc2_smooth_scale,
                                        int weights_tiled, void* const* return_rows, void* const* return_flags,
                                        void* workspace, size_t workspace_bytes, void* stream) {
  if (n < 1 || n > kMaxSources) return fail(FP8MOE_EINVAL, "n must be in [1, %d]", kMaxSources);
  if ((return_rows == nullptr) != (return_flags == nullptr))
    return fail(FP8MOE_EINVAL, "return_rows and return_flags are given together or not at all");
  if (Tq < 0 || static_cast<long long>(Tq) * n >= (1ll << 31)) return fail(FP8MOE_EINVAL, "bad Tq");
  if (!a8 || !a1_scale) return fail(FP8MOE_EINVAL, "null pointer argument");
  GatherSources srcs{};
  for (int q = 0; q < n; ++q) {
    if (!a8[q] || !a1_scale[q]) return fail(FP8MOE_EINVAL, "null activations of source %d", q);
    if (!aligned16(a8[q])) return fail(FP8MOE_EINVAL, "activations of source %d must be 16-byte aligned", q);
    srcs.a8[q] = a8[q];
    srcs.a1_scale[q] = a1_scale[q];
  }
  srcs.n = n;
  srcs.Tq = Tq;
  return fused_moe_impl("fused_moe_fp8_blockscale_g1u1_multi", weights_tiled != 0, false, nullptr, nullptr, w1, w2,
                        sorted_ids, sorted_weights, sorted_expert_ids, num_valid_ids, n * Tq, H, I, E, topk, block_m,
                        capacity, nullptr, fc1_scale, fc2_scale, scale_blk_n, scale_blk_k, fc2_smooth_scale, workspace,
                        workspace_bytes, stream, &srcs, reinterpret_cast<__nv_bfloat16* const*>(return_rows),
                        reinterpret_cast<uint8_t* const*>(return_flags), Tq * topk);
}

int moe_ep_return(const void* workspace, size_t capacity, int n, int Tq, int topk, int H, int I,
                  const int32_t* sorted_ids, const int32_t* num_valid_ids, void* const* rows, void* const* pair_flags,
                  void* stream) {
  if (n < 1 || n > kMaxSources) return fail(FP8MOE_EINVAL, "moe_ep_return: n must be in [1, %d]", kMaxSources);
  if (Tq < 0 || topk < 1 || H < 128 || H % 128 || I < 128 || I % 128 || capacity >= (1ull << 31))
    return fail(FP8MOE_EINVAL, "moe_ep_return: bad sizes");
  if (static_cast<long long>(Tq) * topk * n >= (1ll << 31)) return fail(FP8MOE_EUNSUPPORTED, "moe_ep_return: too many pairs");
  if (Tq == 0) return FP8MOE_OK;
  if (!workspace || !sorted_ids || !num_valid_ids || !rows || !pair_flags)
    return fail(FP8MOE_EINVAL, "moe_ep_return: null pointer argument");
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return fail(FP8MOE_EINVAL, "moe_ep_return: workspace alignment");
  EpReturn dst{};
  for (int q = 0; q < n; ++q) {
    if (!rows[q] || !pair_flags[q]) return fail(FP8MOE_EINVAL, "moe_ep_return: null buffer of rank %d", q);
    if (!aligned16(rows[q])) return fail(FP8MOE_EINVAL, "moe_ep_return: rows of rank %d must be 16-byte aligned", q);
    dst.rows[q] = static_cast<__nv_bfloat16*>(rows[q]);
    dst.flags[q] = static_cast<uint8_t*>(pair_flags[q]);
  }
  const MoeWorkspace lay = moe_workspace_layout(capacity, n * Tq, topk, H, I);
  const auto* ystage = reinterpret_cast<const __nv_bfloat16*>(static_cast<const uint8_t*>(workspace) + lay.y_off);
  int sms = 0;
  if (int rc = device_setup(&sms)) return rc;
  ep_return_kernel<<<sms * 4, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      sorted_ids, num_valid_ids, static_cast<int>(capacity), ystage, n, Tq * topk, H, dst);
  return check_launch("moe_ep_return");
}

static int ep_barrier_launch(const char* name, int n, int rank_first, int ctas, uint64_t* const* words,
                             void* stream) {
  if (n < 1 || n > kMaxSources) return fail(FP8MOE_EINVAL, "%s: n must be in [1, %d]", name, kMaxSources);
  if (!words) return fail(FP8MOE_EINVAL, "%s: null pointer argument", name);
  EpBarrierArgs a{};
  for (int p = 0; p < n; ++p) {
    if (!words[p] || (reinterpret_cast<uintptr_t>(words[p]) & 7u))
      return fail(FP8MOE_EINVAL, "%s: barrier words of rank %d null or not 8-byte aligned", name, p);
    a.flags[p] = reinterpret_cast<unsigned long long*>(words[p]);
  }
  a.n = n;
  int sms = 0;
  if (int rc = device_setup(&sms)) return rc;
  const cudaError_t e = launch_cooperative(ep_barrier_kernel, dim3(ctas), dim3(32), static_cast<cudaStream_t>(stream),
                                           a, rank_first);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FP8MOE_ECUDA, "%s: launch failed: %s", name, cudaGetErrorString(e));
  }
  return check_launch(name);
}

int moe_ep_barrier(int n, int rank, uint64_t* const* words, void* stream) {
  if (rank < 0 || rank >= n) return fail(FP8MOE_EINVAL, "moe_ep_barrier: bad rank");
  return ep_barrier_launch("moe_ep_barrier", n, rank, 1, words, stream);
}

int moe_ep_barrier_emulated(int n, uint64_t* const* words, void* stream) {
  return ep_barrier_launch("moe_ep_barrier_emulated", n, 0, n, words, stream);
}

int moe_combine_pairs(const uint16_t* rows, const void* flag_region, int T, int topk, int H, uint16_t* out,
                      void* stream) {
  if (T < 0 || topk < 1 || topk > 32 || H < 8 || H % 8) return fail(FP8MOE_EINVAL, "moe_combine_pairs: bad sizes");
  if (static_cast<long long>(T) * topk >= (1ll << 31)) return fail(FP8MOE_EUNSUPPORTED, "moe_combine_pairs: T too large");
  if (T == 0) return FP8MOE_OK;
  if (!rows || !flag_region || !out) return fail(FP8MOE_EINVAL, "moe_combine_pairs: null pointer argument");
  if (!aligned16(rows) || !aligned16(out) || (reinterpret_cast<uintptr_t>(flag_region) & 15u))
    return fail(FP8MOE_EINVAL, "moe_combine_pairs: rows, out and the flag region must be 16-byte aligned");
  const int* count = static_cast<const int*>(flag_region);
  const uint8_t* flags = static_cast<const uint8_t*>(flag_region) + 16;
  const size_t threads = static_cast<size_t>(T) * (H / 8);
  moe_combine_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(rows), flags, count, T, topk, H, reinterpret_cast<__nv_bfloat16*>(out));
  return check_launch("moe_combine_pairs");
}

}  // extern "C"

// ------------------------------------------------------------------ MLA decode
extern "C" {

int mla_decode_num_splits(int batch, int num_heads) {
  if (batch < 1 || num_heads < kMlaHeads) return 1;
  const long long ctas = static_cast<long long>(batch) * (num_heads / kMlaHeads);
  return static_cast<int>(std::max(1ll, std::min<long long>(kMlaMaxSplits, FP8MOE_MLA_TARGET_CTAS / ctas)));
}

size_t mla_decode_workspace(int batch, int num_heads, int num_kv_splits) {
  const int splits = num_kv_splits > 0 ? num_kv_splits : mla_decode_num_splits(batch, num_heads);
  if (batch < 1 || num_heads < 1 || splits <= 1) return 0;
  return static_cast<size_t>(batch) * num_heads * splits * (kMlaDv + 1) * sizeof(float);
}

int mla_decode_fwd(const uint16_t* q, const uint16_t* kv_buffer, uint16_t* o, const int32_t* kv_indptr,
                   const int32_t* kv_indices, const int32_t* kv_last_page_lens, float* lse, int batch, int num_heads,
                   int num_pages, int page_size, int num_indices, float sm_scale, float logit_cap, int num_kv_splits,
                   void* workspace, size_t workspace_bytes, void* stream) {
  if (batch < 0 || num_pages < 0 || num_indices < 0) return fail(FP8MOE_EINVAL, "mla_decode_fwd: negative size");
  if (num_heads < kMlaHeads || num_heads > 128 || num_heads % kMlaHeads)
    return fail(FP8MOE_EUNSUPPORTED, "mla_decode_fwd: num_heads must be 16, 32, ..., 128 (got %d)", num_heads);
  if (page_size < 1) return fail(FP8MOE_EINVAL, "mla_decode_fwd: page_size must be >= 1");
  if (!(sm_scale > 0.0f) || !std::isfinite(sm_scale)) return fail(FP8MOE_EINVAL, "mla_decode_fwd: sm_scale must be finite and > 0");
  if (!(logit_cap >= 0.0f) || !std::isfinite(logit_cap)) return fail(FP8MOE_EINVAL, "mla_decode_fwd: logit_cap must be finite and >= 0");
  if (num_kv_splits > kMlaMaxSplits) return fail(FP8MOE_EUNSUPPORTED, "mla_decode_fwd: at most %d splits", kMlaMaxSplits);
  if (batch == 0) return FP8MOE_OK;
  if (batch > 65535) return fail(FP8MOE_EUNSUPPORTED, "mla_decode_fwd: batch above 65535");
  if (!q || !o || !kv_indptr || !kv_last_page_lens) return fail(FP8MOE_EINVAL, "mla_decode_fwd: null pointer argument");
  if ((num_indices > 0 && (!kv_indices || !kv_buffer || num_pages < 1)))
    return fail(FP8MOE_EINVAL, "mla_decode_fwd: page indices given without a KV buffer");
  if (!aligned16(q) || !aligned16(o) || (kv_buffer && !aligned16(kv_buffer)))
    return fail(FP8MOE_EINVAL, "mla_decode_fwd: q, o and kv_buffer must be 16-byte aligned");
  if (static_cast<long long>(num_pages) * page_size * kMlaDk >= (1ll << 40))
    return fail(FP8MOE_EUNSUPPORTED, "mla_decode_fwd: KV buffer too large");
  if (static_cast<long long>(num_indices) * page_size >= (1ll << 31))   // token positions are int32 in the kernel
    return fail(FP8MOE_EUNSUPPORTED, "mla_decode_fwd: num_indices x page_size must stay below 2^31");
  const int splits = num_kv_splits > 0 ? num_kv_splits : mla_decode_num_splits(batch, num_heads);
  const size_t need = mla_decode_workspace(batch, num_heads, splits);
  if (need && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(FP8MOE_EWORKSPACE, "mla_decode_fwd: workspace of %zu bytes (16-byte aligned) needed", need);
  int sms = 0;
  if (int rc = device_setup(&sms)) return rc;
  MlaArgs a{};
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.kv = reinterpret_cast<const __nv_bfloat16*>(kv_buffer);
  a.o = reinterpret_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.indptr = kv_indptr;
  a.indices = kv_indices;
  a.last_lens = kv_last_page_lens;
  a.part_o = need ? static_cast<float*>(workspace) : nullptr;
  a.part_lse = need ? a.part_o + static_cast<size_t>(batch) * num_heads * splits * kMlaDv : nullptr;
  a.B = batch;
  a.Hq = num_heads;
  a.num_pages = num_pages;
  a.page_size = page_size;
  a.num_indices = num_indices;
  a.splits = splits;
  a.sm_scale = sm_scale;
  a.logit_cap = logit_cap;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 grid(num_heads / kMlaHeads, splits, batch);
  mla_decode_kernel<<<grid, kMlaThreads, kMlaSmemBytes, st>>>(a);
  if (int rc = check_launch("mla_decode_fwd")) return rc;
  if (splits > 1) {
    const int bh = batch * num_heads;
    mla_combine_kernel<<<(bh + 7) / 8, 256, 0, st>>>(a.part_o, a.part_lse, bh, splits, a.o, lse);
    return check_launch("mla_decode_fwd (combine)");
  }
  return FP8MOE_OK;
}

}  // extern "C"
