// Block-scaled FP8 GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang":
//   section "General Linear Layer"  - Y = XQ * WQ^T, one fp32 scale per 1x128
//     block of X and per 128x128 block of W (gemm_a8w8_blockscale);
//   section "Blockscale FP8 MoE Computation" - the g1u1 grouped GEMMs of
//     fmoe_fp8_blockscale_g1u1: GEMM1 over the gate+up rows of w1 with SiLU(gate)*up,
//     GEMM2 over w2, weighted by the routing weights.
//
// One kernel, three epilogues (Mode). Tile: 128 rows x 256 MMA columns x 128 K
// per pipeline stage (one scale block). Warp roles in a persistent CTA of three
// warpgroups; warpgroup 0 gives registers to the two epilogue warpgroups
// (setmaxnreg: 56 / 224 / 224 per thread, the launch's 3 x 168 in total):
//   warp 0      producer: TMA loads of the A and B tiles into a 4-stage
//               shared-memory ring;
//   warp 1      MMA issuer: per K block, 4 x tcgen05.mma (K=32 each) into one
//               of two 256-column TMEM buffers, fresh (not accumulated) so the
//               buffer holds that block's partial sums;
//   warp 2      scale loader: each K block's row and column scales into an
//               8-slot ring (cp.async);
//   warp 3      tile info: one tile ahead, the tile's coordinates, its MMA
//               shape and its rows' pair ids and routing weights into a 2-slot
//               shared ring for the MMA issuer and the epilogue;
//   warps 4..11 epilogue: tcgen05.ld the partials, multiply by
//               a_scale[row, kb] * b_scale[col/128, kb] (the down GEMM also by
//               the row's routing weight) and add into fp32 registers (the
//               per-128-K promotion), then the mode's output:
//               32-byte (whole-sector) stores of each thread's row, or for the
//               down GEMM's weighted bf16 rows a transpose through a small
//               shared buffer per warp so that each store writes 8 whole 64-byte
//               row segments.
// In the MoE modes the rows are the sorted token-expert slots: A is the
// slot-ordered activation matrix (gathered by moe_gather_kernel for GEMM1, the
// re-quantised intermediate for GEMM2), one expert per 128-row block.
// The MoE GEMMs read the weights either row-major ([E * rows, K]: a box is 128 rows
// x 128 bytes, the rows a full K apart) or tiled (each 128 x 128 block stored as 16
// KB of consecutive bytes, blocks ordered (row block, K block): a box is one block,
// read through a 3-D tensor map), chosen by the template flag TILED_B.
// A MoE tile that runs M=64 MMAs (its second 64 slots are padding) loads only its
// first 64 A rows (tmA64, a 64-row box), which spares shared-memory and L2 traffic.
// All waits are bounded; on expiry the CTA flags FP8MOE_DEVERR_TIMEOUT, sets a
// shared abort flag so the other roles stop, frees TMEM and exits.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace fp8moe {

enum GemmMode : int { kModeDense = 0, kModeMoeUp = 1, kModeMoeDown = 2 };

constexpr int kBM = 128;                      // rows (tokens / token-expert slots) per tile
constexpr int kBN = 256;                      // MMA columns per tile
constexpr int kBK = 128;                      // K per stage = one scale block
constexpr int kUmmaK = 32;                    // K of one tcgen05.mma kind::f8f6f4
constexpr int kStages = 4;
constexpr int kScaleSlots = 8;
constexpr int kEpiWarps = 8;
constexpr int kGemmThreads = 128 + 32 * kEpiWarps;   // warpgroup 0 + two epilogue warpgroups
constexpr uint32_t kRegsWg0 = 56;                     // producer / MMA / scale-loader / tile-info warpgroup
constexpr uint32_t kRegsEpilogue = 224;               // 56 + 2 x 224 == 3 x 168 (launch budget)
constexpr int kStageA = kBM * kBK;            // bytes
constexpr int kStageB = kBN * kBK;
constexpr int kStagingBytes = 32 * 64;        // per epilogue warp: 32 rows x 64 bytes
constexpr uint32_t kTmemCols = 512;           // two 256-column partial buffers
constexpr uint32_t kIdesc = umma_idesc_e4m3_f32(kBM, kBN);
constexpr uint32_t kIdescHalf = umma_idesc_e4m3_f32(kBM / 2, kBN);   // M=64: tiles with <= 64 occupied rows

struct GemmArgs {
  int M;                  // dense: rows of A; MoE: capacity (sorted slots)
  int N;                  // dense: columns of C; MoE up: I; MoE down: H
  int num_kb;             // ceil(K / 128)
  int n_tiles;            // tiles along N
  int group_m;            // M blocks visited together for each N tile (L2 reuse)
  const float* a_scale;   // dense: [M, num_kb]; MoE: slot-ordered [num_kb, M]
  const float* b_scale;   // [E][nb_per_expert][num_kb] (dense: E = 1)
  int nb_per_expert;      // 128-row scale blocks per expert matrix
  int nb_valid;           // dense: ceil(N/128) (clamp for the last tile)
  int c_vec;              // dense: C rows allow 32-byte stores (ldc % 16 == 0, C 32-byte aligned)
  __nv_bfloat16* C;       // dense output [M, ldc]
  int ldc;
  const int32_t* sorted_ids;
  const int32_t* sorted_expert_ids;
  const int32_t* num_valid_ids;
  const float* sorted_weights;
  int T, topk, E;
  int b_rows_per_expert;  // up: 2I; down: H
  uint8_t* a2;            // up output [M, I] (slot-ordered FP8 intermediate)
  float* s2;              // up output [I/128, M]
  __nv_bfloat16* ystage;  // down output [T*topk, H] (weighted rows by pair id, bf16)
  // down, expert parallelism: when set, pair p = q * y_src_pairs + lp is stored into
  // y_src_rows[q] + lp * H (rank q's return rows, possibly another GPU's memory) and
  // y_src_flags[q][lp] set to 1, instead of into ystage (device arrays of pointers)
  __nv_bfloat16* const* y_src_rows;
  uint8_t* const* y_src_flags;
  int y_src_pairs;
  // Failure-handling test hook (0 = off): with k + 1, the scale loader withholds
  // K block k's scales, so the epilogue's bounded wait for them runs out and the
  // CTA takes its abort path (device error word, TMEM freed, clean exit).
  int stall_kb1;
};

struct GemmSmem {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t sfull[kScaleSlots];
  uint64_t sempty[kScaleSlots];
  uint64_t xbar[2];                       // up: amax exchange between the two column halves
  uint64_t tifull[2];                     // tile-info ring (warp 3 -> MMA issuer + epilogue)
  uint64_t tiempty[2];
  uint32_t tmem_base;
  int abort;
  float sa[kScaleSlots][kBM];
  float sw[kScaleSlots][4];
  float amax_x[2][2][kBM];
  // tile-info ring: the tile's coordinates, whether it runs with M=64, and per
  // row the pair id and routing weight (MoE), prepared one tile ahead
  int ti_mb[2], ti_nt[2], ti_m64[2];
  int ti_pair[2][kBM];
  float ti_w[2][kBM];
};

constexpr size_t kGemmSmemBytes =
    1024 /*alignment slack*/ + kStages * (kStageA + kStageB) + kEpiWarps * kStagingBytes + sizeof(GemmSmem);

__device__ __forceinline__ void dense_tile_coords(int tile, int m_blocks, int n_tiles, int group_m, int& mb,
                                                  int& nt) {
  const int per_group = n_tiles * group_m;
  const int g = tile / per_group;
  const int first = g * group_m;
  const int gm = min(group_m, m_blocks - first);
  const int within = tile - g * per_group;
  nt = within / gm;
  mb = first + within % gm;
}

// MoE tile order: the row blocks of one expert inside an aligned window of
// kGroupBlocks blocks form a group, and a group's tiles run column tile by
// column tile, so that all of the expert's blocks read each weight tile at the
// same time (one DRAM read, the others hit L2). An expert's blocks are
// contiguous, so tiles [g0 * n_tiles, g1 * n_tiles) are exactly the group
// [g0, g1) and block tile / n_tiles lies inside it.
constexpr int kGroupBlocks = 16;
__device__ __forceinline__ void moe_tile_coords(const GemmArgs& a, int tile, int m_blocks, int& mb, int& nt) {
  const int n = a.n_tiles;
  const int b = tile / n;
  const int w = b & ~(kGroupBlocks - 1);
  const int eb = a.sorted_expert_ids[b];
  int g0 = b, g1 = b + 1;
#pragma unroll
  for (int i = 0; i < kGroupBlocks; ++i) {
    const int j = w + i;
    if (j < m_blocks && a.sorted_expert_ids[j] == eb) {
      g0 = min(g0, j);
      g1 = max(g1, j + 1);
    }
  }
  const int gs = g1 - g0;
  const int local = tile - g0 * n;
  nt = local / gs;
  mb = g0 + local % gs;
}

// The gate/up GEMM (56 K blocks per tile, 1.8 MB weight tiles) takes the
// expert-grouped order; the dense and down GEMMs visit group_m consecutive row
// blocks per column tile, which measured faster for the down GEMM's short tiles.
template <int MODE>
__device__ __forceinline__ void tile_coords(const GemmArgs& a, int tile, int m_blocks, int& mb, int& nt) {
  if (MODE == kModeMoeUp)
    moe_tile_coords(a, tile, m_blocks, mb, nt);
  else
    dense_tile_coords(tile, m_blocks, a.n_tiles, a.group_m, mb, nt);
}

__device__ __forceinline__ int moe_m_blocks(const GemmArgs& a) {
  int nv = *a.num_valid_ids;
  if (nv < 0 || nv > a.M || (nv % kBM) != 0) {
    raise_device_error(FP8MOE_DEVERR_NUM_VALID);
    nv = max(0, min(nv, a.M));
  }
  return nv / kBM;
}

__device__ __forceinline__ int moe_expert(const GemmArgs& a, int mb) {
  int e = a.sorted_expert_ids[mb];
  if (e < 0 || e >= a.E) {
    raise_device_error(FP8MOE_DEVERR_EXPERT_ID);
    e = 0;
  }
  return e;
}

__device__ __forceinline__ void abort_all(GemmSmem* s) {
  if (!s->abort) raise_device_error(FP8MOE_DEVERR_TIMEOUT);
  s->abort = 1;
}

// Writes a warp's 32 rows x 64 bytes (row = lane, data d) to global memory with
// coalesced stores: each lane puts its row into the warp's shared staging buffer
// (16-byte chunk c of row r at chunk c ^ ((r >> 1) & 3): no bank conflicts), then
// each of four store instructions writes 8 whole 64-byte row segments. In store
// i a lane writes 16 bytes of row store_rows_row(i, lane); row_addr(i) gives that
// row segment's destination, or nullptr to skip it.
__device__ __forceinline__ int store_rows_row(int i, int lane) { return i * 8 + (lane >> 2); }
template <typename RowAddr>
__device__ __forceinline__ void store_rows_64B(uint8_t* staging, int lane, const uint4 (&d)[4], RowAddr row_addr) {
  uint8_t* mine = staging + lane * 64;
  const int swz = (lane >> 1) & 3;
#pragma unroll
  for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(mine + ((c ^ swz) << 4)) = d[c];
  __syncwarp();
  const int c = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = store_rows_row(i, lane);
    const uint4 v = *reinterpret_cast<const uint4*>(staging + r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
    uint8_t* dst = row_addr(i);
    if (dst) *reinterpret_cast<uint4*>(dst + c * 16) = v;
  }
  __syncwarp();
}

// The epilogue warpgroups: promotion of each K block's partial sums into fp32
// registers, then the mode's output through the per-warp staging buffer.
// ROUTED (down GEMM, expert parallelism): every pair row goes to its origin's return
// rows (args.y_src_*) instead of ystage.
template <int MODE, bool ROUTED = false>
__device__ __forceinline__ void epilogue_role(const GemmArgs& args, GemmSmem* s, uint8_t* staging,
                                              uint32_t tmem_base, int warp, int lane, int m_blocks,
                                              int total_tiles, int num_kb, int P) {
  volatile int* abort_flag = &s->abort;
  // ------------------------------------------------------------ epilogue
  const int ew = warp - 4;
  const int half = ew >> 2;                  // which 128 of the 256 MMA columns (up: which 64 of I)
  const int quarter = warp & 3;              // TMEM lanes this warp may access
  const int row = quarter * 32 + lane;       // tile row = TMEM lane
  const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
  // TMEM columns of this thread's two 64-column segments
  const int col0 = (MODE == kModeMoeUp) ? half * 64 : half * 128;
  const int col1 = (MODE == kModeMoeUp) ? kBN / 2 + half * 64 : half * 128 + 64;
  int buf = 0, sslot = 0, tislot = 0;
  uint32_t tphase = 0, scphase = 0, tiphase = 0;
  bool ok = true;
  for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
    // The tile's coordinates and rows. The dense and down epilogues take them
    // from the tile-info ring (shared memory): the slot is held until the
    // tile's output is written, and values needed only there are read there, so
    // that they take no registers during the promotion loop. The gate/up
    // epilogue loads its own copy from global memory at the tile start and keeps
    // it in registers, which measured about 4% faster for that GEMM.
    if (!mbar_wait(&s->tifull[tislot], tiphase, abort_flag)) { ok = false; break; }
    // An M=64 tile keeps its row r in TMEM lane (r % 16) + 32 * (r / 16): lanes
    // 0..15 of each warp hold rows 16*quarter + lane, lanes 16..31 hold none.
    auto lane_row = [&](bool m64) { return m64 ? (lane < 16 ? quarter * 16 + lane : -1) : row; };
    int up_mb = 0, up_nt = 0, up_trow = -1, up_pair = P;
    if (MODE == kModeMoeUp) {
      tile_coords<MODE>(args, tile, m_blocks, up_mb, up_nt);
      const int id_half = args.sorted_ids[up_mb * kBM + kBM / 2];
      up_trow = lane_row(id_half < 0 || id_half >= P);
      if (up_trow >= 0) up_pair = args.sorted_ids[up_mb * kBM + up_trow];
    }
    auto tile_row = [&]() { return MODE == kModeMoeUp ? up_trow : lane_row(s->ti_m64[tislot] != 0); };
    const int sa_row = max(tile_row(), 0);
    float acc[128];
#pragma unroll
    for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
    // a warp whose 32 rows are all padding skips the promotion (its outputs are never stored)
    bool warp_active = true;
    if (MODE != kModeDense) {
      const int pr = MODE == kModeMoeUp ? up_pair : (tile_row() >= 0 ? s->ti_pair[tislot][sa_row] : P);
      warp_active = __any_sync(0xffffffffu, pr >= 0 && pr < P);
    }

    for (int kb = 0; kb < num_kb; ++kb) {
      if (!mbar_wait(&s->sfull[sslot], scphase, abort_flag)) { ok = false; break; }
      const float sa = s->sa[sslot][sa_row];
      const float swa = s->sw[sslot][0], swb = s->sw[sslot][1];
      __syncwarp();
      if (lane == 0) mbar_arrive(&s->sempty[sslot]);
      if (++sslot == kScaleSlots) { sslot = 0; scphase ^= 1u; }
      float f0, f1;
      if (MODE == kModeMoeUp) {
        f0 = sa * swa;
        f1 = sa * swb;
      } else if (MODE == kModeMoeDown) {
        // the routing weight rides on every block's scale (read from the ring:
        // no register held across the loop)
        f0 = f1 = sa * (half ? swb : swa) * s->ti_w[tislot][sa_row];
      } else {
        f0 = f1 = sa * (half ? swb : swa);
      }

      if (!mbar_wait(&s->tfull[buf], tphase, abort_flag)) { ok = false; break; }
      tc_fence_after();
      if (!warp_active) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s->tempty[buf]);
        if (++buf == 2) { buf = 0; tphase ^= 1u; }
        continue;
      }
      const uint32_t tb = lane_base + buf * kBN;
      float v[2][32];
      // four 32-column chunks; the load of chunk c+1 overlaps the FMAs of chunk c
      tmem_ld_32x32b_x32(tb + col0, v[0]);
      tmem_wait_ld();
      reg_fence_32(v[0]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c + 1 < 4) tmem_ld_32x32b_x32(tb + ((c + 1) < 2 ? col0 : col1) + ((c + 1) & 1) * 32, v[(c + 1) & 1]);
        const float f = (c < 2) ? f0 : f1;
        const float2 ff = make_float2(f, f);
        // packed fp32 FMA (two lanes per instruction, each rounded to nearest)
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 r = __ffma2_rn(ff, make_float2(v[c & 1][j], v[c & 1][j + 1]),
                                      make_float2(acc[c * 32 + j], acc[c * 32 + j + 1]));
          acc[c * 32 + j] = r.x;
          acc[c * 32 + j + 1] = r.y;
        }
        if (c + 1 < 4) {
          tmem_wait_ld();
          reg_fence_32(v[(c + 1) & 1]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s->tempty[buf]);
      if (++buf == 2) { buf = 0; tphase ^= 1u; }
    }
    if (!ok) break;

    const int mb = MODE == kModeMoeUp ? up_mb : s->ti_mb[tislot];
    const int nt = MODE == kModeMoeUp ? up_nt : s->ti_nt[tislot];
    const int trow = tile_row();
    const bool has_row = trow >= 0;
    const int slot = mb * kBM + (has_row ? trow : 0);
    int pair = P;
    if (MODE != kModeDense && has_row) pair = MODE == kModeMoeUp ? up_pair : s->ti_pair[tislot][trow];
    // Outputs. Dense and gate/up: each thread writes its own row with 32-byte
    // stores (whole sectors) straight from registers.
    if (MODE == kModeDense) {
      const int grow = mb * kBM + row;
      const int x0 = nt * kBN + half * 128;
      if (grow < args.M) {
        __nv_bfloat16* crow = args.C + static_cast<size_t>(grow) * args.ldc;
        const bool vec = args.c_vec != 0 && x0 + 128 <= args.N;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {      // 8 chunks of 16 bf16 columns
          uint32_t w[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const __nv_bfloat162 pk = __floats2bfloat162_rn(acc[ch * 16 + 2 * u], acc[ch * 16 + 2 * u + 1]);
            w[u] = *reinterpret_cast<const uint32_t*>(&pk);
          }
          const int x = x0 + ch * 16;
          if (vec) {
            st_global_v8(crow + x, w);
          } else {                            // ragged edge or unaligned C: element stores
            const __nv_bfloat16* vals = reinterpret_cast<const __nv_bfloat16*>(w);
#pragma unroll
            for (int u = 0; u < 16; ++u)
              if (x + u < args.N) crow[x + u] = vals[u];
          }
        }
      }
    } else if (MODE == kModeMoeUp) {
      // h = silu(gate) * up for this thread's 64 intermediate columns
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const float g = acc[j];
        const float h = __fdividef(g, 1.0f + __expf(-g)) * acc[64 + j];
        acc[j] = h;
        amax = fmaxf(amax, fabsf(h));
      }
      // the 128-wide requantisation group spans both column halves of the row
      // the ring slot alternates per tile and its phase every two tiles: the
      // exchange buffer and its phase follow the same pattern
      const int xb = tislot;
      s->amax_x[xb][half][row] = amax;
      __syncwarp();
      if (lane == 0) mbar_arrive(&s->xbar[xb]);
      if (!mbar_wait(&s->xbar[xb], tiphase, abort_flag)) { ok = false; break; }
      amax = fmaxf(amax, s->amax_x[xb][half ^ 1][row]);
      const float scale = __fdiv_rn(amax, 448.0f);
      const float inv = scale != 0.0f ? __frcp_rn(scale) : 0.0f;
      if (pair >= 0 && pair < P) {
        uint8_t* dst = args.a2 + static_cast<size_t>(slot) * args.N + nt * 128 + half * 64;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {      // 2 x 32 codes
          uint32_t w[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = ch * 32 + 4 * u;
            w[u] = static_cast<uint32_t>(cvt_e4m3x2(acc[j] * inv, acc[j + 1] * inv)) |
                   (static_cast<uint32_t>(cvt_e4m3x2(acc[j + 2] * inv, acc[j + 3] * inv)) << 16);
          }
          st_global_v8(dst + ch * 32, w);
        }
      }
      if (half == 0 && has_row) args.s2[static_cast<size_t>(nt) * args.M + slot] = scale;
    } else {
      // weighted rows (the weight is already in the sums), 256 bytes of bf16 per
      // row: a transpose through the warp's staging buffer lets each store
      // instruction write 8 whole 64-byte row segments
      const bool valid = pair >= 0 && pair < P;
      if (!valid && pair != P) raise_device_error(FP8MOE_DEVERR_PAIR_ID);
      const int x0 = nt * kBN + half * 128;
      if (x0 < args.N) {
        const int H = args.N;
        __nv_bfloat16* y = args.ystage;
        uint8_t* my_staging = staging + ew * kStagingBytes;
        // destinations of the four rows this lane stores (null for padding rows)
        uint8_t* dst[4];
        int prs[4];
        if constexpr (!ROUTED) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int pr = __shfl_sync(0xffffffffu, pair, store_rows_row(i, lane));
            dst[i] = (pr >= 0 && pr < P) ? reinterpret_cast<uint8_t*>(y + static_cast<size_t>(pr) * H + x0) : nullptr;
          }
        } else {                              // each row into its origin's return rows
          // (pair ids held, the address made per store: fewer live registers)
#pragma unroll
          for (int i = 0; i < 4; ++i) prs[i] = __shfl_sync(0xffffffffu, pair, store_rows_row(i, lane));
          if (valid && nt == 0 && half == 0) {   // one thread per row sets the pair's flag
            const int q = pair / args.y_src_pairs;
            uint8_t* flags = reinterpret_cast<uint8_t*>(
                __ldg(reinterpret_cast<const unsigned long long*>(args.y_src_flags) + q));
            flags[pair - q * args.y_src_pairs] = 1;
          }
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {      // 4 chunks of 32 bf16 columns
          uint4 d[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int j = ch * 32 + u * 8 + 2 * q;
              const __nv_bfloat162 pk = __floats2bfloat162_rn(acc[j], acc[j + 1]);
              w[q] = *reinterpret_cast<const uint32_t*>(&pk);
            }
            d[u] = make_uint4(w[0], w[1], w[2], w[3]);
          }
          store_rows_64B(my_staging, lane, d, [&](int i) -> uint8_t* {
            if constexpr (!ROUTED) {
              return dst[i] ? dst[i] + ch * 64 : nullptr;
            } else {
              const int pr = prs[i];
              if (pr < 0 || pr >= P) return nullptr;
              const int q = pr / args.y_src_pairs;
              __nv_bfloat16* base = reinterpret_cast<__nv_bfloat16*>(
                  __ldg(reinterpret_cast<const unsigned long long*>(args.y_src_rows) + q));
              return reinterpret_cast<uint8_t*>(base + static_cast<size_t>(pr - q * args.y_src_pairs) * H + x0) +
                     ch * 64;
            }
          });
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s->tiempty[tislot]);
    if (++tislot == 2) { tislot = 0; tiphase ^= 1u; }
  }
  if (!ok) abort_all(s);
}

template <int MODE, bool TILED_B = false, bool ROUTED = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
blockscale_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmA64, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* tiles = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* tiles_a = tiles;                                  // kStages x 16 KB
  uint8_t* tiles_b = tiles + kStages * kStageA;              // kStages x 32 KB
  uint8_t* staging = tiles + kStages * (kStageA + kStageB);  // kEpiWarps x 2 KB
  GemmSmem* s = reinterpret_cast<GemmSmem*>(staging + kEpiWarps * kStagingBytes);
  volatile int* abort_flag = &s->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s->full[i], 1);
      mbar_init(&s->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s->tfull[i], 1);
      mbar_init(&s->tempty[i], kEpiWarps);
      mbar_init(&s->xbar[i], kEpiWarps);
      mbar_init(&s->tifull[i], 32);
      mbar_init(&s->tiempty[i], kEpiWarps + 1);   // the epilogue warps and the MMA issuer
    }
    for (int i = 0; i < kScaleSlots; ++i) {
      mbar_init(&s->sfull[i], 32);
      mbar_init(&s->sempty[i], kEpiWarps);
    }
    s->abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmA);
    if (MODE != kModeDense) prefetch_tensormap(&tmA64);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&s->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s->tmem_base;

  const int m_blocks = (MODE == kModeDense) ? (args.M + kBM - 1) / kBM : moe_m_blocks(args);
  const int total_tiles = m_blocks * args.n_tiles;
  const int num_kb = args.num_kb;
  const int P = args.T * args.topk;

  if (warp >= 4) {
    warpgroup_reg_alloc<kRegsEpilogue>();
    epilogue_role<MODE, ROUTED>(args, s, staging, tmem_base, warp, lane, m_blocks, total_tiles, num_kb, P);
  } else {
    warpgroup_reg_dealloc<kRegsWg0>();     // one instruction for all four warps of warpgroup 0
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t sphase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        int mb, nt;
        tile_coords<MODE>(args, tile, m_blocks, mb, nt);
        const int e = (MODE == kModeDense) ? 0 : moe_expert(args, mb);
        // a MoE tile whose slot kBM/2 is padding runs M=64 MMAs: load its first 64 A rows only
        bool a64 = false;
        if (MODE != kModeDense) {
          const int id_half = args.sorted_ids[mb * kBM + kBM / 2];
          a64 = id_half < 0 || id_half >= P;
        }
        const uint32_t a_bytes = a64 ? kStageA / 2 : kStageA;
        const int brow0 = (MODE == kModeMoeUp) ? e * args.b_rows_per_expert + nt * 128
                                               : e * args.b_rows_per_expert + nt * kBN;
        const int brow1 = (MODE == kModeMoeUp) ? brow0 + args.N : brow0 + 128;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&s->empty[stage], sphase ^ 1u, abort_flag)) { ok = false; break; }
          if (lane == 0) {
            uint8_t* sa_tile = tiles_a + stage * kStageA;
            uint8_t* sb_tile = tiles_b + stage * kStageB;
            mbar_arrive_expect_tx(&s->full[stage], a_bytes + kStageB);
            tma_load_2d(sa_tile, a64 ? &tmA64 : &tmA, &s->full[stage], kb * kBK, mb * kBM);
            if constexpr (TILED_B) {
              // block (row block r, K block kb) is box (0, 0, r * num_kb + kb)
              tma_load_3d(sb_tile, &tmB, &s->full[stage], 0, 0, (brow0 / 128) * num_kb + kb);
              tma_load_3d(sb_tile + kStageB / 2, &tmB, &s->full[stage], 0, 0, (brow1 / 128) * num_kb + kb);
            } else {
              tma_load_2d(sb_tile, &tmB, &s->full[stage], kb * kBK, brow0);
              tma_load_2d(sb_tile + kStageB / 2, &tmB, &s->full[stage], kb * kBK, brow1);
            }
          }
          __syncwarp();
          if (++stage == kStages) { stage = 0; sphase ^= 1u; }
        }
      }
      if (!ok) {
        abort_all(s);
        // let copies already in flight land before the CTA's shared memory goes away
        const unsigned long long t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 10000000ull) {}
      }
    } else if (warp == 2) {
      // ------------------------------------------------------------ scale loader
      int sslot = 0;
      uint32_t scphase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        int mb, nt;
        tile_coords<MODE>(args, tile, m_blocks, mb, nt);
        const int e = (MODE == kModeDense) ? 0 : moe_expert(args, mb);
        // this lane's four rows of the tile: 4*lane .. 4*lane+3
        const float* sa_src[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = mb * kBM + 4 * lane + i;
          sa_src[i] = (MODE == kModeDense) ? args.a_scale + static_cast<size_t>(min(r, args.M - 1)) * num_kb
                                           : args.a_scale + r;   // + kb * M
        }
        const size_t kstride = (MODE == kModeDense) ? 1 : static_cast<size_t>(args.M);
        int nb0, nb1;
        if (MODE == kModeMoeUp) {
          nb0 = nt;
          nb1 = args.N / 128 + nt;
        } else {
          nb0 = min(2 * nt, args.nb_valid - 1);
          nb1 = min(2 * nt + 1, args.nb_valid - 1);
        }
        const float* sw_src0 = args.b_scale + (static_cast<size_t>(e) * args.nb_per_expert + nb0) * num_kb;
        const float* sw_src1 = args.b_scale + (static_cast<size_t>(e) * args.nb_per_expert + nb1) * num_kb;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&s->sempty[sslot], scphase ^ 1u, abort_flag)) { ok = false; break; }
          if (kb + 1 != args.stall_kb1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) cp_async_4(&s->sa[sslot][4 * lane + i], sa_src[i] + kb * kstride);
            if (lane == 0) {
              cp_async_4(&s->sw[sslot][0], sw_src0 + kb);
              cp_async_4(&s->sw[sslot][1], sw_src1 + kb);
            }
            cp_async_mbar_arrive(&s->sfull[sslot]);
          }
          if (++sslot == kScaleSlots) { sslot = 0; scphase ^= 1u; }
        }
      }
      if (!ok) abort_all(s);
      asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        int stage = 0, buf = 0, tislot = 0;
        uint32_t sphase = 0, tphase = 0, tiphase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
          if (!mbar_wait(&s->tifull[tislot], tiphase, abort_flag)) { ok = false; break; }
          const uint32_t idesc = s->ti_m64[tislot] ? kIdescHalf : kIdesc;
          mbar_arrive(&s->tiempty[tislot]);
          if (++tislot == 2) { tislot = 0; tiphase ^= 1u; }
          for (int kb = 0; kb < num_kb; ++kb) {
            if (!mbar_wait(&s->full[stage], sphase, abort_flag)) { ok = false; break; }
            if (!mbar_wait(&s->tempty[buf], tphase ^ 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(tiles_a + stage * kStageA);
            const uint32_t b_addr = smem_u32(tiles_b + stage * kStageB);
            const uint32_t d_tmem = tmem_base + buf * kBN;
#pragma unroll
            for (int k = 0; k < kBK / kUmmaK; ++k)
              umma_f8(d_tmem, umma_desc_sw128(a_addr + k * kUmmaK), umma_desc_sw128(b_addr + k * kUmmaK), idesc,
                      k > 0 ? 1u : 0u);
            umma_commit(&s->empty[stage]);
            umma_commit(&s->tfull[buf]);
            if (++stage == kStages) { stage = 0; sphase ^= 1u; }
            if (++buf == 2) { buf = 0; tphase ^= 1u; }
          }
        }
        if (!ok) abort_all(s);
      }
      __syncwarp();
    } else {
      // ------------------------------------------------------------ tile info
      // One tile ahead of the epilogue: the coordinates (for the gate/up GEMM a
      // scan of the block-expert list), the M=64 decision and the rows' pair ids
      // and routing weights, so that neither the MMA issuer nor the epilogue
      // waits on dependent global loads at a tile boundary.
      int tislot = 0;
      uint32_t tiphase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
        int mb, nt;
        tile_coords<MODE>(args, tile, m_blocks, mb, nt);
        int ids[4] = {P, P, P, P};
        float wts[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (MODE != kModeDense) {
#pragma unroll
          for (int i = 0; i < 4; ++i) ids[i] = args.sorted_ids[mb * kBM + 4 * lane + i];
          if (MODE == kModeMoeDown) {
#pragma unroll
            for (int i = 0; i < 4; ++i) wts[i] = args.sorted_weights[mb * kBM + 4 * lane + i];
          }
        }
        // A MoE tile whose second half holds only padding slots (an expert's last
        // block with at most 64 pairs) runs its MMAs with M=64. The sort puts an
        // expert's pairs before its padding, so slot kBM/2 (lane 16's first row) decides.
        const int id_half = __shfl_sync(0xffffffffu, ids[0], kBM / 8);
        const int m64 = (MODE != kModeDense) && (id_half < 0 || id_half >= P);
        if (!mbar_wait_idle(&s->tiempty[tislot], tiphase ^ 1u, abort_flag)) { ok = false; break; }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          s->ti_pair[tislot][4 * lane + i] = ids[i];
          s->ti_w[tislot][4 * lane + i] = wts[i];
        }
        if (lane == 0) {
          s->ti_mb[tislot] = mb;
          s->ti_nt[tislot] = nt;
          s->ti_m64[tislot] = m64;
        }
        mbar_arrive(&s->tifull[tislot]);
        if (++tislot == 2) { tislot = 0; tiphase ^= 1u; }
      }
      if (!ok) abort_all(s);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace fp8moe
