/*
 * fp8moe.h - C ABI of the B200 (sm_100a) FP8 block-scaled biased MoE layer.
 *
 * The operations, their argument order and their tensor layouts follow
 * "Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang"
 * (rocm.blogs.amd.com), section "Complete MoE Implementation" (Top-K routing,
 * MoE Sorting, Blockscale FP8 MoE Computation) and section "General Linear
 * Layer" (FP8 blockscale GEMM). FP8 is OCP E4M3 "fn" (largest finite 448), not
 * the MI300X "fnuz" variant. The tensor- and expert-parallel entry points at the
 * end follow the same page's TP8 run and custom all-reduce ("Performance
 * Reproduction for AITER-Optimized in SGLang", "Other Operators") and asm_moe's
 * expert_mask. The MLA decode entry point at the very end follows the same page's
 * section "Attention Mechanisms" ("MLA For Decode").
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller; the library never
 *     allocates, frees or keeps them. Scratch memory is passed in as
 *     `workspace`, sized by the matching *_workspace query. The multi-GPU entry
 *     points take host arrays with one device pointer per rank, each as this GPU
 *     addresses that rank's memory (peer memory over NVLink, or local); only the
 *     return_rows / return_flags arrays of fused_moe_fp8_blockscale_g1u1_multi are
 *     device arrays, because its down GEMM reads them.
 *   - Matrices are row-major; `ld*` arguments are row strides in elements.
 *   - FP8 tensors are bytes (uint8_t) holding E4M3fn codes; bf16 tensors are
 *     uint16_t holding bfloat16 bit patterns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Every call
 *     only enqueues work on it and returns without synchronising, so a chain of
 *     calls can be captured in a CUDA graph. No value travels back to the host:
 *     `num_valid_ids` stays on the device and the kernels read it there.
 *   - Return value: FP8MOE_OK, or an error code with nothing launched (argument
 *     errors) or a launch error (FP8MOE_ECUDA). fp8moe_last_error() returns a
 *     message for the calling thread's last failure.
 *   - Faults the kernels detect on the device (an expert id out of range, a
 *     bounded wait that expired) set a device error word instead of trapping;
 *     fp8moe_device_status() reports and clears it.
 */
#ifndef FP8MOE_H
#define FP8MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum fp8moe_status {
  FP8MOE_OK = 0,
  FP8MOE_EINVAL = 1,        /* bad pointer, size, stride or argument combination */
  FP8MOE_EUNSUPPORTED = 2,  /* a valid request this library does not implement   */
  FP8MOE_EWORKSPACE = 3,    /* workspace missing or smaller than the query       */
  FP8MOE_ECUDA = 4,         /* CUDA runtime/driver error (launch, device query)  */
  FP8MOE_EDEVICE = 5        /* device-detected fault (fp8moe_device_status only) */
};

/* Device error word bits reported by fp8moe_device_status(). */
enum fp8moe_device_error {
  FP8MOE_DEVERR_TIMEOUT = 1u,     /* a bounded wait inside a kernel expired       */
  FP8MOE_DEVERR_EXPERT_ID = 2u,   /* an expert id outside [0, E) was met          */
  FP8MOE_DEVERR_PAIR_ID = 4u,     /* a sorted pair id outside [0, T*topk] was met */
  FP8MOE_DEVERR_NUM_VALID = 8u,   /* num_valid_ids above capacity or not a multiple of block_m */
  FP8MOE_DEVERR_BLOCK_ORDER = 16u, /* sorted_expert_ids decreases somewhere: not a moe_align_sort result */
  FP8MOE_DEVERR_PAGE = 32u         /* MLA decode: a page-table entry outside its range (see mla_decode_fwd) */
};

/* Message describing the calling thread's most recent failure ("" if none). */
const char* fp8moe_last_error(void);

/* Synchronises `stream`, then returns and clears the device error word of the
 * current device (0 = no fault seen). Returns -1 with a message if the
 * synchronisation itself fails. */
int fp8moe_device_status(void* stream);

/* Measurement hook (not part of the pages' API). While enabled for the calling
 * thread, each fused_moe_fp8_blockscale_g1u1 call records CUDA events on its
 * stream before the slot-order gather, after it, after the gate/up GEMM, after
 * the down GEMM and after the combine. fp8moe_timing_last() waits for the last
 * of those events and writes the four kernel durations of the most recent call
 * in milliseconds (ms[0] gather, ms[1] gate/up GEMM, ms[2] down GEMM,
 * ms[3] combine; `ms` holds 4 floats). Returns FP8MOE_OK, FP8MOE_EINVAL (null
 * pointer, timing never enabled) or FP8MOE_ECUDA. Events are created on first
 * use on the current device. */
int fp8moe_timing_enable(int on);
int fp8moe_timing_last(float* ms);

/* Failure-handling test hook (not part of the pages' API): fp8_blockscale_gemm
 * on the same arguments, except that in every CTA's tiles the scales of K block
 * stall_kb are withheld. The epilogue's bounded wait for them runs out (about
 * 2 s), the CTA sets FP8MOE_DEVERR_TIMEOUT, stops its other warps, frees its
 * tensor memory and exits; C is left unspecified. fp8moe_device_status() then
 * reports the bit and the context stays usable. Nothing faults or hangs. */
int fp8moe_selftest_gemm_stall(const uint8_t* A, const uint8_t* B,
                               const float* a_scale, const float* b_scale,
                               uint16_t* C, int ldc, int M, int N, int K,
                               int stall_kb, void* stream);

/* Block size of the M (token-expert pair) dimension that the fused MoE kernels
 * tile by; moe_align_sort must be called with block_m equal to this. */
int fp8moe_moe_block_m(void);

/*
 * S1 - biased grouped top-k routing.  (Top-K routing: biased_grouped_topk(
 *      gating_output, correction_bias, topk_weights, topk_ids,
 *      num_expert_group, topk_group, need_renorm, routed_scaling_factor).)
 *
 * gating_output   fp32 [T, E], row stride ld_in >= E
 * correction_bias fp32 [E]
 * topk_weights    fp32 [T, topk], row stride ld_out >= topk (gap columns are
 *                 not written; the pages allocate these outputs strided)
 * topk_ids        int32 [T, topk], same row stride ld_out
 * Per token: s = sigmoid(logit), b = s + bias. Group score = sum of the two
 * largest b of the group's E/num_expert_group experts. The topk_group best
 * groups are kept (ties: lower group index), then the topk best experts by b
 * among them (ties: lower expert index), written in that rank order. Weights
 * are the unbiased s, divided by their sum if need_renorm, then multiplied by
 * routed_scaling_factor. sigmoid uses a fixed fp32 operation sequence so the
 * ids are reproducible bit for bit.
 * Limits: 1 <= E <= 512, E % num_expert_group == 0, num_expert_group <= 32,
 * 1 <= topk_group <= num_expert_group, 1 <= topk <= 32,
 * topk <= topk_group * (E / num_expert_group). T == 0 is a no-op.
 */
int moe_biased_grouped_topk(const float* gating_output, int ld_in,
                            const float* correction_bias,
                            float* topk_weights, int32_t* topk_ids, int ld_out,
                            int T, int E, int topk, int num_expert_group,
                            int topk_group, int need_renorm,
                            float routed_scaling_factor, void* stream);

/*
 * S1 with bf16 router logits (the page's routing test runs over a `dtype`).
 * gating_output is bf16 [T, E] (uint16_t bit patterns), row stride ld_in >= E;
 * everything else as moe_biased_grouped_topk. A bf16 logit widens to fp32
 * exactly, so the result equals moe_biased_grouped_topk on the widened logits
 * bit for bit.
 */
int moe_biased_grouped_topk_bf16(const uint16_t* gating_output, int ld_in,
                                 const float* correction_bias,
                                 float* topk_weights, int32_t* topk_ids,
                                 int ld_out, int T, int E, int topk,
                                 int num_expert_group, int topk_group,
                                 int need_renorm, float routed_scaling_factor,
                                 void* stream);

/*
 * S2 - MoE align/sort.  (MoE Sorting: moe_sorting(topk_ids, topk_weights, E,
 *      model_dim, dtype) -> sorted_token_ids, sorted_weight_buf,
 *      sorted_expert_ids, num_valid_ids.)
 *
 * topk_ids int32 [T, topk] and topk_weights fp32 [T, topk], row stride ld.
 * Pair (t, k) is named by its flat id p = t*topk + k. Experts are laid out in
 * ascending id order, each expert's pairs in ascending p, each segment padded
 * to a multiple of block_m with id T*topk and weight 0; experts without pairs
 * get no block.
 * Outputs (device): sorted_ids int32 [capacity], sorted_weights fp32
 * [capacity], sorted_expert_ids int32 [capacity / block_m] (one expert per
 * block), num_valid_ids int32 [1] (= padded length). Entries past the padded
 * length are left untouched. capacity must be >= moe_align_sort_capacity().
 * An id outside [0, E) is dropped and flagged (FP8MOE_DEVERR_EXPERT_ID).
 * Limits: 1 <= E <= 1024, 1 <= block_m <= 1024, T*topk < 2^31.
 */
size_t moe_align_sort_capacity(int T, int topk, int E, int block_m);
size_t moe_align_sort_workspace(int T, int topk, int E, int block_m);
int moe_align_sort(const int32_t* topk_ids, const float* topk_weights, int ld,
                   int T, int topk, int E, int block_m,
                   int32_t* sorted_ids, float* sorted_weights,
                   int32_t* sorted_expert_ids, int32_t* num_valid_ids,
                   size_t capacity, void* workspace, size_t workspace_bytes,
                   void* stream);

/*
 * S2 with an expert mask: the expert_mask argument of the page's asm_moe call
 * (section "MoE Sorting"), the hook for expert parallelism. expert_mask is a
 * DEVICE int32 [E]; pairs routed to an expert e with expert_mask[e] == 0 are
 * dropped (no slot, no flag), so the sorted list holds only this GPU's experts.
 * NULL keeps every expert (= moe_align_sort). Everything else as
 * moe_align_sort, including the capacity and workspace queries.
 * fused_moe_fp8_blockscale_g1u1 on the result gives the sum over the kept
 * experts only: the partial output an expert-parallel rank contributes.
 */
int moe_align_sort_masked(const int32_t* topk_ids, const float* topk_weights,
                          int ld, int T, int topk, int E, int block_m,
                          const int32_t* expert_mask,
                          int32_t* sorted_ids, float* sorted_weights,
                          int32_t* sorted_expert_ids, int32_t* num_valid_ids,
                          size_t capacity, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * S3 - dynamic per-token-group FP8 quantisation (1 x group).
 *      (dynamic_per_token_scaled_fp8_quant on hidden states viewed as
 *      [M*H/128, 128]; per_token_group_quant_fp8(x, 128, column_major_scales).)
 *
 * x      bf16 [M, K], row stride ld_x (elements)
 * q      fp8 [M, K], row stride K
 * scales fp32 [M, ceil(K/group)] if scale_layout == FP8MOE_SCALE_ROW_MAJOR, or
 *        [ceil(K/group), M] if FP8MOE_SCALE_COL_MAJOR (the transposed layout the
 *        fused MoE call takes).
 * scale = amax / 448 (fp32), q = E4M3fn(x / scale) rounded to nearest even and
 * saturated; an all-zero group gives scale 0 and codes 0.
 * Limits: group == 128; K % 8 == 0; ld_x % 8 == 0; x 16-byte aligned.
 */
enum { FP8MOE_SCALE_ROW_MAJOR = 0, FP8MOE_SCALE_COL_MAJOR = 1 };
int fp8_per_token_group_quant(const uint16_t* x, int ld_x, int M, int K, int group,
                              uint8_t* q, float* scales, int scale_layout,
                              void* stream);

/*
 * Weight preparation - FP8 quantisation in 128 x 128 blocks (the recipe behind
 * the "*_weight_scale_inv" tensors of the pages' MoE and linear layers).
 *
 * w      fp32 [N, K], row stride ld_w
 * q      fp8 [N, K], row stride K
 * scales fp32 [ceil(N/128), ceil(K/128)]; scale = amax / 448 over the block,
 *        q = E4M3fn(w / scale); dequantised weight = q * scale.
 * Limits: block == 128.
 */
int fp8_per_block_quant(const float* w, int ld_w, int N, int K, int block,
                        uint8_t* q, float* scales, void* stream);

/*
 * Weight preparation - re-pack into the tiled layout. (The B200 counterpart of the
 * pages' offline weight pre-shuffle: the MoE section passes w1 and w2 through
 * shuffle_weight(w, (16, 16)) before asm_moe, and the linear section notes a
 * shuffled-weight variant, both in "Blockscale FP8 MoE Computation" and "General
 * Linear Layer". The pages print that layout only for AMD's kernels; this one is
 * this library's own.)
 *
 * w    fp8 [E, N, K] row-major (E expert matrices), 16-byte aligned
 * out  fp8 [E, N/128, K/128, 128, 128]: block (e, nb, kb) holds rows
 *      nb*128 .. nb*128+127 and columns kb*128 .. kb*128+127 of matrix e,
 *      row-major inside the block, so each 128 x 128 block is 16 KB of
 *      consecutive bytes (16-byte aligned, not overlapping w). The block scales
 *      are unchanged ([E, N/128, K/128] in either layout).
 * Limits: N and K positive multiples of 128, E <= 65535.
 */
int fp8_tile_weights(const uint8_t* w, int E, int N, int K, uint8_t* out, void* stream);

/*
 * S0 - FP8 block-scale GEMM.  (General Linear Layer:
 *      gemm_a8w8_blockscale(XQ, WQ, x_scale, w_scale, dtype) -> Y.)
 *
 * A       fp8 [M, K] row-major (K contiguous)
 * B       fp8 [N, K] row-major (the weight, K contiguous)
 * a_scale fp32 [M, ceil(K/128)] row-major (one scale per 1x128 group of A)
 * b_scale fp32 [ceil(N/128), ceil(K/128)] (one scale per 128x128 block of B)
 * C       bf16 [M, N], row stride ldc >= N
 * C[m,n] = bf16( sum_kb a_scale[m,kb] * b_scale[n/128,kb] *
 *                sum_{k in kb} A[m,k] * B[n,k] ), fp32 accumulation.
 * Limits: K % 16 == 0 (TMA row alignment); A, B 16-byte aligned; M, N >= 1.
 */
int fp8_blockscale_gemm(const uint8_t* A, const uint8_t* B,
                        const float* a_scale, const float* b_scale,
                        uint16_t* C, int ldc, int M, int N, int K, void* stream);

/*
 * S4-S7 - fused g1u1 MoE with 128x128 weight scales.
 *      (Blockscale FP8 MoE Computation: fmoe_fp8_blockscale_g1u1(out, a8, w1,
 *      w2, sorted_ids, sorted_weights, sorted_expert_ids, num_valid_ids, topk,
 *      a1_scale, fc1_scale, fc2_scale, scale_blk_n, scale_blk_k,
 *      fc2_smooth_scale).)
 *
 * out        bf16 [T, H] (every row written)
 * a8         fp8 [T, H] quantised hidden states
 * w1         fp8 [E, 2I, H]; rows [0, I) of each expert are the gate
 *            projection, rows [I, 2I) the up projection
 * w2         fp8 [E, H, I]
 * sorted_*   the outputs of moe_align_sort with block_m == fp8moe_moe_block_m(); a
 *            sorted_expert_ids that decreases from one block to the next is flagged
 *            FP8MOE_DEVERR_BLOCK_ORDER (the output is then unspecified)
 * a1_scale   fp32 [H/128, T] (transposed 1x128 scales of a8)
 * fc1_scale  fp32 [E, 2I/128, H/128];  fc2_scale fp32 [E, H/128, I/128]
 * For every pair p = (t, k) with expert e:
 *   g = blockscale(a8[t], w1[e]) (fp32), h = silu(g[:I]) * g[I:],
 *   a2 = 1x128 FP8 quantisation of h (as fp8_per_token_group_quant),
 *   y_p = blockscale(a2, w2[e]),
 *   out[t] = bf16( sum_{k=0..topk-1} bf16(w_{t,k} * y_{t,k}) ), each weighted
 * row rounded once to bf16 and the topk rows summed in fp32 in k order, which
 * makes the output independent of scheduling (deterministic). A pair absent
 * from the sorted list (its expert masked out by moe_align_sort_masked, or its
 * id dropped as out of range) adds nothing; a token with no pair present gets
 * a zero row.
 * Limits: scale_blk_n == scale_blk_k == 128; H % 128 == 0; I % 128 == 0;
 * topk <= 32 (it may exceed E: an expert-parallel rank holds fewer experts than a
 * token picks);
 * fc2_smooth_scale must be NULL (the pages do not define it); workspace >=
 * fused_moe_fp8_blockscale_g1u1_workspace(); capacity >= the sort's padded
 * length; workspace 256-byte aligned.
 * Workspace contents after a call (parts in this order, each starting at the
 * next multiple of 256 bytes; cap = capacity, P = T*topk): the slot-ordered
 * activations fp8 [cap, H] and their scales fp32 [H/128, cap]; the re-quantised
 * intermediate a2 fp8 [cap, I] and its scales fp32 [I/128, cap] (slot s holds
 * pair sorted_ids[s]; padding slots are not written); the weighted
 * down-projection rows bf16 [P, H] by pair id; a listed-pair count (16 bytes)
 * and one flag byte per pair.
 */
size_t fused_moe_fp8_blockscale_g1u1_workspace(int T, int topk, int E, int H, int I,
                                                int block_m);
int fused_moe_fp8_blockscale_g1u1(uint16_t* out, const uint8_t* a8,
                                  const uint8_t* w1, const uint8_t* w2,
                                  const int32_t* sorted_ids,
                                  const float* sorted_weights,
                                  const int32_t* sorted_expert_ids,
                                  const int32_t* num_valid_ids,
                                  int T, int H, int I, int E, int topk,
                                  int block_m, size_t capacity,
                                  const float* a1_scale, const float* fc1_scale,
                                  const float* fc2_scale, int scale_blk_n,
                                  int scale_blk_k, const float* fc2_smooth_scale,
                                  void* workspace, size_t workspace_bytes,
                                  void* stream);

/*
 * S4-S7 on tiled weights: fused_moe_fp8_blockscale_g1u1 with w1 and w2 in the
 * layout fp8_tile_weights writes (w1 tiled as [E, 2I/128, H/128, 128, 128], w2 as
 * [E, H/128, I/128, 128, 128]); every other argument, the workspace and the result
 * (bit for bit) as fused_moe_fp8_blockscale_g1u1. Each 128 x 128 weight block is
 * then one contiguous 16 KB read instead of 128 reads of 128 bytes a row apart.
 */
int fused_moe_fp8_blockscale_g1u1_tiled(uint16_t* out, const uint8_t* a8,
                                        const uint8_t* w1, const uint8_t* w2,
                                        const int32_t* sorted_ids,
                                        const float* sorted_weights,
                                        const int32_t* sorted_expert_ids,
                                        const int32_t* num_valid_ids,
                                        int T, int H, int I, int E, int topk,
                                        int block_m, size_t capacity,
                                        const float* a1_scale, const float* fc1_scale,
                                        const float* fc2_scale, int scale_blk_n,
                                        int scale_blk_k, const float* fc2_smooth_scale,
                                        void* workspace, size_t workspace_bytes,
                                        void* stream);

/*
 * Fused g1u1 MoE without any device allocation by the caller.
 * (No counterpart in the source pages: an addition for callers that cannot
 * allocate.)
 *
 * Same computation, arguments, layouts and limits as
 * fused_moe_fp8_blockscale_g1u1, minus the workspace: the call uses a scratch
 * array built into this library instead. It is for callers that must not
 * allocate device memory at the point of the call, for example a serving loop
 * whose memory manager owns all device memory after start-up, or a
 * latency-critical path that cannot afford cudaMalloc's implicit device-wide
 * synchronisation.
 *
 * The scratch is a fixed FP8MOE_NOALLOC_SCRATCH_BYTES array that every GPU
 * loading the library keeps until the process exits. A problem whose scratch
 * (fused_moe_fp8_blockscale_g1u1_workspace for the given capacity) is larger
 * is rejected with FP8MOE_EUNSUPPORTED before anything is launched. The first
 * call on a device looks up the array's device address (cudaGetSymbolAddress);
 * make that first call before capturing any stream on that device. A lookup
 * that fails returns FP8MOE_ECUDA and is tried again by the next call. All
 * calls on a device share the one array and it keeps whatever the previous
 * call left in it. The parts that must start at zero (the listed-pair count
 * and flags) are cleared by every call. The padding rows of the slot-ordered
 * activations and intermediate are never written: the GEMMs read them (and
 * their scales), possibly holding an earlier call's data, but rows are
 * independent and padding rows are never stored, so they cannot affect the
 * output. Calls that can overlap on the GPU (different streams without
 * ordering between them) race and corrupt each other: order them on one
 * stream.
 */
#define FP8MOE_NOALLOC_SCRATCH_BYTES (64ull << 20)
int fused_moe_fp8_blockscale_g1u1_noalloc(uint16_t* out, const uint8_t* a8,
                                          const uint8_t* w1, const uint8_t* w2,
                                          const int32_t* sorted_ids,
                                          const float* sorted_weights,
                                          const int32_t* sorted_expert_ids,
                                          const int32_t* num_valid_ids,
                                          int T, int H, int I, int E, int topk,
                                          int block_m, size_t capacity,
                                          const float* a1_scale,
                                          const float* fc1_scale,
                                          const float* fc2_scale, int scale_blk_n,
                                          int scale_blk_k,
                                          const float* fc2_smooth_scale,
                                          void* stream);

/*
 * S4-S6 for tensor parallelism: the fused call without its combine.
 * ("Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang", sections
 * "Blockscale FP8 MoE Computation" and "Performance Reproduction for
 * AITER-Optimized in SGLang": the layer at --tp 8, each rank holding a slice of
 * every expert's intermediate columns.)
 *
 * Arguments, limits and workspace as fused_moe_fp8_blockscale_g1u1 (weights_tiled
 * == 0) or fused_moe_fp8_blockscale_g1u1_tiled (weights_tiled != 0), minus out:
 * the call stops after the down GEMM and leaves the weighted pair rows, the
 * listed-pair count and the pair flags in the workspace (the layout given
 * above), where moe_combine_allreduce reads them. I is the rank's share of the
 * intermediate columns.
 */
int fused_moe_fp8_blockscale_g1u1_pairs(const uint8_t* a8, const uint8_t* w1,
                                        const uint8_t* w2,
                                        const int32_t* sorted_ids,
                                        const float* sorted_weights,
                                        const int32_t* sorted_expert_ids,
                                        const int32_t* num_valid_ids,
                                        int T, int H, int I, int E, int topk,
                                        int block_m, size_t capacity,
                                        const float* a1_scale, const float* fc1_scale,
                                        const float* fc2_scale, int scale_blk_n,
                                        int scale_blk_k, const float* fc2_smooth_scale,
                                        int weights_tiled, void* workspace,
                                        size_t workspace_bytes, void* stream);

/*
 * S7 fused with the tensor-parallel all-reduce, over peer (NVLink) memory.
 * ("Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang", section
 * "Other Operators": the custom all-reduce that sums the TP ranks' outputs.)
 *
 * Rank `rank` of `nranks` (<= FP8MOE_TP_MAX_RANKS), after its
 * fused_moe_fp8_blockscale_g1u1_pairs call on `workspace` (same capacity, T,
 * topk, H and I): with Ts = ceil(T / nranks), token t belongs to rank t / Ts.
 *   1. For every token t, partial_r[t] = bf16(fp32 sum of the rank's listed pair
 *      rows of t in k order) is stored into recv[p] at [r][t - p*Ts] of the
 *      owning rank p.
 *   2. For the tokens of its slice, every rank sums the nranks partials in rank
 *      order in fp32, rounds to bf16 once and stores the row into out[p] of every
 *      rank p. Every rank's out ends up bitwise identical:
 *        out[t] = bf16( sum_{q=0..n-1} partial_q[t] ).
 * One cooperative launch per rank; the call's kernel returns once every rank
 * has written this rank's out.
 *
 * recv[p]   rank p's receive buffer, bf16 [nranks][Ts][H]
 *           (moe_tp_recv_bytes bytes), 16-byte aligned
 * out[p]    rank p's output, bf16 [T][H], 16-byte aligned
 * flags[p]  rank p's FP8MOE_TP_FLAG_WORDS 64-bit words, zero before the first
 *           call, 8-byte aligned
 *           (recv, out and flags are host arrays of nranks device pointers, each
 *           as this GPU addresses that rank's memory: peer memory mapped by
 *           CUDA IPC or virtual memory management, or local memory for this rank)
 * barrier   FP8MOE_TP_BARRIER_WORDS 64-bit words in this GPU's memory, zero
 *           before the first call: where the rank's CTAs meet, and the rank's
 *           count of calls, which gives each call its flag value (epoch). No
 *           value comes from the host, so the call can be captured in a CUDA
 *           graph: every replay advances the count as a launch does.
 * Ownership: every buffer belongs to the caller; nothing is allocated. Every rank
 * must make the same sequence of calls; a rank that does not arrive leaves the
 * others waiting until the bounded wait (about 2 s) expires, which sets
 * FP8MOE_DEVERR_TIMEOUT, after which the output is unspecified and flags and
 * barrier words must be zeroed again on every rank before the next call. out may
 * be read by later work on the same stream; a second call overwrites it.
 * Returns FP8MOE_EINVAL for a bad rank, size, alignment or null pointer and
 * FP8MOE_ECUDA when the cooperative launch fails.
 */
#define FP8MOE_TP_MAX_RANKS 8
#define FP8MOE_TP_FLAG_WORDS 16
#define FP8MOE_TP_BARRIER_WORDS 3
size_t moe_tp_recv_bytes(int T, int H, int nranks);
int moe_combine_allreduce(const void* workspace, size_t capacity, int T, int topk,
                          int H, int I, int nranks, int rank, void* const* recv,
                          void* const* out, uint64_t* const* flags, uint64_t* barrier,
                          void* stream);

/*
 * All nranks ranks of moe_combine_allreduce on this one GPU, in one cooperative
 * launch (each rank's share of the CTAs runs exactly the code of a one-rank
 * launch; the ranks wait on one another through the same flags and barriers).
 * workspaces[r] and barriers[r] are rank r's; every buffer is in this GPU's
 * memory. For testing the multi-rank protocol on a single GPU; the ranks' CTAs
 * must fit on the GPU at once (FP8MOE_EUNSUPPORTED otherwise).
 */
int moe_combine_allreduce_emulated(const void* const* workspaces, size_t capacity,
                                   int T, int topk, int H, int I, int nranks,
                                   void* const* recv, void* const* out,
                                   uint64_t* const* flags, uint64_t* const* barriers,
                                   void* stream);

/*
 * Expert parallelism over peer (NVLink) memory: the dispatch and the return as
 * stores and loads across GPUs instead of all-to-alls.
 * ("Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang", section
 * "Blockscale FP8 MoE Computation": asm_moe's expert_mask, the hook of expert
 * parallelism.)
 *
 * n ranks (<= FP8MOE_EP_MAX_RANKS), rank r holding experts [e0, e0 + ne) of E and
 * its own Tq tokens; global token g = q*Tq + t is token t of rank q and global
 * pair p = g*topk + k. Every rank publishes, in memory all ranks can address, its
 * routing (topk_ids int32 [Tq, topk], topk_weights fp32 [Tq, topk]), its
 * activations (a8 fp8 [Tq, H], scales fp32 [H/128, Tq]) and a return buffer (bf16
 * rows [Tq*topk, H], then a 16-byte count that must be 0 and one flag byte per
 * pair, zeroed before each forward). One forward on rank r:
 *   moe_ep_barrier                     (every rank's inputs published)
 *   moe_ep_routing                     every rank's pairs as r's local ids
 *   moe_align_sort_masked              over n*Tq tokens and ne + 1 experts, the
 *                                      last (the sentinel) masked out
 *   fused_moe_fp8_blockscale_g1u1_multi  the owner's fused MoE on its experts; the
 *                                      gather reads each pair's row where it lies,
 *                                      the down GEMM stores each pair's weighted
 *                                      row into its origin's return buffer and
 *                                      sets its flag (or moe_ep_return does it
 *                                      after the call)
 *   moe_ep_barrier                     (every rank's rows returned)
 *   moe_combine_pairs                  r's output from its return buffer
 * The result on every rank is that of fused_moe_fp8_blockscale_g1u1 on its own
 * tokens with all E experts, bit for bit (the same rows, combined in k order).
 * Host arrays `ids`, `w`, `a8`, `a1_scale`, `rows`, `pair_flags` and `words` hold
 * one device pointer per rank, as this GPU addresses that rank's memory.
 * Ownership: every buffer belongs to the caller; nothing is allocated.
 */
#define FP8MOE_EP_MAX_RANKS 8
#define FP8MOE_EP_BARRIER_WORDS 9

/* ids_out int32 [n*Tq, topk]: id - e0 for the owner's experts, ne for another
 * rank's, -1 for an id outside [0, E) (which the sort drops and flags);
 * w_out fp32 [n*Tq, topk]: the weights as they are. */
int moe_ep_routing(const int32_t* const* ids, const float* const* w, int n, int Tq,
                   int topk, int E, int e0, int ne, int32_t* ids_out, float* w_out,
                   void* stream);

/* fused_moe_fp8_blockscale_g1u1_pairs over the n*Tq global tokens, with the
 * activations a8[q] (fp8 [Tq, H], 16-byte aligned) and scales a1_scale[q] (fp32
 * [H/128, Tq]) read from rank q's memory; w1, w2 and their scales are the
 * owner's ne experts; sorted_* come from moe_align_sort_masked over the routing
 * of moe_ep_routing (T = n*Tq, ne + 1 experts); workspace as for
 * fused_moe_fp8_blockscale_g1u1 with T = n*Tq and that capacity.
 * return_rows, return_flags: NULL (the weighted pair rows stay in the workspace,
 * for moe_ep_return), or DEVICE arrays of n pointers to every rank's return rows
 * (bf16 [Tq*topk, H], 16-byte aligned) and pair flags (bytes [Tq*topk]): the down
 * GEMM's epilogue then stores each pair's row straight into its origin's return
 * rows and sets its flag, which takes the place of moe_ep_return. */
int fused_moe_fp8_blockscale_g1u1_multi(const uint8_t* const* a8,
                                        const float* const* a1_scale, int n, int Tq,
                                        const uint8_t* w1, const uint8_t* w2,
                                        const int32_t* sorted_ids,
                                        const float* sorted_weights,
                                        const int32_t* sorted_expert_ids,
                                        const int32_t* num_valid_ids, int H, int I,
                                        int E, int topk, int block_m, size_t capacity,
                                        const float* fc1_scale, const float* fc2_scale,
                                        int scale_blk_n, int scale_blk_k,
                                        const float* fc2_smooth_scale, int weights_tiled,
                                        void* const* return_rows,
                                        void* const* return_flags, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* Every listed pair of the owner's sorted list: its weighted row (in `workspace`
 * after fused_moe_fp8_blockscale_g1u1_multi with the same capacity, n, Tq, topk, H
 * and I) is stored into rows[q] at the origin's pair id (rows[q] bf16
 * [Tq*topk, H], 16-byte aligned) and pair_flags[q] at that id set to 1. */
int moe_ep_return(const void* workspace, size_t capacity, int n, int Tq, int topk,
                  int H, int I, const int32_t* sorted_ids,
                  const int32_t* num_valid_ids, void* const* rows,
                  void* const* pair_flags, void* stream);

/* Flag barrier. Every rank has FP8MOE_EP_BARRIER_WORDS 64-bit words (zero before
 * the first call; 8-byte aligned): one per rank, then its own count of barrier
 * calls. Rank `rank` takes epoch = its count + 1, stores it into word `rank` of
 * every rank's words, waits until its own words 0..n-1 hold >= epoch and stores
 * the new count. No value comes from the host, so the call can be captured in a
 * CUDA graph. Every rank makes the same sequence of barrier calls. The stream's
 * earlier work (peer stores included) is visible to every rank past the barrier.
 * A rank that never arrives leaves the others waiting until the bounded wait
 * (about 2 s) expires: FP8MOE_DEVERR_TIMEOUT, after which every rank's words must
 * be zeroed again. The _emulated form runs all n ranks' barriers on this GPU in
 * one launch. */
int moe_ep_barrier(int n, int rank, uint64_t* const* words, void* stream);
int moe_ep_barrier_emulated(int n, uint64_t* const* words, void* stream);

/* out bf16 [T, H] = the combine of fused_moe_fp8_blockscale_g1u1 over pair rows
 * (bf16 [T*topk, H]) and a flag region laid out as the workspace's: a 16-byte
 * count of listed pairs (T*topk: no flag is read), then one flag byte per pair
 * (a pair whose flag is 0 adds nothing). rows, out, flag_region 16-byte aligned. */
int moe_combine_pairs(const uint16_t* rows, const void* flag_region, int T, int topk,
                      int H, uint16_t* out, void* stream);

/* ---------------------------------------------------------------- MLA decode
 * "Accelerate DeepSeek-R1 Inference: Integrate AITER into SGLang", section
 * "Attention Mechanisms", subsection "MLA For Decode" (mla_decode_fwd(q,
 * kv_buffer, o, kv_indptr, kv_indices, kv_last_page_lens, sm_scale, logit_cap,
 * num_kv_splits)): multi-head latent attention for one decode step, the latent KV
 * shared by every query head.
 *
 *   q            bf16 [batch, num_heads, 576], contiguous (512 latent + 64 rotary
 *                entries per head, weights absorbed), 16-byte aligned
 *   kv_buffer    bf16 [num_pages, page_size, 1, 576], contiguous, 16-byte aligned:
 *                each row is a token's key; its first 512 entries are its value
 *   o            bf16 [batch, num_heads, 512], contiguous, 16-byte aligned (output)
 *   kv_indptr    int32 [batch + 1]: sequence b's pages are
 *                kv_indices[kv_indptr[b] .. kv_indptr[b + 1]), in token order
 *   kv_indices   int32 [num_indices], each in [0, num_pages)
 *   kv_last_page_lens  int32 [batch]: tokens in each sequence's last page, in
 *                [1, page_size] (ones for page_size 1, as in the section)
 *   lse          fp32 [batch, num_heads] or NULL: ln(sum_j exp(s_j)) (output)
 *   sm_scale     > 0 (the section's default is 1/sqrt(576))
 *   logit_cap    0: scores unchanged; > 0: s -> logit_cap * tanh(s / logit_cap)
 *   num_kv_splits  <= 0: mla_decode_num_splits(batch, num_heads); otherwise the
 *                number of parts (<= 64) each sequence's tokens are split into,
 *                merged by a second kernel (log-sum-exp weights, split order)
 *   workspace    mla_decode_workspace(batch, num_heads, num_kv_splits) bytes
 *                (0 when there is one split), 16-byte aligned
 * The score of token j is s_j = sm_scale * <q, key_j> over the 576 entries, and
 * o = sum_j softmax(s)_j value_j. A sequence with no page gets o = 0 and lse =
 * -inf. num_heads must be a multiple of 16 up to 128, batch at most 65535 and
 * num_indices * page_size below 2^31 (FP8MOE_EUNSUPPORTED otherwise). Scores and sums are fp32; the softmax weights are rounded to bf16
 * before they multiply the values (their running sum adds the rounded weights).
 * A page-table entry out of range (an index outside [0, num_pages), kv_indptr not
 * non-decreasing within [0, num_indices], a last-page length outside [1,
 * page_size]) is not read: the device error word gets FP8MOE_DEVERR_PAGE and that
 * sequence's output is unspecified. Deterministic: the same inputs give the same
 * bits.
 */
#define FP8MOE_MLA_TARGET_CTAS 296   /* two resident CTAs on each of the B200's 148 SMs */
int mla_decode_num_splits(int batch, int num_heads);
size_t mla_decode_workspace(int batch, int num_heads, int num_kv_splits);
int mla_decode_fwd(const uint16_t* q, const uint16_t* kv_buffer, uint16_t* o,
                   const int32_t* kv_indptr, const int32_t* kv_indices,
                   const int32_t* kv_last_page_lens, float* lse,
                   int batch, int num_heads, int num_pages, int page_size,
                   int num_indices, float sm_scale, float logit_cap,
                   int num_kv_splits, void* workspace, size_t workspace_bytes,
                   void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8MOE_H */
