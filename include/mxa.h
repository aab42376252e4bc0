/*
 * mxa.h — C ABI of libmxa.so: exact paged grouped-query decode attention
 * for NVIDIA B200 (sm_100a).
 *
 *   O = softmax(scale * Q K^T) V,   LSE = ln sum_j exp(scale * q . k_j)
 *
 * for decode and small-qLen (speculative / MTP) queries against a paged KV
 * cache shared by groups of query heads.  The operation is the one stated in
 * the "SmallQ FlashAttention (Vector)" README (section 接口, Interface:
 * O = softmax(Q K^T / sqrt(headDim)) V with small qLen and long kvLen), on the
 * paged KV cache of the "MXFlashAttn 1.4.0" project page (能力矩阵, the
 * capability matrix: paged KV cache, FP16/BF16 forward, head_dim 64/128,
 * GQA; head_dim 256, which the same page's split-KV kernel hands back to a
 * fallback path, is served here by the same kernel), computed with the online softmax of the "ops-transformer
 * FlashAttention" walkthrough (section "FlashAttention 的数学细节"), the
 * query-head packing and KV-axis split of "Flash-Attention GQA 性能调优:
 * pack_gqa 与 num_splits 两个开关怎么选" (section "两个开关在 kernel 层面各做
 * 了什么"), and a log-sum-exp merge of the split results.
 *
 * Conventions for every call:
 *  - Pointers named as device pointers must point to device memory of the
 *    current device, 16-byte aligned, in the layouts stated (row-major,
 *    contiguous).  Scalars are passed by value.
 *  - The library allocates no device memory and keeps no pointer after a
 *    call returns.  The caller owns every buffer; scratch memory is the
 *    caller's `workspace`, sized by mxa_plan().
 *  - Launches are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL is the legacy default stream).  A returned status describes
 *    argument checking and launch only; a device-side failure (a bounded
 *    wait that ran out) is reported by mxa_device_error().
 *  - No call aborts the process, traps the GPU or falls back to another
 *    implementation: an unsupported shape is refused with a status code.
 */
#ifndef MXA_H_
#define MXA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MXA_API __attribute__((visibility("default")))
#else
#define MXA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes (integer codes, in the style of the aclnn
 * ACLNN_ERR_PARAM_INVALID family in "MixedQuantSparseFlashMlaMetadata
 * 算子解析", section 参数说明 / 约束说明). */
typedef enum {
  MXA_OK = 0,
  MXA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad shape or stride */
  MXA_ERR_UNSUPPORTED = 2,   /* a shape the kernels do not implement (e.g. D not 64/128/256) */
  MXA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than mxa_plan() says */
  MXA_ERR_CUDA = 4,          /* a CUDA runtime call failed (no device, launch error) */
  MXA_ERR_TIMEOUT = 5        /* a device-side bounded wait ran out (see mxa_device_error) */
} mxa_status_t;

typedef enum { MXA_F16 = 0, MXA_BF16 = 1 } mxa_dtype_t;

/* Work schedules of the split kernel.
 * UNIFORM:  every (batch row, KV head, row tile) unit has its KV axis cut at
 *           multiples of one chunk, chunk = ceil(max_seqlen_k / num_splits)
 *           tokens rounded up to the pipeline block; grid = units * num_splits.
 *           num_splits = 1 means one CTA per unit and no combine pass.
 * BALANCED: the work of all units, laid end to end (unit-major), is
 *           divided into `grid` equal contiguous ranges, one per CTA; a unit
 *           that straddles ranges is merged by the combine pass.  A unit's
 *           work is its KV blocks plus a fixed cost of `unit_cost` quarter
 *           blocks (its query load, the merge of its warps' results and its
 *           output stores; a cost below a whole block is shared out over the
 *           rows in whole blocks), so every CTA gets the same work however
 *           ragged the lengths are (a length-aware split in the spirit of the
 *           cost-balanced core assignment of "MixedQuantSparseFlashMlaMetadata
 *           算子解析", section 源码级原理, which also charges each task a fixed
 *           cost besides its KV length). */
typedef enum { MXA_SCHED_UNIFORM = 0, MXA_SCHED_BALANCED = 1 } mxa_schedule_t;

/* Problem shape.
 *   q            [B, q_len, Hq, D]                 dtype
 *   k/v cache    [num_pages, page_size, Hkv, D]     dtype   (paged)
 *                [B, page_size, Hkv, D]             dtype   (contiguous: block_table == NULL,
 *                                                            num_pages == B, page_size = row capacity)
 *   block_table  [B, max_pages_per_seq] int32: page id of logical page p of row b
 *                (an id outside [0, num_pages) is never dereferenced: its keys
 *                and values read as zeros, and mxa_device_error reports
 *                MXA_ERR_INVALID_ARG)
 *   cache_seqlens[B] int32: number of valid keys L_b, 0 <= L_b <= max_seqlen_k
 *                (a length outside that range is clamped into it, so no access
 *                leaves the buffers, and mxa_device_error reports
 *                MXA_ERR_INVALID_ARG)
 *   out          [B, q_len, Hq, D]                 dtype
 *   lse          [B, Hq, q_len]                    float32, natural log
 * Query head h reads KV head h / (Hq / Hkv).
 * max_seqlen_k is an upper bound on every L_b known on the host; it sizes
 * the uniform split without reading device memory. */
typedef struct {
  int B, q_len, Hq, Hkv, D;
  int num_pages, page_size;
  int max_pages_per_seq;
  int max_seqlen_k;
  mxa_dtype_t dtype;
} mxa_decode_params_t;

/* A resolved execution plan (the host half of the two-phase call: plan,
 * then run; compare the GetWorkspaceSize-then-execute pattern of the aclnn
 * API in the "SmallQ FlashAttention (Vector)" README, section aclnn API 调用). */
typedef struct {
  int num_splits;        /* splits per unit (>= 1); BALANCED: grid / units */
  int schedule;          /* mxa_schedule_t */
  int grid;              /* CTAs of the split kernel */
  int units;             /* B * Hkv * ceil(q_len * G / 16) */
  int rows_per_tile;     /* packed query rows per tile (16) */
  int block_tokens;      /* KV tokens per pipeline stage: 8192 / D for D <= 128, 64 for D = 256 */
  int ctas_per_sm;       /* resident CTAs per SM the plan assumed: 2, or 1 for D = 256 */
  int sm_count;          /* SMs the plan assumed */
  int needs_combine;     /* 1 if units may be split across CTAs and merged (needs the workspace) */
  int unit_cost;         /* BALANCED: fixed cost of a unit, in QUARTER KV blocks, added to
                            its blocks when the work is divided (0..256; mxa_plan sets one
                            block for units of one or two packed query rows, a block and a
                            half for three or four, else one block per two rows, at most 6
                            blocks; for D = 256, whose blocks are twice as large, one per
                            four rows, at least 1, at most 3); UNIFORM: unused */
  size_t workspace_bytes;/* device scratch the run needs (0 if none) */
} mxa_plan_t;

/* Text for a status code; never NULL. */
MXA_API const char *mxa_status_string(mxa_status_t status);

/* The GQA packing rule of "Flash-Attention GQA 性能调优", section
 * "pack_gqa 怎么选": varlen queries always pack; otherwise pack iff the row
 * efficiency without packing, seqlen_q / round_up(seqlen_q, block_m), is
 * below 0.9 times the efficiency with packing,
 * seqlen_q*qpk / round_up(seqlen_q*qpk, block_m).  Returns 1 (pack) or 0.
 * Pure host function.  The kernels here always pack; this rule is exported
 * so callers and tests can see that it agrees for every decode shape. */
MXA_API int mxa_should_pack_gqa(int varlen_q, int seqlen_q, int qhead_per_khead, int block_m);

/* The num_splits rule of the same page, section "num_splits 怎么选":
 *  (i)  if the tiles (batch x KV heads x query tiles) reach 80% of the SM
 *       count, use 1 split (except a non-causal problem whose single KV head
 *       exceeds the ~50 MB L2 figure with several query tiles, which splits
 *       by the ratio of KV-head bytes to that figure);
 *  (ii) if the KV axis has at most 4 blocks of block_n tokens, use 1;
 *  (iii) otherwise take, over s = 1..max_splits, the wave efficiency
 *       n_waves / ceil(n_waves) with n_waves = tiles * s / slots, and return
 *       the smallest s whose efficiency is at least 85% of the best.
 * `slots` is the number of CTAs one wave holds (SMs x resident CTAs per SM);
 * `kv_head_bytes` is the K+V bytes of one KV head of one sequence.
 * Pure host function; returns >= 1, or 0 on a bad argument. */
MXA_API int mxa_num_splits_heuristic(int tiles, int sm_count, int slots, int num_n_blocks,
                             int max_splits, int causal, int num_m_blocks,
                             double kv_head_bytes);

/* Resolve a plan for `params`.
 *   num_splits > 0 : UNIFORM schedule with that many splits per unit.
 *   num_splits == 0: automatic: BALANCED schedule over one full wave of
 *                    resident CTAs (grid = SMs x CTAs per SM, the wave
 *                    efficiency optimum when every CTA carries the same
 *                    work), capped at units * ceil(blocks per unit / 4) so
 *                    no unit is cut into pieces under 4 blocks on average;
 *                    for B above 12288 rows, UNIFORM with s from
 *                    mxa_num_splits_heuristic.
 *   sm_count > 0   : plan for that many SMs (pure host computation);
 *   sm_count <= 0  : query the current CUDA device (MXA_ERR_CUDA without one).
 * Errors: MXA_ERR_INVALID_ARG for a NULL pointer or an inconsistent shape
 * (B < 0, q_len < 1, Hq % Hkv != 0, page_size < 1, ...);
 * MXA_ERR_UNSUPPORTED for D not in {64, 128, 256} or sizes past the int32
 * index range.  The page size is checked by the run calls, which know
 * whether the cache is paged: a paged cache needs page_size to divide the
 * stage of block_tokens tokens and be a multiple of 8, or to be a multiple
 * of block_tokens (else MXA_ERR_UNSUPPORTED); a contiguous cache takes any
 * row capacity >= max_seqlen_k. */
MXA_API mxa_status_t mxa_plan(const mxa_decode_params_t *params, int num_splits, int sm_count,
                      mxa_plan_t *plan);

/* A BALANCED plan over an explicit number of CTAs (grid >= 1), for tuning
 * the split and for tests: the same as mxa_plan's automatic plan with its
 * grid replaced.  Pure host computation apart from sm_count <= 0, which
 * queries the current device.  Errors as mxa_plan; MXA_ERR_UNSUPPORTED if
 * B exceeds the 12288 rows the balanced prologue scans. */
MXA_API mxa_status_t mxa_plan_balanced(const mxa_decode_params_t *params, int grid, int sm_count,
                                       mxa_plan_t *plan);

/* Bytes of device workspace that a run of mxa_plan(params, num_splits, ...)
 * needs: the first phase of the two-phase call ("SmallQ FlashAttention
 * (Vector)" README, section aclnn API 调用: ...GetWorkspaceSize, then the
 * operator with that workspace).  0 means no workspace is needed.
 *   num_splits > 0 : the UNIFORM plan with that many splits (a pure host
 *                    computation: the size does not depend on the device);
 *   num_splits == 0: the automatic plan for the current CUDA device.
 * Returns SIZE_MAX when mxa_plan would refuse the arguments (a NULL or
 * inconsistent params, an unsupported shape, num_splits < 0) or, for the
 * automatic plan, when no CUDA device can be queried.  mxa_plan returns the
 * same number in plan.workspace_bytes, with the rest of the plan. */
MXA_API size_t mxa_decode_workspace_size(const mxa_decode_params_t *params, int num_splits);

/* Decode attention, one call: plan (num_splits as in mxa_plan, on the
 * current device) and run.
 *   q, k_cache, v_cache, block_table, cache_seqlens : device, read only
 *   block_table may be NULL for a contiguous cache (see mxa_decode_params_t).
 *   scale      : multiplies Q K^T (usually 1/sqrt(D))
 *   causal     : 0 = every query row sees all L_b keys; 1 = query t (0-based)
 *                sees the first L_b - q_len + t + 1 keys (the draft tokens are
 *                the last q_len entries of the cache; the RightDownCausal mask
 *                of "MixedQuantSparseFlashMlaMetadata 算子解析", 参数说明)
 *   workspace  : device scratch of at least plan.workspace_bytes (may be NULL
 *                when that is 0); contents on entry are ignored
 *   out        : device [B, q_len, Hq, D] dtype (written in full)
 *   lse        : device [B, Hq, q_len] float32, or NULL to skip
 * A row that sees no key gets O = 0 and LSE = -inf.
 * Returns MXA_ERR_WORKSPACE if the workspace is missing or too small. */
MXA_API mxa_status_t mxa_decode_fwd(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *block_table, const int32_t *cache_seqlens,
                            const mxa_decode_params_t *params, float scale, int causal,
                            int num_splits, void *workspace, size_t workspace_bytes,
                            void *out, float *lse, void *stream);

/* As mxa_decode_fwd, but run a plan the caller resolved (or built) before:
 * the second phase of the two-phase call.  The plan is validated against
 * `params` (schedule, grid >= 1, units, block_tokens); a BALANCED plan may
 * use any grid >= 1 and any unit_cost in 0..256 (quarter blocks). */
MXA_API mxa_status_t mxa_decode_fwd_with_plan(const void *q, const void *k_cache, const void *v_cache,
                                      const int32_t *block_table, const int32_t *cache_seqlens,
                                      const mxa_decode_params_t *params, float scale, int causal,
                                      const mxa_plan_t *plan, void *workspace,
                                      size_t workspace_bytes, void *out, float *lse,
                                      void *stream);

/* As mxa_decode_fwd_with_plan, but `out` receives O in float32: the
 * normalised output before its one rounding to the input type (the
 * precision policy of the "SmallQ FlashAttention (Vector)" README, section
 * 精度策略: fp32 dot products and accumulation, and a single rounding of
 * acc * (1 / rowSum) at the end).  The same kernels and plan run; only the
 * output rows are stored as float32.  Uses: checking the computation itself
 * against a reference at a tolerance tighter than a 16-bit output's own
 * rounding, and callers that merge the result with partial results from
 * elsewhere (another cache segment, another GPU) through mxa_combine, which
 * takes exactly this float32 O with its LSE.
 *   out : device [B, q_len, Hq, D] float32 (written in full)
 * Other arguments and errors as mxa_decode_fwd_with_plan. */
MXA_API mxa_status_t mxa_decode_fwd_f32out(const void *q, const void *k_cache, const void *v_cache,
                                           const int32_t *block_table, const int32_t *cache_seqlens,
                                           const mxa_decode_params_t *params, float scale, int causal,
                                           const mxa_plan_t *plan, void *workspace, size_t workspace_bytes,
                                           float *out, float *lse, void *stream);

/* Append the new tokens' keys and values to the cache, then decode, in one
 * call: the k / v arguments of flash_attn_with_kvcache next to cache_seqlens
 * ("Flash-Attention GQA 性能调优: pack_gqa 与 num_splits", its usage example)
 * and the paged KV append of "MXFlashAttn 1.4.0" (能力矩阵).
 *   k_new, v_new : device [B, q_len, Hkv, D] dtype, read only: the q_len new
 *                  tokens of each row (the tokens the queries belong to)
 *   cache_seqlens: device [B], read only: L_b, the keys the cache holds before
 *                  this call (not updated; the caller adds q_len afterwards)
 *   k_cache, v_cache: written: row b's new token t goes to logical position
 *                  L_b + t (page block_table[b][(L_b + t) / page_size], slot
 *                  (L_b + t) % page_size; contiguous: row b, slot L_b + t)
 * Every query row then attends to the first L_b + q_len keys; with causal = 1
 * query t sees the first L_b + t + 1.  params->max_seqlen_k bounds L_b + q_len
 * (tokens that would land at or past it, or past the row's block-table
 * width, are not written; nor is a token whose page id lies outside
 * [0, num_pages): mxa_device_error then reports MXA_ERR_INVALID_ARG).  The
 * plan is that of mxa_plan for `params`.  One
 * kernel runs on `stream`: the CTA that streams the block holding an
 * appended token writes the token into the cache (for its KV head) and then
 * loads the block, so each token is written before it is read.
 * Other arguments and errors as mxa_decode_fwd_with_plan. */
MXA_API mxa_status_t mxa_decode_fwd_append(const void *q, void *k_cache, void *v_cache, const void *k_new,
                                           const void *v_new, const int32_t *block_table,
                                           const int32_t *cache_seqlens, const mxa_decode_params_t *params,
                                           float scale, int causal, const mxa_plan_t *plan, void *workspace,
                                           size_t workspace_bytes, void *out, float *lse, void *stream);

/* Decode rows that each have their own number of queries: the packed
 * (varlen) layout of flash_attn_varlen_func ("MXFlashAttn 1.4.0", its API
 * list), with the cu_seqlens_q offsets defined in
 * "MixedQuantSparseFlashMlaMetadata 算子解析" (参数说明).
 *   q            : device [total_q, Hq, D] dtype; row b's queries are
 *                  q[cu_seqlens_q[b] .. cu_seqlens_q[b + 1] - 1]
 *   cu_seqlens_q : device [B + 1] int32, read only: 0 = cu[0] <= cu[1] <= ...
 *                  <= cu[B] = total_q
 *   total_q      : packed query tokens (>= 0)
 *   params->q_len: the largest per-row query count (max_seqlen_q); it sizes
 *                  the plan (mxa_plan with these params) and the workspace
 *   out          : device [total_q, Hq, D] dtype (written in full)
 *   lse          : device [Hq, total_q] float32, or NULL to skip
 * Row b with q_b = cu[b+1] - cu[b] queries: non-causal, every query sees L_b
 * keys; causal, query t sees the first L_b - q_b + t + 1 (its queries are
 * the row's last q_b cache entries).  A row with q_b = 0 writes nothing.
 * Offsets are read on the device.  Offsets that break these rules (not
 * starting at 0, decreasing, ending away from total_q, or a count above
 * params->q_len) are clamped into [0, total_q] and a row's count to
 * params->q_len, so that no access leaves the buffers; the result of such a
 * call is unspecified, and mxa_device_error reports MXA_ERR_INVALID_ARG.
 * Other arguments and errors as
 * mxa_decode_fwd_with_plan; MXA_ERR_INVALID_ARG for a NULL or misaligned
 * cu_seqlens_q or total_q < 0. */
MXA_API mxa_status_t mxa_decode_fwd_varlen(const void *q, const int32_t *cu_seqlens_q, int total_q,
                                   const void *k_cache, const void *v_cache, const int32_t *block_table,
                                   const int32_t *cache_seqlens, const mxa_decode_params_t *params,
                                   float scale, int causal, const mxa_plan_t *plan, void *workspace,
                                   size_t workspace_bytes, void *out, float *lse, void *stream);

/* Decode without any device allocation, for callers that cannot allocate.
 * (An addition of this library; the source pages have no counterpart.)
 *
 * Some callers cannot call cudaMalloc at the point where they run a decode
 * step: an engine that reserves all device memory at start-up and forbids
 * allocation inside its step loop, a plugin living under another framework's
 * memory manager, or a latency-critical loop where an allocation call could
 * synchronise the device.  This call is mxa_decode_fwd without the workspace
 * arguments: it plans the same way (num_splits as in mxa_plan) and runs the
 * same kernels, but keeps the split results in one fixed 16 MiB array inside
 * the library.  It calls no allocator at all.
 *  - The array is part of the library's device image: every GPU that loads
 *    the library's device code holds those 16 MiB until the process exits.
 *    Under CUDA's lazy module loading (the default since CUDA 12) that image,
 *    array included, is loaded at the first call on each device that needs
 *    it, not when the library is opened: a caller that reserves its memory
 *    up front makes one call first (any shape whose plan splits, e.g. the
 *    decode it is about to run) and reserves after it.
 *  - A plan that needs more scratch than 16 MiB is refused with
 *    MXA_ERR_WORKSPACE (use mxa_decode_fwd with your own workspace then).
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it; make
 *    that first call before any stream capture.
 *  - Every call on a device shares the one array, which keeps whatever the
 *    last call left in it.  Nothing in it needs to start at zero: each call
 *    rewrites every entry it later reads.  Calls whose kernels overlap on the
 *    GPU (other streams, other host threads) race on the array and corrupt
 *    each other's results; serialise them.
 * Arguments and errors otherwise as mxa_decode_fwd. */
MXA_API mxa_status_t mxa_decode_fwd_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                            const int32_t *block_table, const int32_t *cache_seqlens,
                                            const mxa_decode_params_t *params, float scale, int causal,
                                            int num_splits, void *out, float *lse, void *stream);

/* Merge split results with the log-sum-exp identity (the reduce that
 * follows a KV-axis split, "Flash-Attention GQA 性能调优", section
 * "两个开关在 kernel 层面各做了什么"):
 *   LSE = ln sum_s exp(lse_s),   O = sum_s exp(lse_s - LSE) O_s
 * with the largest lse_s subtracted for stability; splits with lse_s = -inf
 * carry no weight; if all are -inf, O = 0 and LSE = -inf.
 *   o_part   device [num_splits, B, q_len, Hq, D] float32 (each O_s normalised)
 *   lse_part device [num_splits, B, Hq, q_len]    float32 (natural log)
 *   out      device [B, q_len, Hq, D] dtype
 *   lse      device [B, Hq, q_len] float32, or NULL
 * D must be a multiple of 4 and at most 512. */
MXA_API mxa_status_t mxa_combine(const float *o_part, const float *lse_part, int num_splits, int B,
                         int q_len, int Hq, int D, mxa_dtype_t dtype, void *out, float *lse,
                         void *stream);

/* Synchronise the current device and report whether any kernel of this
 * library recorded a device-side failure since the last reset: MXA_OK;
 * MXA_ERR_TIMEOUT if a bounded wait ran out; else MXA_ERR_INVALID_ARG if
 * device-resident inputs broke the call's contract (the kernels confine the
 * call to its buffers and go on): a block-table entry that a kernel used lay
 * outside [0, num_pages) (its keys read as zeros; an appended token there
 * was not written), a cache_seqlens value lay outside [0, max_seqlen_k]
 * (clamped), or varlen query offsets broke their rules (clamped);
 * MXA_ERR_CUDA if the device or the synchronisation itself failed.
 * reset != 0 clears the record.
 * After MXA_ERR_TIMEOUT a split unit's arrival counter in the workspace (or
 * in mxa_decode_fwd_noalloc's array) may be left mid-count.  Every launch
 * normally tags the counters with a fresh epoch, so a direct call recovers
 * by itself; a captured CUDA graph replays one epoch, so zero the workspace
 * (or recapture the graph) before replaying it after a timeout. */
MXA_API mxa_status_t mxa_device_error(int reset);

#ifdef __cplusplus
}
#endif

#endif /* MXA_H_ */
