// C ABI of libmxa: argument checking, the split/pack planner and the entry
// points declared in include/mxa.h.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "mxa.h"
#include "mxa_config.h"
#include "mxa_launch.h"

namespace {

using namespace mxa;

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

long long ceil_div_ll(long long a, long long b) { return (a + b - 1) / b; }

// Shape checks common to planning and running.
mxa_status_t check_shape(const mxa_decode_params_t *p) {
  if (p == nullptr) return MXA_ERR_INVALID_ARG;
  if (p->B < 0 || p->q_len < 1 || p->Hq < 1 || p->Hkv < 1 || p->Hq % p->Hkv != 0)
    return MXA_ERR_INVALID_ARG;
  if (p->dtype != MXA_F16 && p->dtype != MXA_BF16) return MXA_ERR_INVALID_ARG;
  if (p->page_size < 1 || p->num_pages < 1 || p->max_seqlen_k < 0 || p->max_pages_per_seq < 1)
    return MXA_ERR_INVALID_ARG;
  if (p->D != 64 && p->D != 128 && p->D != 256) return MXA_ERR_UNSUPPORTED;
  const long long T = block_tokens(p->D);
  const long long G = p->Hq / p->Hkv;
  const long long RT = ceil_div_ll((long long)p->q_len * G, kRowsPerTile);
  const long long units = (long long)p->B * p->Hkv * RT;
  const long long blocks = units * ceil_div_ll(p->max_seqlen_k, T);
  if (units > INT32_MAX || blocks > INT32_MAX) return MXA_ERR_UNSUPPORTED;
  // the balanced prologue sums every row's blocks plus its unit cost in 32 bits
  if (blocks + (long long)p->B * kMaxUnitCost > INT32_MAX) return MXA_ERR_UNSUPPORTED;
  if ((long long)p->num_pages * p->page_size > INT32_MAX) return MXA_ERR_UNSUPPORTED;  // TMA coordinates
  return MXA_OK;
}

// Checks that need to know whether the cache is paged.
mxa_status_t check_layout(const mxa_decode_params_t *p, bool contiguous) {
  const int T = block_tokens(p->D);
  if (contiguous) {
    if (p->num_pages != p->B && p->B > 0) return MXA_ERR_INVALID_ARG;
    if (p->page_size < p->max_seqlen_k) return MXA_ERR_INVALID_ARG;
    return MXA_OK;
  }
  if ((long long)p->max_pages_per_seq * p->page_size < p->max_seqlen_k) return MXA_ERR_INVALID_ARG;
  const bool tiles = (p->page_size % T == 0) || (T % p->page_size == 0 && p->page_size % 8 == 0);
  return tiles ? MXA_OK : MXA_ERR_UNSUPPORTED;
}

// Fill the derived fields of a plan whose schedule, num_splits and grid are set.
void finish_plan(const mxa_decode_params_t *p, mxa_plan_t *plan) {
  const int G = p->Hq / p->Hkv;
  const int RT = (p->q_len * G + kRowsPerTile - 1) / kRowsPerTile;
  plan->units = p->B * p->Hkv * RT;
  plan->rows_per_tile = kRowsPerTile;
  plan->block_tokens = block_tokens(p->D);
  plan->ctas_per_sm = ctas_per_sm(p->D);
  const bool split = plan->schedule == MXA_SCHED_BALANCED ? plan->grid > 1 : plan->num_splits > 1;
  plan->needs_combine = split && plan->units > 0 ? 1 : 0;
  plan->workspace_bytes = plan->needs_combine ? workspace_bytes(plan->units, plan->grid, p->D) : 0;
}

// Validate a run of `plan` and fill the launch description (len_add 0).
mxa_status_t prepare_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
                            const int32_t *cache_seqlens, const mxa_decode_params_t *p, float scale, int causal,
                            const mxa_plan_t *plan, void *workspace, size_t workspace_bytes, void *out,
                            float *lse, DecodeLaunch *Lout) {
  mxa_status_t st = check_shape(p);
  if (st != MXA_OK) return st;
  st = check_layout(p, block_table == nullptr);
  if (st != MXA_OK) return st;
  if (plan == nullptr) return MXA_ERR_INVALID_ARG;
  if (p->B == 0) return MXA_OK;
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || cache_seqlens == nullptr || out == nullptr)
    return MXA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(cache_seqlens, 4) || (block_table && !aligned(block_table, 4)) || (lse && !aligned(lse, 4)))
    return MXA_ERR_INVALID_ARG;
  if (!isfinite(scale) || (causal != 0 && causal != 1)) return MXA_ERR_INVALID_ARG;

  // Re-derive everything but the schedule choice from the shape.
  mxa_plan_t use = *plan;
  if (use.schedule != MXA_SCHED_UNIFORM && use.schedule != MXA_SCHED_BALANCED) return MXA_ERR_INVALID_ARG;
  if (use.grid < 1 || use.num_splits < 1) return MXA_ERR_INVALID_ARG;
  if (use.schedule == MXA_SCHED_BALANCED && (use.unit_cost < 0 || use.unit_cost > kUnitCostScale * kMaxUnitCost))
    return MXA_ERR_INVALID_ARG;
  if (use.schedule == MXA_SCHED_UNIFORM) use.unit_cost = 0;
  finish_plan(p, &use);
  if (use.schedule == MXA_SCHED_UNIFORM && (long long)use.units * use.num_splits != use.grid)
    return MXA_ERR_INVALID_ARG;
  if (use.schedule == MXA_SCHED_BALANCED && p->B > kMaxBalancedRows) return MXA_ERR_UNSUPPORTED;
  if (use.workspace_bytes > 0 && (workspace == nullptr || workspace_bytes < use.workspace_bytes ||
                                  !aligned(workspace, 256)))
    return MXA_ERR_WORKSPACE;

  DecodeLaunch &L = *Lout;
  L.q = q;
  L.k_cache = k_cache;
  L.v_cache = v_cache;
  L.block_table = block_table;
  L.seqlens = cache_seqlens;
  L.out = out;
  L.lse = lse;
  L.workspace = workspace;
  L.p = *p;
  L.plan = use;
  L.scale = scale;
  L.causal = causal;
  L.len_add = 0;
  L.k_new = L.v_new = nullptr;
  L.cu_q = nullptr;
  L.total_q = 0;
  L.out_f32 = 0;
  return MXA_OK;
}

}  // namespace

extern "C" {

const char *mxa_status_string(mxa_status_t s) {
  switch (s) {
    case MXA_OK: return "MXA_OK";
    case MXA_ERR_INVALID_ARG: return "MXA_ERR_INVALID_ARG: null or misaligned pointer, or inconsistent shape";
    case MXA_ERR_UNSUPPORTED: return "MXA_ERR_UNSUPPORTED: shape not implemented (D must be 64, 128 or 256; page size must tile the gather)";
    case MXA_ERR_WORKSPACE: return "MXA_ERR_WORKSPACE: workspace missing or smaller than the plan needs";
    case MXA_ERR_CUDA: return "MXA_ERR_CUDA: a CUDA runtime call failed";
    case MXA_ERR_TIMEOUT: return "MXA_ERR_TIMEOUT: a device-side bounded wait ran out";
  }
  return "MXA_ERR_UNKNOWN";
}

int mxa_should_pack_gqa(int varlen_q, int seqlen_q, int qhead_per_khead, int block_m) {
  if (varlen_q) return 1;
  if (seqlen_q < 1 || qhead_per_khead < 1 || block_m < 1) return 0;
  auto round_up = [](long long x, long long m) { return (x + m - 1) / m * m; };
  const double nopack = (double)seqlen_q / (double)round_up(seqlen_q, block_m);
  const long long packed_rows = (long long)seqlen_q * qhead_per_khead;
  const double pack = (double)packed_rows / (double)round_up(packed_rows, block_m);
  return nopack < 0.9 * pack ? 1 : 0;
}

int mxa_num_splits_heuristic(int tiles, int sm_count, int slots, int num_n_blocks, int max_splits,
                             int causal, int num_m_blocks, double kv_head_bytes) {
  if (tiles < 1 || sm_count < 1 || slots < 1 || max_splits < 1 || num_n_blocks < 0) return 0;
  const double l2_figure = 50.0 * 1024.0 * 1024.0;
  if (tiles >= 0.8 * sm_count) {
    // enough tiles to fill the SMs; only a very large non-causal KV head
    // with several query tiles splits, by its size relative to L2
    if (!causal && num_m_blocks > 1 && kv_head_bytes > l2_figure) {
      int s = (int)ceil(kv_head_bytes / l2_figure);
      return s < max_splits ? s : max_splits;
    }
    return 1;
  }
  if (num_n_blocks <= 4) return 1;
  double best = 0.0;
  for (int s = 1; s <= max_splits; ++s) {
    const double waves = (double)tiles * s / slots;
    const double eff = waves / ceil(waves);
    if (eff > best) best = eff;
  }
  for (int s = 1; s <= max_splits; ++s) {
    const double waves = (double)tiles * s / slots;
    if (waves / ceil(waves) >= 0.85 * best) return s;
  }
  return 1;
}

mxa_status_t mxa_plan(const mxa_decode_params_t *p, int num_splits, int sm_count, mxa_plan_t *plan) {
  if (plan == nullptr) return MXA_ERR_INVALID_ARG;
  mxa_status_t st = check_shape(p);
  if (st != MXA_OK) return st;
  if (num_splits < 0) return MXA_ERR_INVALID_ARG;
  if (sm_count <= 0) {
    st = current_sm_count(&sm_count);
    if (st != MXA_OK) return st;
  }
  mxa_plan_t out = {};
  out.sm_count = sm_count;
  const int G = p->Hq / p->Hkv;
  const int RT = (p->q_len * G + kRowsPerTile - 1) / kRowsPerTile;
  const long long units = (long long)p->B * p->Hkv * RT;
  const int T = block_tokens(p->D);
  const int rows = p->q_len * G < kRowsPerTile ? p->q_len * G : kRowsPerTile;  // packed rows of a full tile
  if (num_splits > 0) {
    if (units * num_splits > INT32_MAX) return MXA_ERR_UNSUPPORTED;
    out.schedule = MXA_SCHED_UNIFORM;
    out.num_splits = num_splits;
    out.grid = (int)(units * num_splits);
  } else {
    const int slots = sm_count * ctas_per_sm(p->D);
    const long long max_blocks = ceil_div_ll(p->max_seqlen_k, T);
    if (p->B <= kMaxBalancedRows) {
      // Balanced: every CTA streams the same number of KV blocks, so the
      // wave efficiency n_waves / ceil(n_waves) of the num_splits rule is
      // highest (1.0) for exactly one full wave of resident CTAs.  Units are
      // not cut into pieces of fewer than 4 blocks on average (the rule's
      // "no split below 4 blocks" floor), so tiny problems stay whole.
      long long cap = units * (max_blocks + 3) / 4;
      if (cap < 1) cap = 1;
      out.schedule = MXA_SCHED_BALANCED;
      const int cost = unit_cost_for_rows(rows, p->D);
      out.unit_cost = cost < max_unit_cost(p->D) ? cost : max_unit_cost(p->D);
      out.grid = (int)(slots < cap ? slots : cap);
      out.num_splits = units > 0 ? (int)ceil_div_ll(out.grid, units) : 1;
    } else {
      // Too many rows for the balanced prologue: the page's num_splits rule
      // with the uniform schedule.
      const int n_blocks_128 = (int)ceil_div_ll(p->max_seqlen_k, 128);
      int max_splits = (int)(max_blocks > 128 ? 128 : max_blocks);
      if (max_splits < 1) max_splits = 1;
      const double kv_head_bytes = (double)p->max_seqlen_k * p->D * 2.0 * 2.0;
      int s = mxa_num_splits_heuristic((int)units, sm_count, slots, n_blocks_128, max_splits, 0, RT,
                                       kv_head_bytes);
      if (s < 1) s = 1;
      if (units * s > INT32_MAX) return MXA_ERR_UNSUPPORTED;
      out.schedule = MXA_SCHED_UNIFORM;
      out.num_splits = s;
      out.grid = (int)(units * s);
    }
  }
  finish_plan(p, &out);
  *plan = out;
  return MXA_OK;
}

mxa_status_t mxa_plan_balanced(const mxa_decode_params_t *p, int grid, int sm_count,
                               mxa_plan_t *plan) {
  if (plan == nullptr || grid < 1) return MXA_ERR_INVALID_ARG;
  mxa_plan_t out;
  mxa_status_t st = mxa_plan(p, 0, sm_count, &out);
  if (st != MXA_OK) return st;
  if (p->B > kMaxBalancedRows) return MXA_ERR_UNSUPPORTED;
  out.schedule = MXA_SCHED_BALANCED;
  out.grid = grid;
  out.num_splits = out.units > 0 ? (grid + out.units - 1) / out.units : 1;
  finish_plan(p, &out);
  *plan = out;
  return MXA_OK;
}

mxa_status_t mxa_decode_fwd_with_plan(const void *q, const void *k_cache, const void *v_cache,
                                      const int32_t *block_table, const int32_t *cache_seqlens,
                                      const mxa_decode_params_t *p, float scale, int causal,
                                      const mxa_plan_t *plan, void *workspace, size_t workspace_bytes,
                                      void *out, float *lse, void *stream) {
  DecodeLaunch L;
  mxa_status_t st = prepare_decode(q, k_cache, v_cache, block_table, cache_seqlens, p, scale, causal, plan,
                                   workspace, workspace_bytes, out, lse, &L);
  if (st != MXA_OK || p->B == 0) return st;
  return launch_decode(L, static_cast<cudaStream_t>(stream));
}

mxa_status_t mxa_decode_fwd_f32out(const void *q, const void *k_cache, const void *v_cache,
                                   const int32_t *block_table, const int32_t *cache_seqlens,
                                   const mxa_decode_params_t *p, float scale, int causal, const mxa_plan_t *plan,
                                   void *workspace, size_t workspace_bytes, float *out, float *lse,
                                   void *stream) {
  DecodeLaunch L;
  mxa_status_t st = prepare_decode(q, k_cache, v_cache, block_table, cache_seqlens, p, scale, causal, plan,
                                   workspace, workspace_bytes, out, lse, &L);
  if (st != MXA_OK || p->B == 0) return st;
  L.out_f32 = 1;
  return launch_decode(L, static_cast<cudaStream_t>(stream));
}

size_t mxa_decode_workspace_size(const mxa_decode_params_t *p, int num_splits) {
  if (num_splits < 0) return SIZE_MAX;
  mxa_plan_t plan;
  // a uniform plan does not depend on the device; the automatic one is sized
  // for the current device's SMs
  const int sm_count = num_splits > 0 ? 1 : 0;
  if (mxa_plan(p, num_splits, sm_count, &plan) != MXA_OK) return SIZE_MAX;
  return plan.workspace_bytes;
}

mxa_status_t mxa_decode_fwd_append(const void *q, void *k_cache, void *v_cache, const void *k_new,
                                   const void *v_new, const int32_t *block_table, const int32_t *cache_seqlens,
                                   const mxa_decode_params_t *p, float scale, int causal, const mxa_plan_t *plan,
                                   void *workspace, size_t workspace_bytes, void *out, float *lse,
                                   void *stream) {
  DecodeLaunch L;
  mxa_status_t st = prepare_decode(q, k_cache, v_cache, block_table, cache_seqlens, p, scale, causal, plan,
                                   workspace, workspace_bytes, out, lse, &L);
  if (st != MXA_OK || p->B == 0) return st;
  if (k_new == nullptr || v_new == nullptr) return MXA_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return MXA_ERR_INVALID_ARG;
  L.len_add = p->q_len;
  L.k_new = k_new;
  L.v_new = v_new;
  return launch_decode(L, static_cast<cudaStream_t>(stream));
}

mxa_status_t mxa_decode_fwd_varlen(const void *q, const int32_t *cu_seqlens_q, int total_q, const void *k_cache,
                                   const void *v_cache, const int32_t *block_table, const int32_t *cache_seqlens,
                                   const mxa_decode_params_t *p, float scale, int causal, const mxa_plan_t *plan,
                                   void *workspace, size_t workspace_bytes, void *out, float *lse, void *stream) {
  if (p == nullptr || total_q < 0) return MXA_ERR_INVALID_ARG;
  if (p->B > 0 && (cu_seqlens_q == nullptr || !aligned(cu_seqlens_q, 4))) return MXA_ERR_INVALID_ARG;
  if (total_q == 0) {  // no query: nothing is written
    mxa_status_t st = check_shape(p);
    return st != MXA_OK ? st : check_layout(p, block_table == nullptr);
  }
  DecodeLaunch L;
  mxa_status_t st = prepare_decode(q, k_cache, v_cache, block_table, cache_seqlens, p, scale, causal, plan,
                                   workspace, workspace_bytes, out, lse, &L);
  if (st != MXA_OK || p->B == 0) return st;
  // the balanced prologue sums positions of one KV head's tiles per row in 32 bits
  const long long G = p->Hq / p->Hkv;
  const long long RT = ceil_div_ll((long long)p->q_len * G, kRowsPerTile);
  const long long row_max =
      RT * (ceil_div_ll(p->max_seqlen_k, block_tokens(p->D)) + ceil_div_ll(L.plan.unit_cost, kUnitCostScale));
  if (L.plan.schedule == MXA_SCHED_BALANCED && (long long)p->B * row_max > INT32_MAX) return MXA_ERR_UNSUPPORTED;
  L.cu_q = cu_seqlens_q;
  L.total_q = total_q;
  return launch_decode(L, static_cast<cudaStream_t>(stream));
}

mxa_status_t mxa_decode_fwd(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *block_table, const int32_t *cache_seqlens,
                            const mxa_decode_params_t *p, float scale, int causal, int num_splits,
                            void *workspace, size_t workspace_bytes, void *out, float *lse, void *stream) {
  mxa_plan_t plan;
  mxa_status_t st = mxa_plan(p, num_splits, 0, &plan);
  if (st != MXA_OK) return st;
  return mxa_decode_fwd_with_plan(q, k_cache, v_cache, block_table, cache_seqlens, p, scale, causal,
                                  &plan, workspace, workspace_bytes, out, lse, stream);
}

mxa_status_t mxa_combine(const float *o_part, const float *lse_part, int num_splits, int B, int q_len,
                         int Hq, int D, mxa_dtype_t dtype, void *out, float *lse, void *stream) {
  if (num_splits < 1 || B < 0 || q_len < 1 || Hq < 1 || D < 4 || D % 4 != 0 || D > 512)
    return MXA_ERR_INVALID_ARG;
  if (dtype != MXA_F16 && dtype != MXA_BF16) return MXA_ERR_INVALID_ARG;
  if (B == 0) return MXA_OK;
  if (o_part == nullptr || lse_part == nullptr || out == nullptr) return MXA_ERR_INVALID_ARG;
  if (!aligned(o_part, 16) || !aligned(lse_part, 4) || !aligned(out, 8) || (lse && !aligned(lse, 4)))
    return MXA_ERR_INVALID_ARG;
  return launch_combine(o_part, lse_part, num_splits, B, q_len, Hq, D, dtype, out, lse,
                        static_cast<cudaStream_t>(stream));
}

mxa_status_t mxa_device_error(int reset) {
  int flags = 0;
  mxa_status_t st = read_device_error(reset, &flags);
  if (st != MXA_OK) return st;
  if (flags & ~kErrInputMask) return MXA_ERR_TIMEOUT;
  return flags ? MXA_ERR_INVALID_ARG : MXA_OK;  // inputs outside the contract, confined and clamped
}

}  // extern "C"
