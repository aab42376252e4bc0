// Kernel argument blocks and host launch entry points (internal to libmxa).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "mxa.h"

namespace mxa {

// TMA descriptors of the K and V pools: 3-D maps {D, Hkv, pool tokens} with a
// box of {64 elements, 1 head, box_tokens tokens} and 128-byte swizzle.
struct alignas(64) TmapPair {
  CUtensorMap k;
  CUtensorMap v;
};

struct DecodeArgs {
  const void *q;               // [B, q_len, Hq, D], or [total_q, Hq, D] with cu_q
  const int32_t *cu_q;         // [B + 1] offsets of each row's queries (varlen), or null
  const int32_t *block_table;  // [B, mpps] (unused when contiguous)
  const int32_t *seqlens;      // [B]
  void *out;                   // [B, q_len, Hq, D], or [total_q, Hq, D] with cu_q
  float *lse;                  // [B, Hq, q_len], or [Hq, total_q] with cu_q; or null
  unsigned long long *counters;  // [units]: epoch-tagged arrivals of split units
  float *lse_part;             // [grid][2][16]
  float *o_part;               // [grid][2][16][D]
  int B, q_len, Hq, Hkv, G, M, RT;  // varlen: q_len bounds every row's query count
  int total_q;                 // varlen: packed query tokens
  int page_size;               // slots per page (row capacity when contiguous)
  int num_pages;               // pages in the pool (paged)
  int mpps;                    // block-table row stride
  int contiguous;
  int max_seqlen_k;
  int box_tokens;              // tokens per TMA box
  float scale_log2;            // scale * log2(e)
  int causal;
  int schedule;                // mxa_schedule_t
  int splits;                  // UNIFORM: splits per unit
  int chunk_blocks;            // UNIFORM: blocks per split
  int units;
  int unit_cost;               // BALANCED: fixed cost of a unit, in quarter KV blocks
  int len_add;                 // new tokens appended to each row this call (0: none)
  const uint16_t *k_new;       // [B, q_len, Hkv, D]: the appended tokens' keys (len_add > 0)
  const uint16_t *v_new;       //   and values
  uint16_t *k_cache_w;         // the caches, written at the appended positions
  uint16_t *v_cache_w;
  unsigned int epoch;          // tags this launch's arrival counts
  int out_f32;                 // 1: out holds float32 (the value before its one rounding)
};

// Everything launch_decode needs; pointers are device pointers.
struct DecodeLaunch {
  const void *q, *k_cache, *v_cache;
  const int32_t *block_table, *seqlens;
  void *out;
  float *lse;
  void *workspace;
  mxa_decode_params_t p;
  mxa_plan_t plan;
  float scale;
  int causal;
  int len_add;  // q_len when the call appends the new tokens first, else 0
  const void *k_new, *v_new;  // [B, q_len, Hkv, D] when len_add > 0
  const int32_t *cu_q;        // varlen: [B + 1] query offsets (null: q_len queries per row)
  int total_q;                // varlen: packed query tokens
  int out_f32;                // out is float32 instead of the input type
};

// Launch the split kernel (split units are merged inside it).
mxa_status_t launch_decode(const DecodeLaunch &L, cudaStream_t stream);

// Launch the uniform-layout combine of mxa_combine().
mxa_status_t launch_combine(const float *o_part, const float *lse_part, int num_splits, int B,
                            int q_len, int Hq, int D, mxa_dtype_t dtype, void *out, float *lse,
                            cudaStream_t stream);

// Read (and optionally clear) the device-side failure record of the current device.
mxa_status_t read_device_error(int reset, int *flags);

// Multiprocessor count of the current device (cached per device).
mxa_status_t current_sm_count(int *sm_count);

}  // namespace mxa
