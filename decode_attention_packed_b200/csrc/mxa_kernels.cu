// Split-KV paged GQA decode attention for sm_100a.
//
// One kernel streams the KV cache: a producer warp gathers K/V pages through
// the block table with TMA into a ring of shared-memory stages, and four
// consumer warps run QK^T, the online softmax and PV on tensor cores
// (m16n8k16, fp32 accumulation) over the packed query rows of one KV head.
// A second, small kernel merges units whose KV axis was split across CTAs.
//
// Sources of the method:
//  - "SmallQ FlashAttention (Vector)" README, 算法 (Algorithm): K-outer with
//    Q resident on chip and K/V streamed block by block, double-buffered;
//    online softmax with a running max and sum per row and the rescale
//    alpha = exp(m_old - m_new) of the accumulator; 精度策略 (precision
//    policy): fp32 dot products and fp32 PV accumulation, masked reductions
//    on the partial last block, output = acc * (1 / rowSum) rounded once.
//  - "ops-transformer FlashAttention" walkthrough, "FlashAttention 的数学细节":
//    the block-wise online softmax update and the final division by l.
//  - "Flash-Attention GQA 性能调优: pack_gqa 与 num_splits", sections
//    "两个开关在 kernel 层面各做了什么" and "常见坑点": the qhead_per_khead query
//    heads of one KV head become the rows of one tile (packed row
//    m = t * G + g), and a split of the KV axis yields per-split partial
//    outputs plus their logsumexp, merged by a reduce.
//  - "MXFlashAttn 1.4.0" project page, 能力矩阵: paged KV cache, fp16/bf16,
//    head_dim 64/128, grouped query heads.
//  - "MixedQuantSparseFlashMlaMetadata 算子解析", 参数说明: the
//    RightDownCausal mask for the draft tokens of a speculative step.
#include "mxa_config.h"
#include "mxa_device.cuh"
#include "mxa_launch.h"

namespace mxa {

__device__ int g_mxa_err = 0;

constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ int clamp_len(int L, int max_len) {
  return L < 0 ? 0 : (L > max_len ? max_len : L);
}

// ---------------------------------------------------------------------------
// Producer warp: walks this CTA's segments, loads each segment's packed Q
// rows with bulk copies and every KV block of it with TMA tile loads.
// ---------------------------------------------------------------------------
template <int D>
struct Walk {
  // cursor over (row b, KV-head x row-tile hr, block blk) with `remaining`
  // blocks left in this CTA's range
  int b, hr, blk;
  long long remaining;
  long long x;        // flattened index of the next block (balanced schedule)
  long long per_cta;  // blocks per CTA range (balanced schedule)
  int L, nb;
};

template <int D>
__device__ __forceinline__ void walk_load_row(Walk<D> &w, const DecodeArgs &a) {
  w.L = clamp_len(a.seqlens[w.b], a.max_seqlen_k);
  w.nb = (w.L + block_tokens(D) - 1) / block_tokens(D);
}

// Skip rows without blocks (L_b = 0); they hold no work for the walk.
template <int D>
__device__ __forceinline__ void walk_skip_empty(Walk<D> &w, const DecodeArgs &a) {
  while (w.remaining > 0 && w.nb == 0 && w.b + 1 < a.B) {
    ++w.b;
    w.hr = 0;
    w.blk = 0;
    walk_load_row(w, a);
  }
}

template <int D, bool kBf16>
__device__ void producer_warp(const TmapPair &tm, const DecodeArgs &a, Walk<D> w, uint8_t *smem,
                              int lane) {
  constexpr int T = block_tokens(D);
  constexpr int CH = D / 64;
  constexpr uint32_t KV_BYTES = (uint32_t)T * D * 2;
  const uint32_t ring = smem_addr(smem + smem_ring_off());
  const uint32_t qtile = smem_addr(smem + smem_q_off(D));
  const uint32_t bar0 = smem_addr(smem + smem_bar_off(D));
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  const uint32_t qfull = bar0 + 8u * (2 * kStages);
  const uint32_t qempty = bar0 + 8u * (2 * kStages + 1);
  SegmentDesc *desc = reinterpret_cast<SegmentDesc *>(smem + smem_desc_off(D));

  const int HR = a.Hkv * a.RT;
  const int bt = a.box_tokens;
  const uint16_t *q = reinterpret_cast<const uint16_t *>(a.q);

  if (lane == 0) {
    prefetch_tmap(&tm.k);
    prefetch_tmap(&tm.v);
  }

  int it = 0;     // KV stages issued
  int seg_k = 0;  // segments issued
  int win_b = -1, win_base = 0, win_val = 0;  // block-table window: lane i holds entry win_base + i
  bool ok = true;

  while (ok && w.remaining > 0 && w.nb > 0) {
    const int seg_len = (int)((long long)(w.nb - w.blk) < w.remaining ? (w.nb - w.blk) : w.remaining);
    const int blk_beg = w.blk, blk_end = w.blk + seg_len;
    const int h = w.hr / a.RT, rt = w.hr % a.RT;
    const int kind = (blk_beg == 0 && blk_end == w.nb) ? 0 : (blk_beg > 0 ? 1 : 2);
    const int rows = min(kRowsPerTile, a.M - rt * kRowsPerTile);
    const int unit = (w.b * a.Hkv + h) * a.RT + rt;

    // first block of a unit: record which CTAs hold its pieces
    if (blk_beg == 0 && lane == 0 && a.meta != nullptr) {
      int c_last;
      if (a.schedule == MXA_SCHED_BALANCED) {
        c_last = (int)((w.x + w.nb - 1) / w.per_cta);
      } else {
        c_last = (int)blockIdx.x + (w.nb + a.chunk_blocks - 1) / a.chunk_blocks - 1;
      }
      a.meta[unit] = make_int2((int)blockIdx.x, c_last);
    }

    // ---- Q tile of this unit (packed rows m = t * G + g) ----
    if (!warp_wait_bounded(qempty, (seg_k & 1) ^ 1, &g_mxa_err, kErrWaitQ, lane)) { ok = false; break; }
    if (lane == 0) {
      SegmentDesc d;
      d.b = w.b; d.h = h; d.rt = rt; d.blk_beg = blk_beg; d.blk_end = blk_end;
      d.L = w.L; d.kind = kind; d.pad = 0;
      *desc = d;
      mbar_arrive_expect_tx(qfull, (uint32_t)rows * D * 2);
    }
    __syncwarp();
    if (lane < rows) {
      const int m = rt * kRowsPerTile + lane;
      const int t = m / a.G, g = m % a.G;
      const uint16_t *src = q + ((size_t)(w.b * a.q_len + t) * a.Hq + (size_t)h * a.G + g) * D;
      bulk_load(qtile + (uint32_t)lane * q_row_pitch(D), src, D * 2, qfull);
    }
    ++seg_k;

    // ---- KV blocks ----
    const int npages_b = a.contiguous ? 1 : (w.L + a.page_size - 1) / a.page_size;
    for (int blk = blk_beg; blk < blk_end; ++blk) {
      const int s = it % kStages;
      const int k = it / kStages;
      const int tok0 = blk * T;
      const int valid = min(T, w.L - tok0);
      const int nbox = (valid + bt - 1) / bt;

      int page_src_lane = 0;
      if (!a.contiguous) {
        const int first = tok0 / a.page_size;
        const int last = (tok0 + (nbox - 1) * bt) / a.page_size;
        if (win_b != w.b || first < win_base || last >= win_base + 32) {
          win_b = w.b;
          win_base = first;
          const int e = win_base + lane;
          win_val = e < npages_b ? a.block_table[(size_t)w.b * a.mpps + e] : 0;
        }
      }
      const int n_ops = nbox * CH * 2;
      const int box = lane / (CH * 2);
      const int ch = (lane / 2) % CH;
      const int kv = lane & 1;
      const int tok = tok0 + box * bt;
      if (!a.contiguous) {
        int idx = tok / a.page_size - win_base;
        page_src_lane = idx < 0 ? 0 : (idx > 31 ? 31 : idx);
      }
      const int page = __shfl_sync(0xffffffffu, win_val, page_src_lane);

      if (!warp_wait_bounded(empty_bar(s), (k & 1) ^ 1, &g_mxa_err, kErrWaitEmpty, lane)) { ok = false; break; }
      if (lane == 0) mbar_arrive_expect_tx(full_bar(s), (uint32_t)nbox * bt * D * 2 * 2);
      __syncwarp();
      if (lane < n_ops) {
        const int row = a.contiguous ? w.b * a.page_size + tok
                                     : page * a.page_size + tok % a.page_size;
        const uint32_t dst = ring + (uint32_t)s * (2 * KV_BYTES) + (uint32_t)kv * KV_BYTES +
                             (uint32_t)ch * (T * 128) + (uint32_t)(box * bt) * 128;
        tma_load_3d(dst, kv ? (const void *)&tm.v : (const void *)&tm.k, ch * 64, h, row, full_bar(s));
      }
      ++it;
    }
    if (!ok) break;

    // advance the cursor past this segment
    w.remaining -= seg_len;
    w.x += seg_len;
    w.blk = blk_end;
    if (w.blk == w.nb) {
      w.blk = 0;
      if (++w.hr == HR) {
        w.hr = 0;
        if (w.remaining > 0 && w.b + 1 < a.B) {
          ++w.b;
          walk_load_row(w, a);
          walk_skip_empty(w, a);
        } else {
          w.remaining = 0;
        }
      }
    }
  }

  grid_launch_dependents();

  if (ok) {
    // end-of-work marker for the consumers
    if (warp_wait_bounded(qempty, (seg_k & 1) ^ 1, &g_mxa_err, kErrWaitQ, lane)) {
      if (lane == 0) {
        SegmentDesc d{};
        d.kind = -1;
        *desc = d;
        mbar_arrive(qfull);
      }
      return;
    }
  }
  // Failure path: do not leave the CTA while copies this warp issued may
  // still be writing shared memory.  Wait (bounded) for the last stages.
  const int n_inflight = it < kStages ? it : kStages;
  for (int j = it - n_inflight; j < it; ++j) {
    mbar_wait_bounded(full_bar(j % kStages), (j / kStages) & 1, &g_mxa_err, kErrDrain);
  }
  if (seg_k > 0) mbar_wait_bounded(qfull, (seg_k - 1) & 1, &g_mxa_err, kErrDrain);
}

// ---------------------------------------------------------------------------
// Consumer warps
// ---------------------------------------------------------------------------

// Output of a unit whose row sees no key at all (L_b = 0): O = 0, LSE = -inf.
template <int D>
__device__ void write_empty_unit(const DecodeArgs &a, int unit, int tid) {
  const int rt = unit % a.RT, hr = unit / a.RT, h = hr % a.Hkv, b = hr / a.Hkv;
  const int rows = min(kRowsPerTile, a.M - rt * kRowsPerTile);
  uint16_t *out = reinterpret_cast<uint16_t *>(a.out);
  for (int i = tid; i < rows * D; i += kConsumerWarps * 32) {
    const int rr = i / D, d = i % D;
    const int m = rt * kRowsPerTile + rr, t = m / a.G, g = m % a.G;
    out[((size_t)(b * a.q_len + t) * a.Hq + (size_t)h * a.G + g) * D + d] = 0;  // +0 in fp16 and bf16
  }
  if (a.lse != nullptr) {
    for (int rr = tid; rr < rows; rr += kConsumerWarps * 32) {
      const int m = rt * kRowsPerTile + rr, t = m / a.G, g = m % a.G;
      a.lse[((size_t)b * a.Hq + (size_t)h * a.G + g) * a.q_len + t] = -INFINITY;
    }
  }
  if (tid == 0 && a.meta != nullptr) a.meta[unit] = make_int2((int)blockIdx.x, (int)blockIdx.x);
}

template <int D, bool kBf16>
__device__ void consumer_warps(const DecodeArgs &a, uint8_t *smem, int warp, int lane) {
  constexpr int T = block_tokens(D);
  constexpr int TW = T / kConsumerWarps;  // tokens of one warp per stage
  constexpr int NT = TW / 8;              // score n-tiles of one warp per stage
  constexpr int KS = D / 16;              // k-steps of Q K^T
  constexpr int DN = D / 8;               // n-tiles of the output
  constexpr uint32_t KV_BYTES = (uint32_t)T * D * 2;
  constexpr float NEG_INF = -INFINITY;

  const uint32_t ring = smem_addr(smem + smem_ring_off());
  const uint32_t qtile = smem_addr(smem + smem_q_off(D));
  const uint32_t bar0 = smem_addr(smem + smem_bar_off(D));
  const uint32_t qfull = bar0 + 8u * (2 * kStages);
  const uint32_t qempty = bar0 + 8u * (2 * kStages + 1);
  const uint32_t epbar = bar0 + 8u * (2 * kStages + 2);  // epilogue sync of the consumer warps
  const volatile int *desc = reinterpret_cast<const volatile int *>(smem + smem_desc_off(D));
  float *ml = reinterpret_cast<float *>(smem + smem_ml_off(D));
  float *merge = reinterpret_cast<float *>(smem + smem_merge_off(D));

  const int r = lane >> 2, c = lane & 3;
  const float sl2 = a.scale_log2;

  // Consumer-group barrier with a bounded wait (a warp that gave up on a
  // wait returns; the others then give up here instead of hanging).
  int ep_k = 0;
  auto ep_sync = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(epbar);
    const bool ok = warp_wait_bounded(epbar, ep_k & 1, &g_mxa_err, kErrWaitFull, lane);
    ++ep_k;
    return ok;
  };

  int it = 0, seg_k = 0;
  for (;;) {
    if (!warp_wait_bounded(qfull, seg_k & 1, &g_mxa_err, kErrWaitQ, lane)) return;
    const int kind = desc[6];
    if (kind < 0) return;
    const int b = desc[0], h = desc[1], rt = desc[2], blk_beg = desc[3], blk_end = desc[4];
    const int L = desc[5];
    const int rows = min(kRowsPerTile, a.M - rt * kRowsPerTile);

    // Q tile -> A fragments, resident in registers for the whole segment
    uint32_t qa[KS][4];
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
      const int col = kk * 16 + (lane >> 4) * 8;
      ldsm_x4(qtile + (uint32_t)row * q_row_pitch(D) + (uint32_t)col * 2, qa[kk][0], qa[kk][1],
              qa[kk][2], qa[kk][3]);
      if (r >= rows) qa[kk][0] = qa[kk][2] = 0u;
      if (r + 8 >= rows) qa[kk][1] = qa[kk][3] = 0u;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(qempty);
    ++seg_k;

    // keys visible to this thread's two rows (r and r + 8)
    int lim0 = L, lim1 = L, tile_lim = L;
    if (a.causal) {
      const int m0 = rt * kRowsPerTile + r, m1 = m0 + 8;
      if (r < rows) lim0 = min(L, L - a.q_len + m0 / a.G + 1);
      if (r + 8 < rows) lim1 = min(L, L - a.q_len + m1 / a.G + 1);
      tile_lim = min(L, L - a.q_len + (rt * kRowsPerTile) / a.G + 1);
    }

    float m_0 = NEG_INF, m_1 = NEG_INF, l_0 = 0.f, l_1 = 0.f;
    float o[DN][4];
#pragma unroll
    for (int dn = 0; dn < DN; ++dn) o[dn][0] = o[dn][1] = o[dn][2] = o[dn][3] = 0.f;

    for (int blk = blk_beg; blk < blk_end; ++blk) {
      const int s = it % kStages;
      const int k = it / kStages;
      if (!warp_wait_bounded(bar0 + 8u * s, k & 1, &g_mxa_err, kErrWaitFull, lane)) return;
      const uint32_t kbase = ring + (uint32_t)s * (2 * KV_BYTES);
      const uint32_t vbase = kbase + KV_BYTES;
      const int j0 = blk * T + warp * TW;  // first key of this warp's slice

      // Keys at or past L_b (page tail, unloaded boxes, stale data): their
      // weights are 0, and their V rows are zeroed so that 0 * V stays 0.
      if (j0 + TW > L) {
        for (int idx = lane; idx < TW * (D / 64) * 8; idx += 32) {
          const int jl = idx / ((D / 64) * 8);
          const int rem = idx % ((D / 64) * 8);
          if (j0 + jl >= L) {
            const uint32_t addr = vbase + (uint32_t)(rem >> 3) * (T * 128) +
                                  (uint32_t)(warp * TW + jl) * 128 + (uint32_t)(rem & 7) * 16;
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
      }

      // S = Q K^T over this warp's TW keys (fp32 accumulation)
      float sc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
        const int jl = warp * TW + nt * 8 + (lane & 7);
#pragma unroll
        for (int kk2 = 0; kk2 < KS / 2; ++kk2) {
          const int d8 = kk2 * 4 + (lane >> 3);
          const uint32_t addr = kbase + (uint32_t)(d8 >> 3) * (T * 128) + (uint32_t)jl * 128 +
                                (uint32_t)(((d8 & 7) ^ (lane & 7)) << 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(addr, b0, b1, b2, b3);
          mma_16816<kBf16>(sc[nt], qa[2 * kk2][0], qa[2 * kk2][1], qa[2 * kk2][2], qa[2 * kk2][3], b0, b1);
          mma_16816<kBf16>(sc[nt], qa[2 * kk2 + 1][0], qa[2 * kk2 + 1][1], qa[2 * kk2 + 1][2],
                           qa[2 * kk2 + 1][3], b2, b3);
        }
      }

      // online softmax in the base-2 domain: x = s * scale * log2(e)
      const bool need_mask = (j0 + TW > tile_lim);
      float mx0 = NEG_INF, mx1 = NEG_INF;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float x0 = sc[nt][e] * sl2, x1 = sc[nt][2 + e] * sl2;
          if (need_mask) {
            const int j = j0 + nt * 8 + 2 * c + e;
            x0 = j < lim0 ? x0 : NEG_INF;
            x1 = j < lim1 ? x1 : NEG_INF;
          }
          sc[nt][e] = x0;
          sc[nt][2 + e] = x1;
          mx0 = fmaxf(mx0, x0);
          mx1 = fmaxf(mx1, x1);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m_0, mx0), mn1 = fmaxf(m_1, mx1);
      const float base0 = mn0 == NEG_INF ? 0.f : mn0;  // a row with no visible key yet keeps p = 0
      const float base1 = mn1 == NEG_INF ? 0.f : mn1;
      const float alpha0 = ex2(m_0 - base0), alpha1 = ex2(m_1 - base1);
      m_0 = mn0;
      m_1 = mn1;
      float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        sc[nt][0] = ex2(sc[nt][0] - base0);
        sc[nt][1] = ex2(sc[nt][1] - base0);
        sc[nt][2] = ex2(sc[nt][2] - base1);
        sc[nt][3] = ex2(sc[nt][3] - base1);
        sum0 += sc[nt][0] + sc[nt][1];
        sum1 += sc[nt][2] + sc[nt][3];
      }
      l_0 = l_0 * alpha0 + sum0;
      l_1 = l_1 * alpha1 + sum1;
      if (__any_sync(0xffffffffu, alpha0 != 1.f || alpha1 != 1.f)) {
#pragma unroll
        for (int dn = 0; dn < DN; ++dn) {
          o[dn][0] *= alpha0;
          o[dn][1] *= alpha0;
          o[dn][2] *= alpha1;
          o[dn][3] *= alpha1;
        }
      }

      // O += P V.  P enters the tensor core as hi + lo in the input type so
      // the weights keep about 16 significant bits (fp32-like PV).
#pragma unroll
      for (int ks = 0; ks < TW / 16; ++ks) {
        uint32_t ah[4], al[4];
        split_pack<kBf16>(sc[2 * ks][0], sc[2 * ks][1], ah[0], al[0]);
        split_pack<kBf16>(sc[2 * ks][2], sc[2 * ks][3], ah[1], al[1]);
        split_pack<kBf16>(sc[2 * ks + 1][0], sc[2 * ks + 1][1], ah[2], al[2]);
        split_pack<kBf16>(sc[2 * ks + 1][2], sc[2 * ks + 1][3], ah[3], al[3]);
        const int mi = lane >> 3;
        const int jl = warp * TW + ks * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int dn2 = 0; dn2 < D / 16; ++dn2) {
          const int d8 = dn2 * 2 + (mi >> 1);
          const uint32_t addr = vbase + (uint32_t)(d8 >> 3) * (T * 128) + (uint32_t)jl * 128 +
                                (uint32_t)(((d8 & 7) ^ (lane & 7)) << 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(addr, b0, b1, b2, b3);
          mma_16816<kBf16>(o[2 * dn2], ah[0], ah[1], ah[2], ah[3], b0, b1);
          mma_16816<kBf16>(o[2 * dn2], al[0], al[1], al[2], al[3], b0, b1);
          mma_16816<kBf16>(o[2 * dn2 + 1], ah[0], ah[1], ah[2], ah[3], b2, b3);
          mma_16816<kBf16>(o[2 * dn2 + 1], al[0], al[1], al[2], al[3], b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar0 + 8u * (kStages + s));
      ++it;
    }

    // ---- epilogue: merge the four warps' (m, l, O) of this segment ----
    l_0 += __shfl_xor_sync(0xffffffffu, l_0, 1);
    l_0 += __shfl_xor_sync(0xffffffffu, l_0, 2);
    l_1 += __shfl_xor_sync(0xffffffffu, l_1, 1);
    l_1 += __shfl_xor_sync(0xffffffffu, l_1, 2);
    if (c == 0) {
      ml[(warp * 16 + r) * 2] = m_0;
      ml[(warp * 16 + r) * 2 + 1] = l_0;
      ml[(warp * 16 + r + 8) * 2] = m_1;
      ml[(warp * 16 + r + 8) * 2 + 1] = l_1;
    }
    if (!ep_sync()) return;
    float Mx0 = NEG_INF, Mx1 = NEG_INF;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      Mx0 = fmaxf(Mx0, ml[(w * 16 + r) * 2]);
      Mx1 = fmaxf(Mx1, ml[(w * 16 + r + 8) * 2]);
    }
    float Lx0 = 0.f, Lx1 = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw0 = ml[(w * 16 + r) * 2], mw1 = ml[(w * 16 + r + 8) * 2];
      if (mw0 != NEG_INF) Lx0 += ex2(mw0 - Mx0) * ml[(w * 16 + r) * 2 + 1];
      if (mw1 != NEG_INF) Lx1 += ex2(mw1 - Mx1) * ml[(w * 16 + r + 8) * 2 + 1];
    }
    const float f0 = (m_0 != NEG_INF && Lx0 > 0.f) ? ex2(m_0 - Mx0) / Lx0 : 0.f;
    const float f1 = (m_1 != NEG_INF && Lx1 > 0.f) ? ex2(m_1 - Mx1) / Lx1 : 0.f;
    const float lse0 = Lx0 > 0.f ? (Mx0 + log2f(Lx0)) * kLn2 : NEG_INF;
    const float lse1 = Lx1 > 0.f ? (Mx1 + log2f(Lx1)) * kLn2 : NEG_INF;
#pragma unroll
    for (int dn = 0; dn < DN; ++dn) {
      o[dn][0] *= f0;
      o[dn][1] *= f0;
      o[dn][2] *= f1;
      o[dn][3] *= f1;
    }
    const int npass = rows > 8 ? 2 : 1;
    const int slot = kind - 1;  // partial slot (kind 1 -> 0, kind 2 -> 1)
    for (int hf = 0; hf < npass; ++hf) {
      if (hf && !ep_sync()) return;  // warp 0 has read the first half
      if (warp > 0) {
#pragma unroll
        for (int dn = 0; dn < DN; ++dn)
          *reinterpret_cast<float2 *>(&merge[((warp - 1) * 8 + r) * D + dn * 8 + 2 * c]) =
              make_float2(o[dn][2 * hf], o[dn][2 * hf + 1]);
      }
      if (!ep_sync()) return;
      if (warp == 0) {
        const int rr = r + 8 * hf;
        if (rr < rows) {
          const int m = rt * kRowsPerTile + rr, t = m / a.G, g = m % a.G, hq = h * a.G + g;
          const float lse_v = hf ? lse1 : lse0;
#pragma unroll
          for (int dn = 0; dn < DN; ++dn) {
            float v0 = o[dn][2 * hf], v1 = o[dn][2 * hf + 1];
#pragma unroll
            for (int w = 0; w < kConsumerWarps - 1; ++w) {
              const float2 p = *reinterpret_cast<const float2 *>(&merge[(w * 8 + r) * D + dn * 8 + 2 * c]);
              v0 += p.x;
              v1 += p.y;
            }
            const int d = dn * 8 + 2 * c;
            if (kind == 0) {
              uint32_t *dst = reinterpret_cast<uint32_t *>(
                  reinterpret_cast<uint16_t *>(a.out) + ((size_t)(b * a.q_len + t) * a.Hq + hq) * D + d);
              *dst = pack2<kBf16>(v0, v1);
            } else {
              *reinterpret_cast<float2 *>(a.o_part + (((size_t)blockIdx.x * 2 + slot) * kRowsPerTile + rr) * D + d) =
                  make_float2(v0, v1);
            }
          }
          if (c == 0) {
            if (kind == 0) {
              if (a.lse != nullptr) a.lse[((size_t)b * a.Hq + hq) * a.q_len + t] = lse_v;
            } else {
              a.lse_part[((size_t)blockIdx.x * 2 + slot) * kRowsPerTile + rr] = lse_v;
            }
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// The split kernel: CTA prologue (find this CTA's range of KV blocks), then
// warp-specialised producer / consumers.
// ---------------------------------------------------------------------------
template <int D, bool kBf16>
__global__ void __launch_bounds__(kThreads, 2)
    mxa_split_kernel(const __grid_constant__ TmapPair tm, const DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int T = block_tokens(D);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((smem_addr(smem) & 1023u) != 0) {  // the 128-byte swizzle needs 1024-byte aligned stages
    if (tid == 0) atomicOr(&g_mxa_err, kErrAlign);
    return;
  }
  const uint32_t bar0 = smem_addr(smem + smem_bar_off(D));
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar0 + 8u * s, 1);                          // full: producer arrival + bytes
      mbar_init(bar0 + 8u * (kStages + s), kConsumerWarps);  // empty: one arrival per consumer warp
    }
    mbar_init(bar0 + 8u * (2 * kStages), 1);                 // qfull
    mbar_init(bar0 + 8u * (2 * kStages + 1), kConsumerWarps);// qempty
    mbar_init(bar0 + 8u * (2 * kStages + 2), kConsumerWarps);// epilogue sync
    fence_mbar_init();
  }

  const int HR = a.Hkv * a.RT;
  long long *info = reinterpret_cast<long long *>(smem + smem_ml_off(D));  // scratch until the first epilogue
  if (a.schedule == MXA_SCHED_BALANCED) {
    // Blocks per row, prefix-summed in shared memory (the ring is still free).
    int *scan = reinterpret_cast<int *>(smem + smem_ring_off());
    int *part = scan + kMaxBalancedRows;
    for (int b = tid; b < a.B; b += kThreads)
      scan[b] = (clamp_len(a.seqlens[b], a.max_seqlen_k) + T - 1) / T;
    __syncthreads();
    const int chunk = (a.B + kThreads - 1) / kThreads;
    const int lo = min(tid * chunk, a.B), hi = min(lo + chunk, a.B);
    int sum = 0;
    for (int i = lo; i < hi; ++i) sum += scan[i];
    part[tid] = sum;
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int i = 0; i < kThreads; ++i) {
        const int v = part[i];
        part[i] = run;
        run += v;
      }
      info[7] = run;
    }
    __syncthreads();
    int run = part[tid];
    for (int i = lo; i < hi; ++i) {
      run += scan[i];
      scan[i] = run;  // inclusive prefix
    }
    __syncthreads();
    if (tid == 0) {
      const long long NB = (long long)HR * info[7];
      const long long P = NB == 0 ? 1 : (NB + a.grid - 1) / a.grid;
      const long long x0 = (long long)blockIdx.x * P;
      long long b0 = 0, hr0 = 0, blk0 = 0, rem = 0;
      if (x0 < NB) {
        int lo_b = 0, hi_b = a.B - 1;  // first row whose blocks end past x0
        while (lo_b < hi_b) {
          const int mid = (lo_b + hi_b) >> 1;
          if ((long long)HR * scan[mid] > x0) hi_b = mid; else lo_b = mid + 1;
        }
        b0 = lo_b;
        const long long pre = b0 > 0 ? scan[b0 - 1] : 0;
        const long long nb = scan[b0] - pre;
        const long long off = x0 - (long long)HR * pre;
        hr0 = off / nb;
        blk0 = off % nb;
        rem = P < NB - x0 ? P : NB - x0;
      }
      info[0] = b0; info[1] = hr0; info[2] = blk0; info[3] = rem; info[4] = x0; info[5] = P;
    }
    fence_proxy_async_smem();  // generic writes above precede TMA writes to the ring
    __syncthreads();
  } else {
    if (tid == 0) {
      const int u = blockIdx.x / a.splits, si = blockIdx.x % a.splits;
      const int b = u / HR, hr = u % HR;
      const int L = clamp_len(a.seqlens[b], a.max_seqlen_k);
      const int nb = (L + T - 1) / T;
      const int beg = si * a.chunk_blocks, end = min(beg + a.chunk_blocks, nb);
      info[0] = b; info[1] = hr; info[2] = beg; info[3] = end > beg ? end - beg : 0;
      info[4] = 0; info[5] = 1;
    }
    __syncthreads();
  }

  if (warp == kConsumerWarps) {
    Walk<D> w;
    w.b = (int)info[0];
    w.hr = (int)info[1];
    w.blk = (int)info[2];
    w.remaining = info[3];
    w.x = info[4];
    w.per_cta = info[5];
    w.L = 0;
    w.nb = 0;
    if (w.remaining > 0) walk_load_row(w, a);
    producer_warp<D, kBf16>(tm, a, w, smem, lane);
    return;
  }

  // Rows with L_b = 0 belong to no KV block; one CTA per such unit writes
  // its empty result.
  if (a.schedule == MXA_SCHED_BALANCED) {
    for (int u = blockIdx.x; u < a.units; u += a.grid) {
      const int b = u / HR;
      if (clamp_len(a.seqlens[b], a.max_seqlen_k) == 0) write_empty_unit<D>(a, u, tid);
    }
  } else if (blockIdx.x % a.splits == 0) {
    const int u = blockIdx.x / a.splits;
    if (clamp_len(a.seqlens[u / HR], a.max_seqlen_k) == 0) write_empty_unit<D>(a, u, tid);
  }
  consumer_warps<D, kBf16>(a, smem, warp, lane);
  grid_launch_dependents();
}

// ---------------------------------------------------------------------------
// Merge of units split across CTAs (balanced or uniform schedule): the
// log-sum-exp reduce of the split results.  One CTA per unit.
// ---------------------------------------------------------------------------
template <int D, bool kBf16>
__global__ void __launch_bounds__(128) mxa_merge_kernel(const MergeArgs a) {
  grid_dependency_wait();  // the split kernel's writes are visible past this point
  const int u = blockIdx.x;
  const int2 mt = a.meta[u];
  if (mt.y <= mt.x) return;  // the unit was finished by one CTA
  if (mt.x < 0 || mt.y >= a.grid) return;  // not written by this call (only after a failed wait)
  const int n = mt.y - mt.x + 1;
  const int rt = u % a.RT, hr = u / a.RT, h = hr % a.Hkv, b = hr / a.Hkv;
  const int rows = min(kRowsPerTile, a.M - rt * kRowsPerTile);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the unit's pieces: the tail slot of its first CTA, then the head slots
  // of the following CTAs
  auto slot = [&](int i) { return i == 0 ? (size_t)mt.x * 2 + 1 : (size_t)(mt.x + i) * 2; };
  __shared__ float s_lse[kRowsPerTile];

  for (int rr = warp; rr < rows; rr += 4) {
    float mx = -INFINITY;
    for (int i = lane; i < n; i += 32) mx = fmaxf(mx, a.lse_part[slot(i) * kRowsPerTile + rr]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    if (mx != -INFINITY)
      for (int i = lane; i < n; i += 32) sum += expf(a.lse_part[slot(i) * kRowsPerTile + rr] - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float lse = mx == -INFINITY ? -INFINITY : mx + logf(sum);
    if (lane == 0) {
      s_lse[rr] = lse;
      if (a.lse != nullptr) {
        const int m = rt * kRowsPerTile + rr, t = m / a.G, g = m % a.G;
        a.lse[((size_t)b * a.Hq + (size_t)h * a.G + g) * a.q_len + t] = lse;
      }
    }
  }
  __syncthreads();
  for (int idx = tid; idx < rows * (D / 4); idx += 128) {
    const int rr = idx / (D / 4), d = (idx % (D / 4)) * 4;
    const float lse = s_lse[rr];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lse != -INFINITY) {
      for (int i = 0; i < n; ++i) {
        const size_t sl = slot(i);
        const float wgt = expf(a.lse_part[sl * kRowsPerTile + rr] - lse);
        const float4 v = *reinterpret_cast<const float4 *>(a.o_part + (sl * kRowsPerTile + rr) * D + d);
        acc.x += wgt * v.x;
        acc.y += wgt * v.y;
        acc.z += wgt * v.z;
        acc.w += wgt * v.w;
      }
    }
    const int m = rt * kRowsPerTile + rr, t = m / a.G, g = m % a.G;
    uint2 packed = make_uint2(pack2<kBf16>(acc.x, acc.y), pack2<kBf16>(acc.z, acc.w));
    *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(a.out) +
                               ((size_t)(b * a.q_len + t) * a.Hq + (size_t)h * a.G + g) * D + d) = packed;
  }
}

// ---------------------------------------------------------------------------
// mxa_combine: split results in the uniform layout o_part[S, B, q_len, Hq, D],
// lse_part[S, B, Hq, q_len].  One warp per (b, t, h) row.
// ---------------------------------------------------------------------------
template <bool kBf16>
__global__ void __launch_bounds__(128)
    mxa_combine_kernel(const float *__restrict__ o_part, const float *__restrict__ lse_part, int S,
                       int B, int q_len, int Hq, int D, void *out, float *lse) {
  const long long rows = (long long)B * q_len * Hq;
  const long long row = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int h = (int)(row % Hq);
  const int t = (int)((row / Hq) % q_len);
  const int b = (int)(row / ((long long)Hq * q_len));
  const size_t li = ((size_t)b * Hq + h) * q_len + t;
  float mx = -INFINITY;
  for (int s = lane; s < S; s += 32) mx = fmaxf(mx, lse_part[(size_t)s * rows + li]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
  if (mx != -INFINITY)
    for (int s = lane; s < S; s += 32) sum += expf(lse_part[(size_t)s * rows + li] - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float L = mx == -INFINITY ? -INFINITY : mx + logf(sum);
  if (lane == 0 && lse != nullptr) lse[li] = L;
  for (int d = lane * 4; d < D; d += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (L != -INFINITY) {
      for (int s = 0; s < S; ++s) {
        const float wgt = expf(lse_part[(size_t)s * rows + li] - L);
        const float4 v = *reinterpret_cast<const float4 *>(o_part + ((size_t)s * rows + row) * D + d);
        acc.x += wgt * v.x;
        acc.y += wgt * v.y;
        acc.z += wgt * v.z;
        acc.w += wgt * v.w;
      }
    }
    *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(out) + (size_t)row * D + d) =
        make_uint2(pack2<kBf16>(acc.x, acc.y), pack2<kBf16>(acc.z, acc.w));
  }
}

}  // namespace mxa

// ===========================================================================
// Host side: tensor maps and launches
// ===========================================================================
#include <cudaTypedefs.h>
#include <mutex>

namespace mxa {
namespace {

constexpr int kMaxDevices = 64;

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_kv_map(CUtensorMap *m, const void *base, int D, int Hkv, long long pool_tokens,
                   int box_tokens, bool bf16) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)pool_tokens};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
  cuuint32_t box[3] = {64u, 1u, (cuuint32_t)box_tokens};
  cuuint32_t estride[3] = {1u, 1u, 1u};
  CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                   const_cast<void *>(base), dims, strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool kBf16>
cudaError_t prepare_split_kernel(int device) {
  static std::mutex mu;
  static bool done[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (device >= 0 && device < kMaxDevices && done[device]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(mxa_split_kernel<D, kBf16>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_total(D));
  if (e == cudaSuccess && device >= 0 && device < kMaxDevices) done[device] = true;
  return e;
}

template <int D, bool kBf16>
mxa_status_t launch_typed(const DecodeLaunch &L, cudaStream_t stream) {
  constexpr int T = block_tokens(D);
  const mxa_decode_params_t &p = L.p;
  const mxa_plan_t &plan = L.plan;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return MXA_ERR_CUDA;
  if (prepare_split_kernel<D, kBf16>(device) != cudaSuccess) return MXA_ERR_CUDA;

  DecodeArgs a{};
  a.q = L.q;
  a.block_table = L.block_table;
  a.seqlens = L.seqlens;
  a.out = L.out;
  a.lse = L.lse;
  a.B = p.B;
  a.q_len = p.q_len;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.G = p.Hq / p.Hkv;
  a.M = p.q_len * a.G;
  a.RT = (a.M + kRowsPerTile - 1) / kRowsPerTile;
  a.contiguous = L.block_table == nullptr;
  a.page_size = p.page_size;
  a.mpps = p.max_pages_per_seq;
  a.max_seqlen_k = p.max_seqlen_k;
  a.box_tokens = a.contiguous ? T : (p.page_size % T == 0 ? T : p.page_size);
  a.scale_log2 = L.scale * 1.4426950408889634f;
  a.causal = L.causal;
  a.schedule = plan.schedule;
  a.grid = plan.grid;
  a.splits = plan.num_splits;
  const int max_blocks = (p.max_seqlen_k + T - 1) / T;
  a.chunk_blocks = plan.schedule == MXA_SCHED_UNIFORM
                       ? (max_blocks + plan.num_splits - 1) / plan.num_splits
                       : 1;
  if (a.chunk_blocks < 1) a.chunk_blocks = 1;
  a.units = plan.units;
  if (plan.workspace_bytes > 0) {
    uint8_t *ws = static_cast<uint8_t *>(L.workspace);
    a.meta = reinterpret_cast<int2 *>(ws);
    a.lse_part = reinterpret_cast<float *>(ws + ws_meta_bytes(plan.units));
    a.o_part = reinterpret_cast<float *>(ws + ws_meta_bytes(plan.units) + ws_lse_bytes(plan.grid));
  }

  TmapPair tm;
  const long long pool_tokens = (long long)(a.contiguous ? p.B : p.num_pages) * p.page_size;
  if (!encode_kv_map(&tm.k, L.k_cache, D, p.Hkv, pool_tokens, a.box_tokens, kBf16) ||
      !encode_kv_map(&tm.v, L.v_cache, D, p.Hkv, pool_tokens, a.box_tokens, kBf16))
    return MXA_ERR_CUDA;

  mxa_split_kernel<D, kBf16><<<plan.grid, kThreads, smem_total(D), stream>>>(tm, a);
  if (cudaGetLastError() != cudaSuccess) return MXA_ERR_CUDA;

  if (plan.needs_combine) {
    MergeArgs m{};
    m.meta = a.meta;
    m.lse_part = a.lse_part;
    m.o_part = a.o_part;
    m.out = L.out;
    m.lse = L.lse;
    m.q_len = a.q_len;
    m.Hq = a.Hq;
    m.Hkv = a.Hkv;
    m.G = a.G;
    m.M = a.M;
    m.RT = a.RT;
    m.grid = plan.grid;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)plan.units);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap the launch with the split kernel's tail
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, mxa_merge_kernel<D, kBf16>, m) != cudaSuccess) return MXA_ERR_CUDA;
  }
  return MXA_OK;
}

}  // namespace

mxa_status_t launch_decode(const DecodeLaunch &L, cudaStream_t stream) {
  const bool bf16 = L.p.dtype == MXA_BF16;
  if (L.p.D == 128) return bf16 ? launch_typed<128, true>(L, stream) : launch_typed<128, false>(L, stream);
  if (L.p.D == 64) return bf16 ? launch_typed<64, true>(L, stream) : launch_typed<64, false>(L, stream);
  return MXA_ERR_UNSUPPORTED;
}

mxa_status_t launch_combine(const float *o_part, const float *lse_part, int num_splits, int B,
                            int q_len, int Hq, int D, mxa_dtype_t dtype, void *out, float *lse,
                            cudaStream_t stream) {
  const long long rows = (long long)B * q_len * Hq;
  if (rows == 0) return MXA_OK;
  const unsigned blocks = (unsigned)((rows + 3) / 4);
  if (dtype == MXA_BF16)
    mxa_combine_kernel<true><<<blocks, 128, 0, stream>>>(o_part, lse_part, num_splits, B, q_len, Hq, D, out, lse);
  else
    mxa_combine_kernel<false><<<blocks, 128, 0, stream>>>(o_part, lse_part, num_splits, B, q_len, Hq, D, out, lse);
  return cudaGetLastError() == cudaSuccess ? MXA_OK : MXA_ERR_CUDA;
}

mxa_status_t read_device_error(int reset, int *flags) {
  int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return MXA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, g_mxa_err, sizeof(int)) != cudaSuccess) return MXA_ERR_CUDA;
  if (reset) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_mxa_err, &zero, sizeof(int)) != cudaSuccess) return MXA_ERR_CUDA;
  }
  *flags = v;
  return MXA_OK;
}

mxa_status_t current_sm_count(int *sm_count) {
  static std::mutex mu;
  static int cache[kMaxDevices] = {};
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return MXA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (device >= 0 && device < kMaxDevices && cache[device] > 0) {
    *sm_count = cache[device];
    return MXA_OK;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0)
    return MXA_ERR_CUDA;
  if (device >= 0 && device < kMaxDevices) cache[device] = n;
  *sm_count = n;
  return MXA_OK;
}

}  // namespace mxa
