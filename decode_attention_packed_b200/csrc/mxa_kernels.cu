// Split-KV paged GQA decode attention for sm_100a.
//
// One kernel streams the KV cache.  Each CTA has three roles:
//  - a producer warp gathers K/V pages through the block table with TMA
//    into a ring of shared-memory stages, and brings each unit's packed Q
//    rows in with bulk copies ahead of time;
//  - four math warps run QK^T, the online softmax and PV on tensor cores
//    (m16n8k16, fp32 accumulation) over the packed query rows of one KV
//    head, each on its own slice of the keys of a stage;
//  - an epilogue warp merges the math warps' partial results of a segment,
//    writes the output (or a partial result when the unit is split across
//    CTAs), and the CTA that completes a split unit merges its pieces with
//    the log-sum-exp identity.
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
//    RightDownCausal mask for the draft tokens of a speculative step; 源码级
//    原理: a balanced division of the KV work over the cores, with a reduce
//    for rows whose keys span several cores.
#include <type_traits>

#include "mxa_config.h"
#include "mxa_device.cuh"
#include "mxa_launch.h"

namespace mxa {

__device__ int g_mxa_err = 0;

constexpr float kLn2 = 0.6931471805599453f;

// A row's key count clamped into [0, max_len]; L is taken in 64 bits so that
// a length plus the appended tokens cannot overflow.
__device__ __forceinline__ int clamp_len(long long L, int max_len) {
  return L < 0 ? 0 : (L > max_len ? max_len : (int)L);
}

__device__ __forceinline__ uint32_t bar_addr(const uint8_t *smem, int D, int i) {
  return smem_addr(smem + smem_bar_off(D)) + 8u * i;
}
// barrier indices
constexpr int B_FULL(int s) { return s; }
constexpr int B_EMPTY(int s) { return kStages + s; }
constexpr int B_QFULL = 2 * kStages;
constexpr int B_QEMPTY = 2 * kStages + 1;
constexpr int B_JOBFULL(int j) { return 2 * kStages + 2 + j; }
constexpr int B_JOBEMPTY(int j) { return 2 * kStages + 2 + kJobs + j; }
constexpr int B_MERGE = 2 * kStages + 2 + 2 * kJobs;  // pieces of a split unit landed by bulk loads
constexpr int B_INIT = B_MERGE + 1;                     // the producer has published the CTA's split units
constexpr int B_FINAL = B_INIT + 1;                     // the epilogue warp has posted the CTA's final merge
constexpr int kRingLseSlots = 32;                       // pieces' LSEs a merge landing in the ring holds

// Posted by the epilogue warp at the end of the CTA's work: whether the
// math warps join the second pass of the merge of the unit of the CTA's last
// job, and where its pieces have landed.
struct FinalMerge {
  SegmentDesc seg;
  int valid;                   // 1: join the merge
  int rows;                    // packed rows of the unit
  uint32_t land, land_rows;    // landing zone (shared-memory address) and its bytes of rows
  float lse2[kRowsPerTile];    // the rows' LSEs, base 2
};
static_assert(sizeof(FinalMerge) <= kFinalBytes, "the final merge's record fits its slot");

// Second pass of the merge of the CTA's final split unit, shared by the
// epilogue warp and the math warps (warp `wid` of kMathWarps + 1) once the
// epilogue warp has landed every piece and found the rows' LSEs:
// O = sum_i w_i O_i with w_i = exp(lse_i - LSE), one (row, 4 columns) item
// at a time, straight to the output.  The terms and their order are those of
// merge_pieces' own second pass, so a unit's result does not depend on which
// path merged it.
template <int D, bool kBf16>
__device__ void merge_pass2_coop(const DecodeArgs &a, const FinalMerge *fm, const uint8_t *smem, int wid,
                                 int lane) {
  constexpr int CW = D / 4;  // 4-column items of a row
  constexpr float kLog2e = 1.4426950408889634f;
  const int rows = fm->rows, n = fm->seg.n_pieces;
  const int rt = fm->seg.rt, h = fm->seg.h, q0 = fm->seg.q0;
  const uint32_t sbase = smem_addr(smem);
  const float *land_o = reinterpret_cast<const float *>(smem + (fm->land - sbase));
  const float *land_l = reinterpret_cast<const float *>(smem + (fm->land + fm->land_rows - sbase));
  // the epilogue warp, which posted the pass and is awake, takes the first items
  const int first = (wid == kMathWarps ? 0 : wid + 1) * 32 + lane;
  for (int item = first; item < rows * CW; item += (kMathWarps + 1) * 32) {
    const int r = item / CW, col = (item % CW) * 4;
    const float row_lse = fm->lse2[r];
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int p = 0; p < n; ++p) {
      const float l = land_l[p * kRowsPerTile + r] * kLog2e;
      const float w = (l == -INFINITY || row_lse == -INFINITY) ? 0.f : ex2(l - row_lse);
      const float4 v = *reinterpret_cast<const float4 *>(land_o + (p * rows + r) * D + col);
      acc[0] += w * v.x; acc[1] += w * v.y; acc[2] += w * v.z; acc[3] += w * v.w;
    }
    const int m = rt * kRowsPerTile + r, t = m / a.G, g = m % a.G;
    const size_t e = ((size_t)(q0 + t) * a.Hq + (size_t)h * a.G + g) * D + col;
    if (a.out_f32)
      *reinterpret_cast<float4 *>(reinterpret_cast<float *>(a.out) + e) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    else
      *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(a.out) + e) =
          make_uint2(pack2<kBf16>(acc[0], acc[1]), pack2<kBf16>(acc[2], acc[3]));
  }
}

// ---------------------------------------------------------------------------
// Producer warp
// ---------------------------------------------------------------------------

// Fixed cost, in KV blocks, of each unit of batch row i: the plan's unit
// cost is in quarter blocks, and the rows share it out in whole blocks
// (row i gets floor((i + 1) q / 4) - floor(i q / 4)), so a cost below one
// block still weighs what it should over a range of many short rows.
__device__ __forceinline__ int row_cost(const DecodeArgs &a, int i) {
  return (int)(((long long)(i + 1) * a.unit_cost) / kUnitCostScale - ((long long)i * a.unit_cost) / kUnitCostScale);
}

// Cursor over this CTA's range of work.  BALANCED: positions in a
// flattened cost space in which every unit (batch row b with nb > 0 KV
// blocks, KV head x row tile hr) spans V_b + nb positions: first its fixed
// cost V_b = row_cost(b), then one position per KV block.  `x` is the
// position of block `blk` of the current unit and `end` closes the CTA's
// range.  UNIFORM: positions are the unit's block indices.
struct Cursor {
  int b, hr, blk;
  int V;              // fixed cost of each unit of row b (balanced schedule)
  long long x, end;
  long long per_cta;  // positions per CTA range (balanced schedule)
  int L, nb;          // length and blocks of row b
  long long L_next;   // prefetched length of row b + 1 (with the appended tokens; not clamped yet)
  int rtb;            // row tiles of row b: its units are hr < Hkv * rtb
  int q0, qn;         // row b's queries: first packed token, count
  int q0_next, qn_next;  // prefetched queries of row b + 1 (per-row queries only)
};

// Queries of batch row b: its first packed token q0 and its count qn.  With
// per-row offsets the offsets read are clamped, so that every index stays in
// [0, total_q) and no row holds more than q_len queries (the bound its tiles
// and arrival counters were sized for).
template <bool kVarlen>
__device__ __forceinline__ void row_queries(const DecodeArgs &a, int b, int &q0, int &qn) {
  if constexpr (kVarlen) {
    const int s = min(max(a.cu_q[b], 0), a.total_q);
    const int e = min(max(a.cu_q[b + 1], s), a.total_q);
    q0 = s;
    qn = min(e - s, a.q_len);
  } else {
    q0 = b * a.q_len;
    qn = a.q_len;
  }
}

// Row tiles of a row with qn queries, and the packed rows of its tile rt.
__device__ __forceinline__ int row_tiles(const DecodeArgs &a, int qn) {
  return (qn * a.G + kRowsPerTile - 1) / kRowsPerTile;
}
__device__ __forceinline__ int tile_rows(const DecodeArgs &a, int qn, int rt) {
  return min(kRowsPerTile, qn * a.G - rt * kRowsPerTile);
}

// Index of the LSE of query t of row b (first packed token q0), head hq:
// [B, Hq, q_len], or [Hq, total_q] with per-row offsets.
__device__ __forceinline__ size_t lse_index(const DecodeArgs &a, int b, int q0, int hq, int t) {
  return a.cu_q != nullptr ? (size_t)hq * a.total_q + q0 + t : ((size_t)b * a.Hq + hq) * a.q_len + t;
}

template <int D, bool kVarlen>
__device__ __forceinline__ void cursor_enter_row(Cursor &c, const DecodeArgs &a, int L) {
  constexpr int T = block_tokens(D);
  c.L = L;
  c.nb = (L + T - 1) / T;
  if constexpr (kVarlen) {
    c.q0 = c.q0_next;
    c.qn = c.qn_next;
    c.rtb = row_tiles(a, c.qn);
    if (c.rtb == 0) c.nb = 0;  // a row without queries holds no units
    if (c.b + 1 < a.B) row_queries<true>(a, c.b + 1, c.q0_next, c.qn_next);
  } else {
    c.q0 = c.b * a.q_len;
    c.qn = a.q_len;
  }
  c.L_next = c.b + 1 < a.B ? (long long)a.seqlens[c.b + 1] + a.len_add : 0;  // consumed a segment later
  c.V = a.schedule == MXA_SCHED_BALANCED ? row_cost(a, c.b) : 0;
}

// The segment at the cursor (a contiguous block range of one unit); the
// cursor moves past it, and past the fixed cost of the unit that follows.
template <int D, bool kVarlen>
__device__ SegmentDesc cursor_take(Cursor &c, const DecodeArgs &a) {
  const int HR = a.Hkv * c.rtb;
  SegmentDesc s;
  const long long left = c.nb - c.blk, room = c.end - c.x;
  const int len = (int)(left < room ? left : room);
  s.b = c.b;
  s.h = c.hr / c.rtb;
  s.rt = c.hr % c.rtb;
  s.blk_beg = c.blk;
  s.blk_end = c.blk + len;
  s.L = c.L;
  s.kind = (s.blk_beg == 0 && s.blk_end == c.nb) ? 0 : (s.blk_beg > 0 ? 1 : 2);
  if (a.schedule == MXA_SCHED_BALANCED) {
    const long long xs = c.x - c.blk;  // position of the unit's first block
    s.c_first = (int)(xs / c.per_cta);
    s.n_pieces = (int)((xs + c.nb - 1) / c.per_cta) - s.c_first + 1;
  } else {
    const int unit = (c.b * a.Hkv + s.h) * a.RT + s.rt;
    s.c_first = unit * a.splits;
    s.n_pieces = (c.nb + a.chunk_blocks - 1) / a.chunk_blocks;
  }
  s.last = 0;
  s.q0 = c.q0;
  s.qn = c.qn;

  c.x += len;
  c.blk += len;
  if (c.blk == c.nb) {
    c.blk = 0;
    if (++c.hr == HR) {
      c.hr = 0;
      if (c.b + 1 < a.B) {
        ++c.b;
        cursor_enter_row<D, kVarlen>(c, a, clamp_len(c.L_next, a.max_seqlen_k));
        while (c.nb == 0 && c.b + 1 < a.B) {  // rows without keys (or queries) hold no units
          ++c.b;
          cursor_enter_row<D, kVarlen>(c, a, clamp_len((long long)a.seqlens[c.b] + a.len_add, a.max_seqlen_k));
        }
        if (c.x + c.V >= c.end) c.end = c.x;  // that unit's first block lies past this range
      } else {
        c.end = c.x;
      }
    }
    c.x += c.V;  // the next unit's first block follows its fixed cost
  }
  return s;
}

// This CTA's range of work.  BALANCED: the cost space of all units laid end
// to end (row-major over (b, KV head, row tile)) is cut into gridDim.x equal
// ranges; the prefix sum over rows, and the lengths themselves, are kept in
// the (still unused) ring by this warp alone, so the rows a range starts
// and ends in are known without another read of global memory.  With
// per-row queries a row's scan width covers one KV head's row tiles (the
// row's tile count is its width over a unit's), and the row's own query
// offsets are read again where a range starts.  UNIFORM: block range
// [si * chunk, (si + 1) * chunk) of unit blockIdx.x / splits.
template <int D, bool kVarlen>
__device__ Cursor cursor_start(const DecodeArgs &a, uint8_t *smem, int lane, Cursor &tail, bool &has_tail) {
  constexpr int T = block_tokens(D);
  const int HR = a.Hkv * a.RT;
  Cursor c;
  c.hr = 0;
  c.blk = 0;
  c.V = 0;
  c.x = c.end = 0;
  c.per_cta = 1;
  c.L = c.nb = c.L_next = 0;
  c.rtb = a.RT;
  c.q0 = c.qn = c.q0_next = c.qn_next = 0;
  has_tail = false;
  tail = c;
  if (a.schedule == MXA_SCHED_UNIFORM) {
    const int u = blockIdx.x / a.splits, si = blockIdx.x % a.splits;
    c.b = u / HR;
    c.hr = u % HR;
    row_queries<kVarlen>(a, c.b, c.q0, c.qn);
    c.L = clamp_len((long long)a.seqlens[c.b] + a.len_add, a.max_seqlen_k);
    c.nb = (c.L + T - 1) / T;
    if (kVarlen && c.hr % a.RT >= row_tiles(a, c.qn)) c.nb = 0;  // a tile past the row's queries
    const int beg = si * a.chunk_blocks, end = min(beg + a.chunk_blocks, c.nb);
    c.blk = beg;
    c.x = beg;
    c.end = end > beg ? end : beg;
    c.L_next = 0;
    return c;
  }
  int *scan = reinterpret_cast<int *>(smem + smem_ring_off());  // [B] prefix of unit positions
  int *lens = scan + a.B;                                        // [B] lengths, clamped
  const int chunk = (a.B + 31) / 32;
  const int lo = min(lane * chunk, a.B), hi = min(lo + chunk, a.B);
  int sum = 0;
  for (int i = lo; i < hi; ++i) {
    const int L = clamp_len((long long)a.seqlens[i] + a.len_add, a.max_seqlen_k);
    lens[i] = L;
    const int nb = (L + T - 1) / T;
    int w = nb > 0 ? nb + row_cost(a, i) : 0;  // positions of one unit of row i
    if constexpr (kVarlen) {      // times the row's tiles: one KV head's units
      int q0, qn;
      row_queries<true>(a, i, q0, qn);
      w *= row_tiles(a, qn);
    }
    scan[i] = w;
    sum += w;
  }
  __syncwarp();
  int incl = sum;  // inclusive warp scan of the lane sums
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  int run = incl - sum;
  for (int i = lo; i < hi; ++i) {
    run += scan[i];
    scan[i] = run;  // inclusive prefix of unit positions per row
  }
  __syncwarp();
  const long long HS = kVarlen ? a.Hkv : HR;  // a row spans HS times its scan width
  const long long NB = HS * total;
  c.per_cta = NB == 0 ? 1 : (NB + gridDim.x - 1) / gridDim.x;
  const long long x0 = (long long)blockIdx.x * c.per_cta;
  c.b = 0;
  if (x0 < NB) {
    const long long x1 = c.per_cta < NB - x0 ? x0 + c.per_cta : NB;
    int lo_b = 0, hi_b = a.B - 1;  // first row whose positions end past x0
    while (lo_b < hi_b) {
      const int mid = (lo_b + hi_b) >> 1;
      if (HS * scan[mid] > x0) hi_b = mid; else lo_b = mid + 1;
    }
    const long long pre = lo_b > 0 ? scan[lo_b - 1] : 0;
    const long long w = scan[lo_b] - pre;  // > 0: the row holds position x0
    const long long off = x0 - HS * pre;
    const int V = row_cost(a, lo_b);
    c.V = V;
    // positions of one unit of the row (from the scan, or its length)
    const long long uw = kVarlen ? (long long)((lens[lo_b] + T - 1) / T + V) : w;
    const long long pos = off % uw;
    c.b = lo_b;
    c.hr = (int)(off / uw);
    c.nb = (int)(uw - V);
    if constexpr (kVarlen) {
      c.rtb = (int)(w / uw);
      row_queries<true>(a, lo_b, c.q0, c.qn);
      if (lo_b + 1 < a.B) row_queries<true>(a, lo_b + 1, c.q0_next, c.qn_next);
    } else {
      c.q0 = lo_b * a.q_len;
      c.qn = a.q_len;
    }
    c.blk = pos > V ? (int)(pos - V) : 0;
    c.x = x0 - pos + V + c.blk;
    c.end = x1;
    c.L = lens[c.b];
    c.L_next = c.b + 1 < a.B ? lens[c.b + 1] : 0;

    // If the range ends inside a unit that starts within it (a tail piece),
    // that piece is handled first: its other pieces are then also done early
    // in their CTAs, and the unit's merge overlaps streaming instead of
    // lengthening the end of the kernel.
    const long long xl = x1 - 1;
    int lb = lo_b, hb = a.B - 1;
    while (lb < hb) {
      const int mid = (lb + hb) >> 1;
      if (HS * scan[mid] > xl) hb = mid; else lb = mid + 1;
    }
    const long long pre_l = lb > 0 ? scan[lb - 1] : 0;
    const long long w_l = scan[lb] - pre_l;
    const long long off_l = xl - HS * pre_l;
    const int Vl = row_cost(a, lb);
    const long long uw_l = kVarlen ? (long long)((lens[lb] + T - 1) / T + Vl) : w_l;
    const long long pos_l = off_l % uw_l;
    if (pos_l >= Vl) {  // xl falls on a KV block of that unit
      const int nb_l = (int)(uw_l - Vl), blk_l = (int)(pos_l - Vl);
      const long long x_t = xl - blk_l;  // position of that unit's first block
      if (blk_l + 1 < nb_l && x_t - Vl > x0) {
        tail.b = lb;
        tail.V = Vl;
        tail.hr = (int)(off_l / uw_l);
        tail.blk = 0;
        tail.x = x_t;
        tail.end = x1;
        tail.per_cta = c.per_cta;
        tail.nb = nb_l;
        tail.L = lens[lb];
        tail.L_next = 0;
        if constexpr (kVarlen) {
          tail.rtb = (int)(w_l / uw_l);
          row_queries<true>(a, lb, tail.q0, tail.qn);
        } else {
          tail.q0 = lb * a.q_len;
          tail.qn = a.q_len;
        }
        has_tail = true;
        c.end = x_t - Vl;  // the main walk stops where that unit begins
      }
    }
  }
  __syncwarp();
  fence_proxy_async_smem();  // these generic writes precede the TMA writes to the ring
  return c;
}

// Block-table window of the producer warp: lane i holds the page ids of
// logical pages base + i (wa) and base + 32 + i (wb) of row b.
struct Window {
  int base, wa, wb;
};

__device__ __forceinline__ int bt_entry(const DecodeArgs &a, int b, int p, int npages) {
  return p < npages ? a.block_table[(size_t)b * a.mpps + p] : 0;
}

// kAppend: the call appends new tokens to the cache (len_add > 0); kVarlen:
// every row has its own query count (offsets cu_q).  The plain decode
// instance carries none of that code.
template <int D, bool kBf16, bool kAppend, bool kVarlen>
__device__ void producer_warp(const TmapPair &tm, const DecodeArgs &a, uint8_t *smem, int lane) {
  constexpr int T = block_tokens(D);
  constexpr int CH = D / 64;
  constexpr uint32_t KV_BYTES = (uint32_t)T * D * 2;
  const uint32_t ring = smem_addr(smem + smem_ring_off());
  const uint32_t qtile = smem_addr(smem + smem_q_off(D));
  const uint32_t qfull = bar_addr(smem, D, B_QFULL), qempty = bar_addr(smem, D, B_QEMPTY);
  SegmentDesc *desc = reinterpret_cast<SegmentDesc *>(smem + smem_desc_off(D));
  const int bt = a.box_tokens;
  const int ps = a.page_size;
  const uint16_t *q = reinterpret_cast<const uint16_t *>(a.q);
  // The KV cache is read once per call: its lines leave L2 first, so the
  // lengths, block table, queries and split partials that every call
  // touches stay there.
  const uint64_t kv_policy = l2_policy_evict_first();

  if (lane == 0) {
    prefetch_tmap(&tm.k);
    prefetch_tmap(&tm.v);
  }
  // Inputs may be written by the kernel this launch depends on: read them
  // only once that grid has completed and its writes are visible.
  grid_dependency_wait();
  Cursor tail;
  bool has_tail;
  Cursor cur = cursor_start<D, kVarlen>(a, smem, lane, tail, has_tail);
  auto more = [&]() { return has_tail || (cur.x < cur.end && cur.nb > 0); };
  // Publish the units of this CTA that are split across CTAs (at most the
  // first unit of its range and the tail unit): the epilogue warp tags their
  // arrival counters with this launch's epoch before any piece is counted.
  if (lane == 0) {
    // unit id (b, KV head, row tile) of a cursor's unit, over the plan's RT tiles per row
    auto unit_of = [&](const Cursor &k) { return (k.b * a.Hkv + k.hr / k.rtb) * a.RT + k.hr % k.rtb; };
    int u_first = -1;
    if (cur.x < cur.end && cur.nb > 0) {
      const bool split = a.schedule == MXA_SCHED_BALANCED ? (cur.blk > 0 || cur.x - cur.blk + cur.nb > cur.end)
                                                          : cur.nb > a.chunk_blocks;
      if (split) u_first = unit_of(cur);
    }
    int *init_units = reinterpret_cast<int *>(smem + smem_bar_off(D) + kInitUnitsOff);
    init_units[0] = u_first;
    init_units[1] = has_tail ? unit_of(tail) : -1;
    mbar_arrive(bar_addr(smem, D, B_INIT));
  }
  auto take = [&]() {
    if (has_tail) {
      has_tail = false;
      return cursor_take<D, kVarlen>(tail, a);
    }
    return cursor_take<D, kVarlen>(cur, a);
  };

  // Publish a segment to the math warps: its descriptor and its Q tile.
  auto issue_q = [&](const SegmentDesc &s) {
    const int rows = tile_rows(a, s.qn, s.rt);
    if (lane == 0) {
      *desc = s;
      mbar_arrive_expect_tx(qfull, (uint32_t)rows * D * 2);
    }
    __syncwarp();
    if (lane < rows) {
      const int m = s.rt * kRowsPerTile + lane;
      const int t = m / a.G, g = m % a.G;
      const uint16_t *src = q + ((size_t)(s.q0 + t) * a.Hq + (size_t)s.h * a.G + g) * D;
      bulk_load(qtile + (uint32_t)lane * q_row_pitch(D), src, D * 2, qfull);
    }
  };
  // Entries past a row's last page are never used for a load; bounding by
  // the table's row width lets the window be read before L_b is known.
  auto load_window = [&](const SegmentDesc &s, Window &w) {
    w.base = 0;
    w.wa = w.wb = 0;
    if (a.contiguous) return;
    w.base = (s.blk_beg * T) / ps;
    w.wa = bt_entry(a, s.b, w.base + lane, a.mpps);
    w.wb = bt_entry(a, s.b, w.base + 32 + lane, a.mpps);
  };

  // Copy the appended tokens at positions [p0, p1) of segment `s`'s row into
  // the caches for its KV head: 16 bytes per lane, K and V rows side by side.
  // Every lane takes part in the page lookups (shuffles).
  auto write_new_tokens = [&](const SegmentDesc &s, const Window &w, int n0, int p0, int p1) {
    constexpr int CW = D * 2 / 16;  // 16-byte chunks of one head's row
    for (int p = p0; p < p1; ++p) {
      long long token;
      if (a.contiguous) {
        token = (long long)s.b * ps + p;
      } else {
        const int idx = p / ps - w.base;
        const int va = __shfl_sync(0xffffffffu, w.wa, idx & 31);
        const int vb = __shfl_sync(0xffffffffu, w.wb, idx & 31);
        const int page = idx < 32 ? va : vb;  // the same in every lane
        if (page < 0 || page >= a.num_pages) {  // not a page of the pool: skip the token, report it
          if (lane == 0) atomicOr(&g_mxa_err, kErrBadPage);
          continue;
        }
        token = (long long)page * ps + p % ps;
      }
      if (lane < 2 * CW) {
        const bool is_v = lane >= CW;
        const int c = is_v ? lane - CW : lane;
        const size_t src = ((size_t)(s.b * a.q_len + (p - n0)) * a.Hkv + s.h) * CW + c;
        const uint4 v = reinterpret_cast<const uint4 *>(is_v ? a.v_new : a.k_new)[src];
        reinterpret_cast<uint4 *>(is_v ? a.v_cache_w : a.k_cache_w)[((size_t)token * a.Hkv + s.h) * CW + c] = v;
      }
    }
  };

  int it = 0;     // KV stages issued
  int seg_k = 0;  // segments published
  bool ok = true;
  bool bad_page = false;  // a block-table entry outside [0, num_pages) was met
  if (more()) {
    SegmentDesc seg = take();
    seg.last = more() ? 0 : 1;
    int new0 = 0;  // first appended position of the row
    if constexpr (kAppend) new0 = a.seqlens[seg.b];
    Window win;
    load_window(seg, win);
    // The first segment's Q rows are requested after its first KV stage:
    // the TMA unit serves copies in turn, and the KV bytes have the longer
    // way to come.  The Q slot is free on first use.
    bool q_first = true;
    while (ok) {
      bool have_next = false, next_known = false, q_next = false;
      SegmentDesc nseg;
      Window nwin;
      int nnew0 = 0;
      for (int blk = seg.blk_beg; blk < seg.blk_end; ++blk) {
        const int s = it % kStages;
        const int k = it / kStages;
        const int tok0 = blk * T;
        const int valid = min(T, seg.L - tok0);
        const int nbox = (valid + bt - 1) / bt;
        const int n_ops = nbox * CH * 2;  // one TMA box per (page box, 64-column chunk, K or V)
        if (!a.contiguous && tok0 / ps - win.base >= 32) {  // slide the window by 32 pages
          win.base += 32;
          win.wa = win.wb;
          win.wb = bt_entry(a, seg.b, win.base + 32 + lane, a.mpps);
        }
        if (!warp_wait_bounded(bar_addr(smem, D, B_EMPTY(s)), (k & 1) ^ 1, &g_mxa_err, kErrWaitEmpty,
                               lane)) {
          ok = false;
          break;
        }
        // Tokens this call appends that fall in this block go into the cache
        // first (this unit's KV head), and are fenced against the loads below.
        if constexpr (kAppend) {
          const int n0 = new0 < 0 ? 0 : new0, n1 = (int)min((long long)new0 + a.len_add, (long long)seg.L);
          const int p0 = max(n0, tok0), p1 = min(n1, tok0 + T);
          if (p1 > p0) {
            write_new_tokens(seg, win, new0, p0, p1);
            fence_proxy_async_global();
            __syncwarp();
          }
        }
        if (lane == 0) mbar_arrive_expect_tx(bar_addr(smem, D, B_FULL(s)), (uint32_t)nbox * bt * D * 2 * 2);
        __syncwarp();
        for (int op0 = 0; op0 < n_ops; op0 += 32) {  // all lanes take part in every shuffle
          const int op = op0 + lane;
          const int box = op / (CH * 2);
          const int ch = (op / 2) % CH;
          const int kv = op & 1;
          const int tok = tok0 + box * bt;
          int page = 0;
          if (!a.contiguous) {
            const int idx = tok / ps - win.base;
            const int src = idx & 31;
            const int va = __shfl_sync(0xffffffffu, win.wa, src);
            const int vb = __shfl_sync(0xffffffffu, win.wb, src);
            page = idx < 32 ? va : vb;
            if (page < 0 || page >= a.num_pages) {  // not a page of the pool: read as zeros, reported
              bad_page |= op < n_ops;
              page = -1;  // rows [-page_size, 0): outside the map, so the box is filled with zeros
            }
          }
          if (op < n_ops) {
            const int row = a.contiguous ? seg.b * ps + tok : page * ps + tok % ps;
            const uint32_t dst = ring + (uint32_t)s * (2 * KV_BYTES) + (uint32_t)kv * KV_BYTES +
                                 (uint32_t)ch * (T * 128) + (uint32_t)(box * bt) * 128;
            tma_load_3d_hint(dst, kv ? (const void *)&tm.v : (const void *)&tm.k, ch * 64, seg.h, row,
                        bar_addr(smem, D, B_FULL(s)), kv_policy);
          }
        }
        ++it;
        if (q_first) {
          q_first = false;
          issue_q(seg);
          ++seg_k;
        }
        // Find the next segment once this one's first stage is on its way
        // (its loads then hide behind this segment's stages).
        if (!next_known) {
          next_known = true;
          have_next = more();
          if (have_next) {
            nseg = take();
            nseg.last = more() ? 0 : 1;
            if constexpr (kAppend) nnew0 = a.seqlens[nseg.b];
            load_window(nseg, nwin);
          }
        }
        // publish the next segment as soon as the math warps hold this one's Q
        if (have_next && !q_next) {
          bool free_slot = false;
          if (lane == 0) free_slot = mbar_test_wait(qempty, (seg_k & 1) ^ 1);
          if (__shfl_sync(0xffffffffu, free_slot ? 1 : 0, 0)) {
            issue_q(nseg);
            ++seg_k;
            q_next = true;
          }
        }
      }
      if (!ok || !have_next) break;
      if (!q_next) {
        if (!warp_wait_bounded(qempty, (seg_k & 1) ^ 1, &g_mxa_err, kErrWaitQ, lane)) {
          ok = false;
          break;
        }
        issue_q(nseg);
        ++seg_k;
      }
      seg = nseg;
      win = nwin;
      new0 = nnew0;
    }
  }

  if (__any_sync(0xffffffffu, bad_page) && lane == 0) atomicOr(&g_mxa_err, kErrBadPage);
  if (ok && warp_wait_bounded(qempty, (seg_k & 1) ^ 1, &g_mxa_err, kErrWaitQ, lane)) {
    if (lane == 0) {  // end-of-work marker for the math warps
      SegmentDesc d{};
      d.kind = -1;
      *desc = d;
      mbar_arrive(qfull);
    }
    return;
  }
  // Failure path: do not leave while copies this warp issued may still be
  // writing shared memory.  Wait (bounded) for the last stages and Q tile.
  const int n_inflight = it < kStages ? it : kStages;
  for (int j = it - n_inflight; j < it; ++j)
    mbar_wait_bounded(bar_addr(smem, D, B_FULL(j % kStages)), (j / kStages) & 1, &g_mxa_err, kErrDrain);
  if (seg_k > 0) mbar_wait_bounded(qfull, (seg_k - 1) & 1, &g_mxa_err, kErrDrain);
}

// ---------------------------------------------------------------------------
// Math warps
// ---------------------------------------------------------------------------

// Address of fp32 element (row, col) of math warp `warp`'s partial output
// inside its own key slice of ring stage `sbase` (the segment's last stage,
// which the warp has finished reading).  Rows of D floats; the 16-byte
// chunks of a row are XOR-swizzled by the row index against bank conflicts.
template <int D>
__device__ __forceinline__ uint32_t handoff_addr(uint32_t sbase, int warp, int row, int col) {
  constexpr int T = block_tokens(D);
  constexpr int TW = T / kMathWarps;
  constexpr int CH = D / 64;
  constexpr uint32_t KV_BYTES = (uint32_t)T * D * 2;
  const uint32_t ro = (uint32_t)row * D * 4;
  const uint32_t piece = ro / (TW * 128), within = ro % (TW * 128);
  const uint32_t region = sbase + (piece >= (uint32_t)CH ? KV_BYTES : 0u) + (piece % CH) * (T * 128) +
                          (uint32_t)warp * TW * 128;
  const uint32_t chunk = (uint32_t)(col >> 2) ^ (uint32_t)(row & 7);
  return region + within + (chunk << 4) + ((uint32_t)(col & 3) << 2);
}

template <int D, bool kBf16>
__device__ void math_warps(const DecodeArgs &a, uint8_t *smem, int warp, int lane) {
  constexpr int T = block_tokens(D);
  constexpr int TW = T / kMathWarps;  // keys of one warp per stage
  constexpr int NT = TW / 8;          // score n-tiles of one warp per stage
  constexpr int KS = D / 16;          // k-steps of Q K^T
  constexpr int DN = D / 8;           // n-tiles of the output
  constexpr uint32_t KV_BYTES = (uint32_t)T * D * 2;
  constexpr float NEG_INF = -INFINITY;

  const uint32_t ring = smem_addr(smem + smem_ring_off());
  const uint32_t qtile = smem_addr(smem + smem_q_off(D));
  const uint32_t qfull = bar_addr(smem, D, B_QFULL), qempty = bar_addr(smem, D, B_QEMPTY);
  const volatile int *desc = reinterpret_cast<const volatile int *>(smem + smem_desc_off(D));
  JobSlot *jobs = reinterpret_cast<JobSlot *>(smem + smem_jobs_off(D));

  const int r = lane >> 2, c = lane & 3;
  const float sl2 = a.scale_log2;

  int it = 0, seg_k = 0;
  for (;;) {
    if (!warp_wait_bounded(qfull, seg_k & 1, &g_mxa_err, kErrWaitQ, lane)) return;
    const int b = desc[0], h = desc[1], rt = desc[2], blk_beg = desc[3], blk_end = desc[4];
    const int L = desc[5], kind = desc[6], c_first = desc[7], n_pieces = desc[8], last = desc[9];
    const int q0 = desc[10], qn = desc[11];
    const int j = seg_k % kJobs, jk = seg_k / kJobs;
    if (kind < 0) {  // end of work: pass the marker on to the epilogue warp
      if (!warp_wait_bounded(bar_addr(smem, D, B_JOBEMPTY(j)), (jk & 1) ^ 1, &g_mxa_err, kErrWaitQ, lane))
        return;
      if (warp == 0 && lane == 0) jobs[j].seg.kind = -1;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_addr(smem, D, B_JOBFULL(j)));
      // Then join the second pass of the CTA's final merge, if the epilogue
      // warp posts one (it lands the pieces and finds the rows' LSEs).
      if (!warp_wait_bounded_idle(bar_addr(smem, D, B_FINAL), 0, &g_mxa_err, kErrWaitQ, lane)) return;
      const FinalMerge *fm = reinterpret_cast<const FinalMerge *>(smem + smem_final_off(D));
      if (fm->valid) merge_pass2_coop<D, kBf16>(a, fm, smem, warp, lane);
      return;
    }
    const int rows = tile_rows(a, qn, rt);

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
    // The Q tile is refilled by the next segment's bulk copies (the async
    // proxy) as soon as every math warp has arrived below.  These fragments
    // are first used by the block loop's tensor-core instructions, after the
    // arrival, so without a proxy fence the last ldmatrix reads may still be
    // in flight when the copies land: the high columns of a row then come
    // from the next segment's queries.  The fence orders this warp's reads
    // before the refill.
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(qempty);
    ++seg_k;

    // keys visible to this thread's two rows (r and r + 8)
    int lim0 = L, lim1 = L, tile_lim = L;
    if (a.causal) {
      const int m0 = rt * kRowsPerTile + r, m1 = m0 + 8;
      if (r < rows) lim0 = min(L, L - qn + m0 / a.G + 1);
      if (r + 8 < rows) lim1 = min(L, L - qn + m1 / a.G + 1);
      tile_lim = min(L, L - qn + (rt * kRowsPerTile) / a.G + 1);
    }

    float m_0 = NEG_INF, m_1 = NEG_INF, l_0 = 0.f, l_1 = 0.f;
    float o[DN][4];
#pragma unroll
    for (int dn = 0; dn < DN; ++dn) o[dn][0] = o[dn][1] = o[dn][2] = o[dn][3] = 0.f;

    int s_last = 0;
    for (int blk = blk_beg; blk < blk_end; ++blk) {
      const int s = it % kStages;
      const int k = it / kStages;
      if (!warp_wait_bounded(bar_addr(smem, D, B_FULL(s)), k & 1, &g_mxa_err, kErrWaitFull, lane)) return;
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
            const int jj = j0 + nt * 8 + 2 * c + e;
            x0 = jj < lim0 ? x0 : NEG_INF;
            x1 = jj < lim1 ? x1 : NEG_INF;
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
      if (blk + 1 < blk_end) {
        if (lane == 0) mbar_arrive(bar_addr(smem, D, B_EMPTY(s)));
      } else {
        s_last = s;  // kept for the hand-off; the epilogue warp releases it
      }
      ++it;
    }

    // ---- hand-off: (m, l) per row and the unnormalised O of this warp ----
    if (!warp_wait_bounded(bar_addr(smem, D, B_JOBEMPTY(j)), (jk & 1) ^ 1, &g_mxa_err, kErrWaitQ, lane))
      return;
    l_0 += __shfl_xor_sync(0xffffffffu, l_0, 1);
    l_0 += __shfl_xor_sync(0xffffffffu, l_0, 2);
    l_1 += __shfl_xor_sync(0xffffffffu, l_1, 1);
    l_1 += __shfl_xor_sync(0xffffffffu, l_1, 2);
    if (c == 0) {
      jobs[j].ml[warp][r][0] = m_0;
      jobs[j].ml[warp][r][1] = l_0;
      jobs[j].ml[warp][r + 8][0] = m_1;
      jobs[j].ml[warp][r + 8][1] = l_1;
    }
    const uint32_t sbase = ring + (uint32_t)s_last * (2 * KV_BYTES);
#pragma unroll
    for (int dn = 0; dn < DN; ++dn) {
      const int col = dn * 8 + 2 * c;
      if (r < rows)
        asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(handoff_addr<D>(sbase, warp, r, col)),
                     "f"(o[dn][0]), "f"(o[dn][1]) : "memory");
      if (r + 8 < rows)
        asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(handoff_addr<D>(sbase, warp, r + 8, col)),
                     "f"(o[dn][2]), "f"(o[dn][3]) : "memory");
    }
    if (warp == 0 && lane == 0) {
      SegmentDesc sd;
      sd.b = b; sd.h = h; sd.rt = rt; sd.blk_beg = blk_beg; sd.blk_end = blk_end; sd.L = L;
      sd.kind = kind; sd.c_first = c_first; sd.n_pieces = n_pieces;
      sd.last = last;
      sd.q0 = q0;
      sd.qn = qn;
      jobs[j].seg = sd;
      jobs[j].stage = s_last;
    }
    fence_proxy_async_smem();  // the stage returns to TMA after the epilogue warp has read it
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_addr(smem, D, B_JOBFULL(j)));
  }
}

// ---------------------------------------------------------------------------
// Epilogue warp
// ---------------------------------------------------------------------------

// D / 32 consecutive float32 values of packed row `rr` into the rows at
// shared address `stage` (row pitch D * 4 bytes): partial results, and the
// output when it is float32.
template <int D>
__device__ __forceinline__ void stage_f32_vec(uint8_t *smem, uint32_t stage, int rr, int col, const float *v) {
  float *dst = reinterpret_cast<float *>(smem + (stage - smem_addr(smem))) + rr * D + col;
  if constexpr (D / 32 == 8) {
    reinterpret_cast<float4 *>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else if constexpr (D / 32 == 4) {
    *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
  } else {
    *reinterpret_cast<float2 *>(dst) = make_float2(v[0], v[1]);
  }
}

// D / 32 consecutive values of packed row `rr`, rounded to the output type,
// into the staging rows at shared address `stage` (row pitch D * 2 bytes).
// A plain store, so the compiler may overlap it with the loads of other rows.
template <int D, bool kBf16>
__device__ __forceinline__ void stage_out_vec(uint8_t *smem, uint32_t stage, int rr, int col, const float *v) {
  uint8_t *dst = smem + (stage - smem_addr(smem)) + (rr * D + col) * 2;
  if constexpr (D / 32 == 8) {
    *reinterpret_cast<uint4 *>(dst) = make_uint4(pack2<kBf16>(v[0], v[1]), pack2<kBf16>(v[2], v[3]),
                                                 pack2<kBf16>(v[4], v[5]), pack2<kBf16>(v[6], v[7]));
  } else if constexpr (D / 32 == 4) {
    *reinterpret_cast<uint2 *>(dst) = make_uint2(pack2<kBf16>(v[0], v[1]), pack2<kBf16>(v[2], v[3]));
  } else {
    *reinterpret_cast<uint32_t *>(dst) = pack2<kBf16>(v[0], v[1]);
  }
}

// Bulk stores of `rows` staged output rows of a unit whose row's first
// packed query token is q0: the rows of one query position t are the
// consecutive heads h * G + g and so one contiguous run of
// out[q0 + t, :, :].  Issued by the calling lane.
template <int D>
__device__ __forceinline__ void store_out_rows(const DecodeArgs &a, int q0, int h, int rt, int rows,
                                               uint32_t stage) {
  const int es = a.out_f32 ? 4 : 2;  // bytes per output element
  int r = 0;
  while (r < rows) {
    const int m = rt * kRowsPerTile + r, t = m / a.G, g = m % a.G;
    const int r_end = min(rows, (t + 1) * a.G - rt * kRowsPerTile);
    uint8_t *dst = reinterpret_cast<uint8_t *>(a.out) + ((size_t)(q0 + t) * a.Hq + (size_t)h * a.G + g) * D * es;
    bulk_store(dst, stage + (uint32_t)(r * D * es), (uint32_t)((r_end - r) * D * es));
    r = r_end;
  }
}

// Output of a unit whose row sees no key at all (L_b = 0): O = 0, LSE = -inf.
// A tile past the row's queries (per-row query counts) has no output.
template <int D>
__device__ void write_empty_unit(const DecodeArgs &a, int unit, int lane) {
  const int rt = unit % a.RT, hr = unit / a.RT, h = hr % a.Hkv, b = hr / a.Hkv;
  int q0, qn;
  if (a.cu_q != nullptr) row_queries<true>(a, b, q0, qn);
  else row_queries<false>(a, b, q0, qn);
  if (rt >= row_tiles(a, qn)) return;  // the same for every lane
  const int rows = tile_rows(a, qn, rt);
  for (int i = lane; i < rows * D; i += 32) {
    const int rr = i / D, d = i % D;
    const int m = rt * kRowsPerTile + rr, t = m / a.G, g = m % a.G;
    const size_t e = ((size_t)(q0 + t) * a.Hq + (size_t)h * a.G + g) * D + d;
    if (a.out_f32) reinterpret_cast<float *>(a.out)[e] = 0.f;
    else reinterpret_cast<uint16_t *>(a.out)[e] = 0;  // +0 in fp16 and bf16
  }
  if (a.lse != nullptr) {
    for (int rr = lane; rr < rows; rr += 32) {
      const int m = rt * kRowsPerTile + rr, t = m / a.G, g = m % a.G;
      a.lse[lse_index(a, b, q0, h * a.G + g, t)] = -INFINITY;
    }
  }
  __syncwarp();
}

// Check the inputs of batch row b against the call's contract and record a
// breach: a length outside [0, max_seqlen_k] (the kernels clamp it into that
// range), and with per-row queries offsets that do not rise from 0 to
// total_q by steps of at most q_len (clamped likewise).  Every access stays
// inside the buffers either way; the record tells the caller that the
// result answers clamped inputs, not the ones passed.
__device__ __forceinline__ void check_row_inputs(const DecodeArgs &a, int b) {
  int bad = 0;
  const int L = a.seqlens[b];
  if (L < 0 || L > a.max_seqlen_k) bad |= kErrBadLen;
  if (a.cu_q != nullptr) {
    const int s = a.cu_q[b], e = a.cu_q[b + 1];
    if (e < s || (long long)e - s > a.q_len || (b == 0 && s != 0) || (b == a.B - 1 && e != a.total_q)) bad |= kErrBadOffsets;
  }
  if (bad) atomicOr(&g_mxa_err, bad);
}

// Room for partial rows in a landing zone that is a whole ring stage; its
// LSEs follow.
template <int D>
constexpr uint32_t stage_land_rows() { return (uint32_t)stage_bytes(D) - 16 * kRowsPerTile * 4; }

// Merge the n pieces of a split unit with the log-sum-exp identity,
// LSE = ln sum_i exp(lse_i) and O = sum_i exp(lse_i - LSE) O_i, in two
// passes.  The pieces' partial rows and LSEs are brought into a landing zone
// (`land`, with `land_rows` bytes for rows and then `lse_slots` pieces'
// LSEs) with bulk loads, as many pieces' rows at a time as fit; the LSEs of
// all pieces come with the first landing when there are at most `lse_slots`
// pieces (else each batch brings its own and the row statistics read them
// from global memory).
// First the row statistics, spread over a power-of-two group of lanes per
// row and reduced with a running maximum; then every lane accumulates its
// D / 32 columns of every row with the weights known up front, so the
// products are independent of one another and the loads overlap.  The
// pieces are the tail slot of the first CTA and the head slots of the
// following ones.  The caller has acquired their writes (the arrival
// count).  `own` >= 0 names a piece the caller has already placed in the
// landing zone (rows and LSEs at its index; then all n pieces fit one
// landing).  `coop`, for the unit of the CTA's last job, is where to post
// the second pass to the math warps, which then share it
// (merge_pass2_coop) when every piece fits one landing; `posted` tells the
// caller that it was posted.  Returns false if a bounded wait ran out.
template <int D, bool kBf16, int NR>
__device__ bool merge_pieces(const DecodeArgs &a, const SegmentDesc &sg, int rows, int unit, int lane,
                             uint8_t *smem, uint32_t ostage, uint32_t land, uint32_t land_rows,
                             uint32_t mbar, uint32_t &mk, int own, int lse_slots, FinalMerge *coop,
                             bool &posted) {
  constexpr int VEC = D / 32;
  constexpr float kLog2e = 1.4426950408889634f;
  const int n = sg.n_pieces, cf = sg.c_first;
  auto slot_of = [&](int i) -> size_t { return i == 0 ? (size_t)cf * 2 + 1 : (size_t)(cf + i) * 2; };
  const uint32_t pbytes = (uint32_t)rows * D * 4;
  const int cap = min(lse_slots, (int)(land_rows / pbytes));
  const bool all_lse = n <= lse_slots;  // every piece's LSEs come with the first landing
  auto issue = [&](int i0, int k) {  // bulk loads of pieces i0 .. i0 + k - 1
    fence_proxy_async_smem();  // earlier reads of the landing zone precede the new loads
    __syncwarp();
    const int l0 = all_lse ? 0 : i0, nl = all_lse ? (i0 == 0 ? n : 0) : k;
    if (lane == 0) {
      const int ko = (own >= i0 && own < i0 + k) ? 1 : 0, lo = (own >= l0 && own < l0 + nl) ? 1 : 0;
      mbar_arrive_expect_tx(mbar, (uint32_t)(k - ko) * pbytes + (uint32_t)(nl - lo) * kRowsPerTile * 4);
    }
    __syncwarp();
    // the lanes issue the copies together: rows of pieces first, then LSEs
    for (int c = lane; c < k + nl; c += 32) {
      if (c < k) {
        if (i0 + c != own)
          bulk_load(land + (uint32_t)c * pbytes, a.o_part + slot_of(i0 + c) * kRowsPerTile * D, pbytes, mbar);
      } else if (l0 + c - k != own) {
        const int p = c - k;
        bulk_load(land + land_rows + (uint32_t)p * kRowsPerTile * 4, a.lse_part + slot_of(l0 + p) * kRowsPerTile,
                  kRowsPerTile * 4, mbar);
      }
    }
    __syncwarp();
  };
  auto landed = [&]() {
    const bool ok = warp_wait_bounded(mbar, mk & 1, &g_mxa_err, kErrWaitFull, lane);
    ++mk;
    return ok;
  };
  if (lane == 0) fence_proxy_async_global();  // the acquired writes precede these async-proxy reads
  __syncwarp();
  issue(0, min(cap, n));

  const uint32_t sbase = smem_addr(smem);
  const float *land_o = reinterpret_cast<const float *>(smem + (land - sbase));
  const float *land_l = reinterpret_cast<const float *>(smem + (land + land_rows - sbase));

  // ---- pass 1: per-row maximum and sum of exponentials (base 2) ----
  const int lpr = rows > 8 ? 2 : rows > 4 ? 4 : rows > 2 ? 8 : rows > 1 ? 16 : 32;  // lanes per row
  const int r1 = lane / lpr, j1 = lane % lpr;
  float mx = -INFINITY, sm = 0.f;
  auto take_lse = [&](float l) {
    if (l == -INFINITY) return;  // an empty piece carries no weight
    const float mn = fmaxf(mx, l);
    sm = sm * ex2(mx - mn) + ex2(l - mn);
    mx = mn;
  };
  if (!all_lse && r1 < rows) {
#pragma unroll 4
    for (int p = j1; p < n; p += lpr)  // read at L2, past L1: written during this launch
      take_lse(__ldcg(a.lse_part + slot_of(p) * kRowsPerTile + r1) * kLog2e);
  }
  if (!landed()) return false;
  if (all_lse && r1 < rows) {
    for (int p = j1; p < n; p += lpr) take_lse(land_l[p * kRowsPerTile + r1] * kLog2e);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    if (o >= lpr) continue;
    const float mo = __shfl_xor_sync(0xffffffffu, mx, o);
    const float so = __shfl_xor_sync(0xffffffffu, sm, o);
    const float mn = fmaxf(mx, mo);
    sm = (mx == -INFINITY ? 0.f : sm * ex2(mx - mn)) + (mo == -INFINITY ? 0.f : so * ex2(mo - mn));
    mx = mn;
  }
  const float lse2 = sm > 0.f ? mx + log2f(sm) : -INFINITY;  // this row's LSE, base 2
  if (r1 < rows && j1 == 0 && a.lse != nullptr) {
    const int mrow = sg.rt * kRowsPerTile + r1, t = mrow / a.G, g = mrow % a.G;
    a.lse[lse_index(a, sg.b, sg.q0, sg.h * a.G + g, t)] = lse2 * kLn2;
  }
  if (coop != nullptr && all_lse && n <= cap && rows * D > 32 * 4) {
    // The CTA's final merge, with more (row, 4-column) items than one warp
    // has lanes: the math warps, idle by now, join the second pass.
    if (r1 < rows && j1 == 0) coop->lse2[r1] = lse2;
    __syncwarp();
    if (lane == 0) {
      coop->seg = sg;
      coop->rows = rows;
      coop->land = land;
      coop->land_rows = land_rows;
      coop->valid = 1;
      mbar_arrive(bar_addr(smem, D, B_FINAL));
    }
    __syncwarp();
    posted = true;
    merge_pass2_coop<D, kBf16>(a, coop, smem, kMathWarps, lane);
    if (lane == 0) a.counters[unit] = 0ull;  // every piece has arrived; leave it clean
    return true;
  }
  // With every LSE landed, the lanes that read a piece's LSE turn it into
  // its weight exp(lse_i - LSE) in place, once for all lanes.
  if (all_lse && r1 < rows) {
    float *lw = const_cast<float *>(land_l);
    for (int p = j1; p < n; p += lpr) {
      const float l = lw[p * kRowsPerTile + r1] * kLog2e;
      lw[p * kRowsPerTile + r1] = (l == -INFINITY || lse2 == -INFINITY) ? 0.f : ex2(l - lse2);
    }
  }
  __syncwarp();
  float row_lse[NR];
#pragma unroll
  for (int rr = 0; rr < NR; ++rr) row_lse[rr] = __shfl_sync(0xffffffffu, lse2, (rr * lpr) & 31);

  // ---- pass 2: O = sum_i w_i O_i with w_i = exp(lse_i - LSE) ----
  // All NR row slots (NR >= rows) are computed without branches so the
  // loads overlap; slots past `rows` read a valid row and are never stored.
  const int col = lane * VEC;
  float acc[NR][VEC];
#pragma unroll
  for (int rr = 0; rr < NR; ++rr)
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[rr][v] = 0.f;
  for (int i0 = 0; i0 < n; i0 += cap) {
    const int k = min(cap, n - i0);
    if (i0 > 0 && !landed()) return false;
    for (int p = 0; p < k; ++p) {
      const float *lp = land_l + (all_lse ? i0 + p : p) * kRowsPerTile;
      const float *op = land_o + p * rows * D + col;
#pragma unroll
      for (int rr = 0; rr < NR; ++rr) {
        const int rc = rr < rows ? rr : rows - 1;
        float w;
        if (all_lse) {
          w = lp[rr];  // already the weight
        } else {
          const float l = lp[rr] * kLog2e;
          w = l == -INFINITY ? 0.f : ex2(l - row_lse[rr]);
        }
        if constexpr (VEC == 8) {
          const float4 v = reinterpret_cast<const float4 *>(op + rc * D)[0];
          const float4 u = reinterpret_cast<const float4 *>(op + rc * D)[1];
          acc[rr][0] += w * v.x; acc[rr][1] += w * v.y; acc[rr][2] += w * v.z; acc[rr][3] += w * v.w;
          acc[rr][4] += w * u.x; acc[rr][5] += w * u.y; acc[rr][6] += w * u.z; acc[rr][7] += w * u.w;
        } else if constexpr (VEC == 4) {
          const float4 v = *reinterpret_cast<const float4 *>(op + rc * D);
          acc[rr][0] += w * v.x; acc[rr][1] += w * v.y; acc[rr][2] += w * v.z; acc[rr][3] += w * v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2 *>(op + rc * D);
          acc[rr][0] += w * v.x; acc[rr][1] += w * v.y;
        }
      }
    }
    if (i0 + cap < n) issue(i0 + cap, min(cap, n - i0 - cap));
  }
  __syncwarp();  // every lane is done with the landing zone, which may be the staging buffer
#pragma unroll
  for (int rr = 0; rr < NR; ++rr)
    if (rr < rows) {
      if (a.out_f32) stage_f32_vec<D>(smem, ostage, rr, col, acc[rr]);
      else stage_out_vec<D, kBf16>(smem, ostage, rr, col, acc[rr]);
    }
  fence_proxy_async_smem();  // staged rows are read by the bulk stores
  __syncwarp();
  if (lane == 0) {
    store_out_rows<D>(a, sg.q0, sg.h, sg.rt, rows, ostage);
    bulk_commit();
    a.counters[unit] = 0ull;  // every piece has arrived; leave it clean
  }
  return true;
}

// merge_pieces for the smallest power-of-two row count (2 to 16) >= rows.
template <int D, bool kBf16>
__device__ __forceinline__ bool merge_unit(const DecodeArgs &a, const SegmentDesc &sg, int rows, int unit,
                                           int lane, uint8_t *smem, uint32_t ostage, uint32_t land,
                                           uint32_t land_rows, uint32_t mbar, uint32_t &mk, int own,
                                           int lse_slots, FinalMerge *coop, bool &posted) {
  if (rows <= 2)
    return merge_pieces<D, kBf16, 2>(a, sg, rows, unit, lane, smem, ostage, land, land_rows, mbar, mk, own,
                                     lse_slots, coop, posted);
  if (rows <= 4)
    return merge_pieces<D, kBf16, 4>(a, sg, rows, unit, lane, smem, ostage, land, land_rows, mbar, mk, own,
                                     lse_slots, coop, posted);
  if (rows <= 8)
    return merge_pieces<D, kBf16, 8>(a, sg, rows, unit, lane, smem, ostage, land, land_rows, mbar, mk, own,
                                     lse_slots, coop, posted);
  return merge_pieces<D, kBf16, 16>(a, sg, rows, unit, lane, smem, ostage, land, land_rows, mbar, mk, own,
                                    lse_slots, coop, posted);
}

template <int D, bool kBf16>
__device__ void epilogue_warp(const DecodeArgs &a, uint8_t *smem, int lane) {
  constexpr int VEC = D / 32;
  constexpr int T = block_tokens(D);
  constexpr uint32_t KV_BYTES = (uint32_t)T * D * 2;
  constexpr float NEG_INF = -INFINITY;
  const uint32_t ring = smem_addr(smem + smem_ring_off());
  JobSlot *jobs = reinterpret_cast<JobSlot *>(smem + smem_jobs_off(D));
  const int HR = a.Hkv * a.RT;

  // Outputs and the workspace may still be in use by the kernel this launch
  // depends on (an earlier call on the same buffers).
  grid_dependency_wait();

  // Units of rows with L_b = 0 hold no KV block; one CTA per unit writes
  // their empty result.  The CTA of a row's first unit also checks the
  // row's inputs against the call's contract.
  if (a.schedule == MXA_SCHED_BALANCED) {
    for (int u = blockIdx.x; u < a.units; u += gridDim.x) {
      if (u % HR == 0 && lane == 0) check_row_inputs(a, u / HR);
      if (clamp_len((long long)a.seqlens[u / HR] + a.len_add, a.max_seqlen_k) == 0) write_empty_unit<D>(a, u, lane);
    }
  } else if (blockIdx.x % a.splits == 0) {
    const int u = blockIdx.x / a.splits;
    if (u % HR == 0 && lane == 0) check_row_inputs(a, u / HR);
    if (clamp_len((long long)a.seqlens[u / HR] + a.len_add, a.max_seqlen_k) == 0) write_empty_unit<D>(a, u, lane);
  }

  // Tag the arrival counters of this CTA's split units with this launch's
  // epoch (count 0), unless a piece in another CTA already did: every piece
  // of a unit does this before it can arrive, so arrivals are plain atomic
  // adds and a stale count (an earlier call's, or garbage) is never added
  // to.  A failed compare-and-swap means another CTA has tagged it.
  if (!warp_wait_bounded(bar_addr(smem, D, B_INIT), 0, &g_mxa_err, kErrWaitQ, lane)) return;
  if (lane == 0) {
    const int *init_units = reinterpret_cast<const int *>(smem + smem_bar_off(D) + kInitUnitsOff);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int u = init_units[i];
      if (u >= 0) {
        unsigned long long *cnt = a.counters + u;
        const unsigned long long cur = ld_relaxed_gpu_u64(cnt);
        if ((cur >> 32) != (unsigned long long)a.epoch) atomicCAS(cnt, cur, (unsigned long long)a.epoch << 32);
      }
    }
  }
  const int col = lane * VEC;
  const uint32_t ostage = smem_addr(smem + smem_out_off(D));
  const uint32_t oland = ostage;  // free again once this job's own rows have been stored
  const uint32_t merge_bar = bar_addr(smem, D, B_MERGE);
  uint32_t mk = 0;  // phases of the merge barrier used so far
  // The math warps wait, at the end of their work, to learn whether they
  // join the second pass of this CTA's final merge; tell them once.
  FinalMerge *fm = reinterpret_cast<FinalMerge *>(smem + smem_final_off(D));
  bool posted = false;
  auto post_none = [&]() {
    if (!posted && lane == 0) mbar_arrive(bar_addr(smem, D, B_FINAL));  // valid stays 0
    posted = true;
  };
  for (int jn = 0;; ++jn) {
    const int j = jn % kJobs, jk = jn / kJobs;
    // Leaving: bulk stores this warp issued must be done with shared memory
    // (and complete) before the CTA exits.
    if (!warp_wait_bounded(bar_addr(smem, D, B_JOBFULL(j)), jk & 1, &g_mxa_err, kErrWaitFull, lane)) {
      post_none();
      if (lane == 0) bulk_wait_all();
      return;
    }
    const SegmentDesc sg = jobs[j].seg;
    if (sg.kind < 0) {
      post_none();
      if (lane == 0) bulk_wait_all();
      return;
    }
    const int stage = jobs[j].stage;
    const uint32_t sbase = ring + (uint32_t)stage * (2 * KV_BYTES);
    // the staging rows are free once earlier bulk stores have read them
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
    const int rows = tile_rows(a, sg.qn, sg.rt);
    const int unit = (sg.b * a.Hkv + sg.h) * a.RT + sg.rt;
    const int slot = sg.kind - 1;  // partial slot (kind 1 -> head slot 0, kind 2 -> tail slot 1)
    // A piece of a split unit reads the unit's count now (acquire); the read
    // completes while this job is merged.  If every other piece has already
    // arrived, this piece merges the unit at once: it neither stores its
    // own partial nor counts itself.
    unsigned long long seen = 0;
    if (sg.kind != 0 && lane == 0) seen = ld_acquire_gpu_u64(a.counters + unit);

    // statistics of row `lane`: the four warps' (m, l) merged
    float wgt[kMathWarps];
    float my_lse = NEG_INF;
#pragma unroll
    for (int w = 0; w < kMathWarps; ++w) wgt[w] = 0.f;
    {
      const int row = lane < rows ? lane : 0;  // every lane computes; rows' lanes are used
      float mw[kMathWarps], lw[kMathWarps];
      float Mx = NEG_INF;
#pragma unroll
      for (int w = 0; w < kMathWarps; ++w) {
        mw[w] = jobs[j].ml[w][row][0];
        lw[w] = jobs[j].ml[w][row][1];
        Mx = fmaxf(Mx, mw[w]);
      }
      float Lx = 0.f;
#pragma unroll
      for (int w = 0; w < kMathWarps; ++w) {
        wgt[w] = mw[w] != NEG_INF ? ex2(mw[w] - Mx) : 0.f;
        Lx += wgt[w] * lw[w];
      }
      const float inv = Lx > 0.f ? 1.f / Lx : 0.f;
#pragma unroll
      for (int w = 0; w < kMathWarps; ++w) wgt[w] *= inv;
      my_lse = Lx > 0.f ? (Mx + log2f(Lx)) * kLn2 : NEG_INF;
    }
    // O of each row: the four warps' unnormalised partials, weighted.  A
    // warp whose weight is 0 left zeros (or finite values) in its slice, so
    // every load is made.  The NR row slots (the smallest power of two from
    // 2 to 16 that holds `rows`) are loaded before anything is staged and
    // without branches, so the loads overlap; slots past `rows` read a valid
    // row and are never stored.
    //
    // A split unit's landing zone is chosen meanwhile.  The CTA's last
    // segment uses the whole ring, which nothing loads into any more.
    // Otherwise a piece that will merge at once (every other piece has
    // arrived) and whose unit's rows do not fit the staging buffer keeps the
    // ring stage this job came in for the merge; all other pieces give the
    // stage straight back, so the ring stays full, and a piece that turns
    // out to be the last to arrive merges through the staging buffer, in as
    // many landings as needed.
    const float *hbase = reinterpret_cast<const float *>(smem + (sbase - smem_addr(smem)));
    const uint32_t pbytes = (uint32_t)rows * D * 4;
    const int own = (int)blockIdx.x - sg.c_first;  // this piece's index in the unit
    bool hold = false, merge_now = false;
    uint32_t land = oland, land_rows = (uint32_t)land_rows_bytes(D), dst_rows = ostage;
    int lse_slots = kRowsPerTile;
    auto merge_warps = [&](auto row_slots) {
      constexpr int NR = decltype(row_slots)::value;
      float acc[NR][VEC];
#pragma unroll
      for (int rr = 0; rr < NR; ++rr) {
        const int rc = rr < rows ? rr : rows - 1;
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[rr][v] = 0.f;
#pragma unroll
        for (int w = 0; w < kMathWarps; ++w) {
          const float wg = __shfl_sync(0xffffffffu, wgt[w], rr);
          const float *src = hbase + (handoff_addr<D>(sbase, w, rc, col) - sbase) / 4;
          if constexpr (VEC == 8) {  // two 16-byte chunks, each at its own swizzled place
            const float4 v = *reinterpret_cast<const float4 *>(src);
            const float4 u =
                *reinterpret_cast<const float4 *>(hbase + (handoff_addr<D>(sbase, w, rc, col + 4) - sbase) / 4);
            acc[rr][0] += wg * v.x; acc[rr][1] += wg * v.y; acc[rr][2] += wg * v.z; acc[rr][3] += wg * v.w;
            acc[rr][4] += wg * u.x; acc[rr][5] += wg * u.y; acc[rr][6] += wg * u.z; acc[rr][7] += wg * u.w;
          } else if constexpr (VEC == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(src);
            acc[rr][0] += wg * v.x; acc[rr][1] += wg * v.y; acc[rr][2] += wg * v.z; acc[rr][3] += wg * v.w;
          } else {
            const float2 v = *reinterpret_cast<const float2 *>(src);
            acc[rr][0] += wg * v.x; acc[rr][1] += wg * v.y;
          }
        }
      }
      seen = __shfl_sync(0xffffffffu, seen, 0);
      const bool all_here = sg.kind != 0 && (seen >> 32) == (unsigned long long)a.epoch &&
                            (int)(seen & 0xffffffffull) == sg.n_pieces - 1;
      hold = all_here && !sg.last && (uint32_t)sg.n_pieces * pbytes > (uint32_t)land_rows_bytes(D) &&
             sg.n_pieces <= min(kRowsPerTile, (int)(stage_land_rows<D>() / pbytes));
      land = sg.last ? ring : hold ? sbase : oland;
      land_rows = sg.last ? kStages * 2 * KV_BYTES - kRingLseSlots * kRowsPerTile * 4
                  : hold ? stage_land_rows<D>() : (uint32_t)land_rows_bytes(D);
      lse_slots = sg.last ? kRingLseSlots : kRowsPerTile;
      merge_now = all_here && sg.n_pieces <= min(lse_slots, (int)(land_rows / pbytes));
      __syncwarp();  // every lane has read the stage before it may become the landing zone
      dst_rows = merge_now ? land + (uint32_t)own * pbytes : ostage;
      // 16-bit output rows, or float32 rows (a partial result, or a float32 output)
      const bool rows16 = sg.kind == 0 && !a.out_f32;
#pragma unroll
      for (int rr = 0; rr < NR; ++rr) {
        if (rr < rows) {
          if (rows16) stage_out_vec<D, kBf16>(smem, ostage, rr, col, acc[rr]);
          else stage_f32_vec<D>(smem, dst_rows, rr, col, acc[rr]);
        }
      }
    };
    if (rows <= 2) merge_warps(std::integral_constant<int, 2>{});
    else if (rows <= 4) merge_warps(std::integral_constant<int, 4>{});
    else if (rows <= 8) merge_warps(std::integral_constant<int, 8>{});
    else merge_warps(std::integral_constant<int, 16>{});
    // row statistics: lane r < rows owns row r
    if (lane < rows) {
      if (sg.kind == 0) {
        const int m = sg.rt * kRowsPerTile + lane, t = m / a.G, g = m % a.G, hq = sg.h * a.G + g;
        if (a.lse != nullptr) a.lse[lse_index(a, sg.b, sg.q0, hq, t)] = my_lse;
      } else if (merge_now) {  // at this piece's index among the landed LSEs
        reinterpret_cast<float *>(smem + (land + land_rows - smem_addr(smem)))[own * kRowsPerTile + lane] = my_lse;
      } else {  // after the 16 staged rows; stored with them
        reinterpret_cast<float *>(smem + (ostage - smem_addr(smem)))[kRowsPerTile * D + lane] = my_lse;
      }
    }
    // Give the stage back to the producer and the hand-off slot to the math
    // warps.  This warp only read the stage; the math warps fenced their
    // generic writes to it before handing it over.  Then write the staged
    // rows out with bulk stores.
    fence_proxy_async_smem();  // staged rows are read by the bulk stores
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(bar_addr(smem, D, B_JOBEMPTY(j)));
      if (!hold) mbar_arrive_cnt(bar_addr(smem, D, B_EMPTY(stage)), kMathWarps);
      if (sg.kind == 0) {
        store_out_rows<D>(a, sg.q0, sg.h, sg.rt, rows, ostage);
      } else if (!merge_now) {
        const size_t ps = (size_t)blockIdx.x * 2 + slot;
        bulk_store(a.o_part + ps * kRowsPerTile * D, ostage, (uint32_t)(rows * D * 4));
        bulk_store(a.lse_part + ps * kRowsPerTile, ostage + (uint32_t)(kRowsPerTile * D * 4), kRowsPerTile * 4);
      }
      bulk_commit();
    }
    if (sg.kind != 0) {
      // A piece of a split unit: the last piece to arrive merges them all.
      // Count it with an acquire-release add: the release publishes this
      // piece's rows and LSEs (written by the async proxy, completed and
      // fenced first); the acquire lets the last piece read everyone's.
      bool ok = true;
      FinalMerge *coop = sg.last ? fm : nullptr;
      if (merge_now) {
        ok = merge_unit<D, kBf16>(a, sg, rows, unit, lane, smem, ostage, land, land_rows, merge_bar, mk, own,
                                    lse_slots, coop, posted);
      } else {
        unsigned long long old = 0;
        if (lane == 0) {
          bulk_wait_all();  // this piece's partial rows and LSEs are in global memory
          fence_proxy_async_global();
          old = atom_add_acq_rel_gpu_u64(a.counters + unit, 1ull);
        }
        old = __shfl_sync(0xffffffffu, old, 0);
        if ((int)(old & 0xffffffffull) + 1 == sg.n_pieces)
          ok = merge_unit<D, kBf16>(a, sg, rows, unit, lane, smem, ostage, land, land_rows, merge_bar, mk, -1,
                                      lse_slots, coop, posted);
      }
      if (hold) {
        fence_proxy_async_smem();  // reads of the landing zone precede the stage's next TMA loads
        __syncwarp();
        if (lane == 0) mbar_arrive_cnt(bar_addr(smem, D, B_EMPTY(stage)), kMathWarps);
      }
      if (!ok) {
        post_none();
        if (lane == 0) bulk_wait_all();
        return;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// The split kernel
// ---------------------------------------------------------------------------
template <int D, bool kBf16, bool kAppend, bool kVarlen>
__global__ void __launch_bounds__(kThreads, ctas_per_sm(D))
    mxa_split_kernel(const __grid_constant__ TmapPair tm, const __grid_constant__ DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((smem_addr(smem) & 1023u) != 0) {  // the 128-byte swizzle needs 1024-byte aligned stages
    if (tid == 0) atomicOr(&g_mxa_err, kErrAlign);
    return;
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_addr(smem, D, B_FULL(s)), 1);            // producer arrival + bytes
      mbar_init(bar_addr(smem, D, B_EMPTY(s)), kMathWarps);  // one arrival per math warp
    }
    mbar_init(bar_addr(smem, D, B_QFULL), 1);
    mbar_init(bar_addr(smem, D, B_QEMPTY), kMathWarps);
    for (int j = 0; j < kJobs; ++j) {
      mbar_init(bar_addr(smem, D, B_JOBFULL(j)), kMathWarps);
      mbar_init(bar_addr(smem, D, B_JOBEMPTY(j)), 1);
    }
    mbar_init(bar_addr(smem, D, B_MERGE), 1);
    mbar_init(bar_addr(smem, D, B_INIT), 1);
    mbar_init(bar_addr(smem, D, B_FINAL), 1);
    reinterpret_cast<FinalMerge *>(smem + smem_final_off(D))->valid = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // A dependent launch (the next call on this stream) may start its CTAs as
  // SM slots free up; it reads and writes global memory only after this
  // grid has completed (grid_dependency_wait in its producer and epilogue
  // warps).  The math warps touch shared memory only.
  grid_launch_dependents();
  if (warp == kProducerWarp) {
    producer_warp<D, kBf16, kAppend, kVarlen>(tm, a, smem, lane);
  } else if (warp == kEpilogueWarp) {
    epilogue_warp<D, kBf16>(a, smem, lane);
  } else {
    math_warps<D, kBf16>(a, smem, warp, lane);
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
      // the splits' loads are independent: keep several in flight
#pragma unroll 8
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

#include <atomic>
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

// 3-D map {D, Hkv, pool tokens} of a K or V pool; box {64 elements, 1 head,
// box_tokens tokens}, 128-byte swizzle, zero fill out of bounds.  L2 fills
// are promoted to whole rows of one head: 256 bytes for D >= 128 (the
// second 64-column box of a row then hits), 128 bytes for D = 64, whose
// 128-byte row a 256-byte fill would widen into the next head's row, read
// from DRAM a second time by the CTA of that head once L2 has let it go.
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
                   CU_TENSOR_MAP_SWIZZLE_128B,
                   D >= 128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The K and V maps of a call, from a small per-thread cache: a decode loop
// calls with the same cache buffers step after step, and encoding the two
// maps is a noticeable part of the host time of a short call.  The key is
// every input of the encoding, so a hit is always the map the call needs.
bool kv_maps(TmapPair *tm, const void *k, const void *v, int D, int Hkv, long long pool_tokens, int box_tokens,
             bool bf16) {
  struct Entry {
    const void *k, *v;
    long long pool_tokens;
    int D, Hkv, box_tokens;
    bool bf16, used;
    TmapPair tm;
  };
  constexpr int kEntries = 4;
  thread_local Entry cache[kEntries] = {};
  thread_local int next = 0;
  for (int i = 0; i < kEntries; ++i) {
    const Entry &e = cache[i];
    if (e.used && e.k == k && e.v == v && e.pool_tokens == pool_tokens && e.D == D && e.Hkv == Hkv &&
        e.box_tokens == box_tokens && e.bf16 == bf16) {
      *tm = e.tm;
      return true;
    }
  }
  if (!encode_kv_map(&tm->k, k, D, Hkv, pool_tokens, box_tokens, bf16) ||
      !encode_kv_map(&tm->v, v, D, Hkv, pool_tokens, box_tokens, bf16))
    return false;
  Entry &e = cache[next];
  next = (next + 1) % kEntries;
  e = Entry{k, v, pool_tokens, D, Hkv, box_tokens, bf16, true, *tm};
  return true;
}

template <int D, bool kBf16, bool kAppend, bool kVarlen>
cudaError_t prepare_split_kernel(int device) {
  static std::mutex mu;
  static bool done[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (device >= 0 && device < kMaxDevices && done[device]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(mxa_split_kernel<D, kBf16, kAppend, kVarlen>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_total(D));
  if (e == cudaSuccess && device >= 0 && device < kMaxDevices) done[device] = true;
  return e;
}

// Epoch of a launch: tags the arrival counters of split units (never 0).
uint32_t next_epoch() {
  static std::atomic<uint32_t> counter{0};
  uint32_t e = ++counter;
  if (e == 0) e = ++counter;
  return e;
}

template <int D, bool kBf16>
mxa_status_t launch_typed(const DecodeLaunch &L, cudaStream_t stream) {
  constexpr int T = block_tokens(D);
  const mxa_decode_params_t &p = L.p;
  const mxa_plan_t &plan = L.plan;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return MXA_ERR_CUDA;
  const bool append = L.len_add > 0, varlen = L.cu_q != nullptr;
  if (append && varlen) return MXA_ERR_UNSUPPORTED;
  const cudaError_t pe = append   ? prepare_split_kernel<D, kBf16, true, false>(device)
                         : varlen ? prepare_split_kernel<D, kBf16, false, true>(device)
                                  : prepare_split_kernel<D, kBf16, false, false>(device);
  if (pe != cudaSuccess) return MXA_ERR_CUDA;

  DecodeArgs a{};
  a.q = L.q;
  a.cu_q = L.cu_q;
  a.total_q = varlen ? L.total_q : p.B * p.q_len;
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
  a.num_pages = p.num_pages;
  a.mpps = p.max_pages_per_seq;
  a.max_seqlen_k = p.max_seqlen_k;
  a.box_tokens = a.contiguous ? T : (p.page_size % T == 0 ? T : p.page_size);
  a.scale_log2 = L.scale * 1.4426950408889634f;
  a.causal = L.causal;
  a.schedule = plan.schedule;
  a.splits = plan.num_splits;
  const int max_blocks = (p.max_seqlen_k + T - 1) / T;
  a.chunk_blocks = plan.schedule == MXA_SCHED_UNIFORM ? (max_blocks + plan.num_splits - 1) / plan.num_splits : 1;
  if (a.chunk_blocks < 1) a.chunk_blocks = 1;
  a.units = plan.units;
  a.unit_cost = plan.schedule == MXA_SCHED_BALANCED ? plan.unit_cost : 0;
  a.len_add = L.len_add;
  a.k_new = static_cast<const uint16_t *>(L.k_new);
  a.v_new = static_cast<const uint16_t *>(L.v_new);
  a.k_cache_w = static_cast<uint16_t *>(const_cast<void *>(L.k_cache));
  a.v_cache_w = static_cast<uint16_t *>(const_cast<void *>(L.v_cache));
  a.epoch = next_epoch();
  a.out_f32 = L.out_f32;
  if (plan.workspace_bytes > 0) {
    uint8_t *ws = static_cast<uint8_t *>(L.workspace);
    a.counters = reinterpret_cast<unsigned long long *>(ws);
    a.lse_part = reinterpret_cast<float *>(ws + ws_count_bytes(plan.units));
    a.o_part = reinterpret_cast<float *>(ws + ws_count_bytes(plan.units) + ws_lse_bytes(plan.grid));
  }

  TmapPair tm;
  const long long pool_tokens = (long long)(a.contiguous ? p.B : p.num_pages) * p.page_size;
  if (!kv_maps(&tm, L.k_cache, L.v_cache, D, p.Hkv, pool_tokens, a.box_tokens, kBf16)) return MXA_ERR_CUDA;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)plan.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_total(D);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = append   ? cudaLaunchKernelEx(&cfg, mxa_split_kernel<D, kBf16, true, false>, tm, a)
                        : varlen ? cudaLaunchKernelEx(&cfg, mxa_split_kernel<D, kBf16, false, true>, tm, a)
                                 : cudaLaunchKernelEx(&cfg, mxa_split_kernel<D, kBf16, false, false>, tm, a);
  if (e != cudaSuccess) return MXA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? MXA_OK : MXA_ERR_CUDA;
}

}  // namespace

mxa_status_t launch_decode(const DecodeLaunch &L, cudaStream_t stream) {
  const bool bf16 = L.p.dtype == MXA_BF16;
  if (L.p.D == 128) return bf16 ? launch_typed<128, true>(L, stream) : launch_typed<128, false>(L, stream);
  if (L.p.D == 64) return bf16 ? launch_typed<64, true>(L, stream) : launch_typed<64, false>(L, stream);
  if (L.p.D == 256) return bf16 ? launch_typed<256, true>(L, stream) : launch_typed<256, false>(L, stream);
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
