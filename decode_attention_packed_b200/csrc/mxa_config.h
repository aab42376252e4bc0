// Tile and resource constants shared by the host planner and the kernels.
#pragma once

#include <stddef.h>

namespace mxa {

constexpr int kMathWarps = 4;                           // warps that run QK^T / softmax / PV
constexpr int kProducerWarp = kMathWarps;               // TMA warp
constexpr int kEpilogueWarp = kMathWarps + 1;           // cross-warp merge and output warp
constexpr int kThreads = 32 * (kMathWarps + 2);
constexpr int kRowsPerTile = 16;                        // packed query rows per tile (mma M)
constexpr int kStages = 3;                              // depth of the K/V shared-memory ring
constexpr int kJobs = 2;                                // epilogue hand-off slots
constexpr int kSmemPerSm = 228 * 1024;                  // B200 shared memory per SM
constexpr int kSmemReservedPerCta = 1024;               // driver-reserved shared memory per CTA
constexpr int kMaxThreadsPerSm = 2048;
constexpr int kMaxBalancedRows = 12288;                 // balanced schedule scans B rows in smem
constexpr int kMaxUnitCost = 64;                       // blocks; unit_cost <= 4 x this

// Device-side failure record (bit flags), read back by mxa_device_error():
// bounded waits that ran out and a misaligned shared-memory base (reported
// as a timeout), and inputs that break the call's contract, which the kernel
// confines to the buffers and reports as an invalid argument: block-table
// entries outside the pool (read as zeros; appended tokens there not
// written), lengths outside [0, max_seqlen_k] (clamped into that range), and
// query offsets that do not run from 0 up to total_q by steps of at most
// q_len (clamped likewise).
enum : int {
  kErrWaitFull = 1, kErrWaitEmpty = 2, kErrWaitQ = 4, kErrAlign = 8, kErrDrain = 16, kErrBadPage = 32,
  kErrBadLen = 64, kErrBadOffsets = 128
};
constexpr int kErrInputMask = kErrBadPage | kErrBadLen | kErrBadOffsets;

// Fixed cost of a unit in the balanced schedule, in quarter KV blocks (the
// plan's unit_cost): the work a unit needs besides streaming its keys (the
// cross-warp merge, the output staging and stores, the arrival and merge of
// a split unit) grows with its packed query rows.  Measured on B200 (sweeps
// per workload): one 32 KiB block for one or two rows, a block and a half
// for three or four, one block per two rows above that (D <= 128); one
// 64 KiB block per four rows for D = 256.
constexpr int kUnitCostScale = 4;  // unit_cost counts quarter blocks
constexpr int unit_cost_for_rows(int rows, int D) {
  return D > 128 ? kUnitCostScale * (rows > 4 ? (rows + 3) / 4 : 1)
                 : (rows <= 2 ? kUnitCostScale : rows <= 4 ? kUnitCostScale * 3 / 2 : kUnitCostScale * ((rows + 1) / 2));
}
// ... and no more than 6 blocks of 32 KiB (3 of 64 KiB): a 16-row unit's
// fixed work measures at that once its merges are cheap.
constexpr int max_unit_cost(int D) { return kUnitCostScale * (D > 128 ? 3 : 6); }

// KV tokens per pipeline stage.  For D <= 128 every stage carries T x D
// elements of K and of V (16 KiB each in 16-bit types), so T = 8192 / D:
// three stages per CTA and two CTAs per SM keep 192 KiB of loads in flight
// per SM, which is what B200's HBM needs at its loaded latency of several
// microseconds; two CTAs also let one stream while the other starts up or
// finishes.  For D = 256 a stage is 64 keys (32 KiB of K and of V) and one
// CTA holds an SM: the same 192 KiB in flight, and the math warps keep the
// whole 256-column accumulator in registers (one CTA per SM leaves them 255
// registers a thread), each on 16 keys of a stage as for D = 128.
constexpr int block_tokens(int D) { return D <= 128 ? 8192 / D : 64; }

constexpr size_t stage_bytes(int D) { return (size_t)2 * block_tokens(D) * D * 2; }
constexpr int q_row_pitch(int D) { return D * 2; }
constexpr size_t q_tile_bytes(int D) { return (size_t)kRowsPerTile * q_row_pitch(D); }

// One unit of work for the math warps: a contiguous block range of one
// (batch row, KV head, row tile) unit.
struct SegmentDesc {
  int b, h, rt;          // batch row, KV head, row tile
  int blk_beg, blk_end;  // KV blocks [blk_beg, blk_end) of this unit
  int L;                 // valid keys of row b
  int kind;              // 0 = whole unit (final output), 1 = head piece (slot 0),
                         // 2 = tail piece (slot 1), -1 = end of work
  int c_first;           // first CTA holding a piece of the unit
  int n_pieces;          // CTAs holding pieces of the unit
  int last;              // 1 if no segment follows in this CTA
  int q0, qn;            // row b's first packed query token and its query count
};

// What the math warps hand to the epilogue warp at the end of a segment:
// the segment, the ring stage that holds their partial outputs, and each
// warp's running max and sum per packed row.
struct JobSlot {
  SegmentDesc seg;
  int stage;
  int pad[3];
  float ml[kMathWarps][kRowsPerTile][2];
};

// full[S], empty[S], qfull, qempty, job_full[J], job_empty[J], merge, init,
// final; then the two split units whose counters the CTA tags (2 ints)
constexpr size_t kBarrierBytes = 128;
constexpr int kNumBarriers = 2 * kStages + 2 + 2 * kJobs + 3;
constexpr size_t kInitUnitsOff = (size_t)kNumBarriers * 8;

// Offsets inside the dynamic shared memory (base aligned to 1024 bytes).
constexpr size_t smem_ring_off() { return 0; }
constexpr size_t smem_q_off(int D) { return smem_ring_off() + kStages * stage_bytes(D); }
constexpr size_t smem_desc_off(int D) { return smem_q_off(D) + q_tile_bytes(D); }
constexpr size_t smem_jobs_off(int D) { return smem_desc_off(D) + sizeof(SegmentDesc); }
// The epilogue warp's staging buffer, used in turn for the rows of a job's
// output before their bulk (TMA) stores (up to 16 rows x D fp32), and as the
// landing zone of the pieces of a split unit being merged (partial rows
// first, at least one whole 16-row piece, then the 16 row values of each of
// up to 16 pieces).
constexpr size_t land_rows_bytes(int D) {
  return (size_t)kRowsPerTile * D * 4 > 8 * 1024 ? (size_t)kRowsPerTile * D * 4 : 8 * 1024;
}
constexpr size_t out_stage_bytes(int D) { return land_rows_bytes(D) + 16 * kRowsPerTile * 4; }
constexpr size_t smem_out_off(int D) { return smem_jobs_off(D) + kJobs * sizeof(JobSlot); }
// The epilogue warp's note to the math warps about the CTA's final merge.
constexpr size_t kFinalBytes = 128;
constexpr size_t smem_final_off(int D) { return smem_out_off(D) + out_stage_bytes(D); }
constexpr size_t smem_bar_off(int D) { return smem_final_off(D) + kFinalBytes; }
constexpr size_t smem_total(int D) { return smem_bar_off(D) + kBarrierBytes; }

constexpr int ctas_per_sm(int D) {
  return (int)(kSmemPerSm / (smem_total(D) + kSmemReservedPerCta)) < (kMaxThreadsPerSm / kThreads)
             ? (int)(kSmemPerSm / (smem_total(D) + kSmemReservedPerCta))
             : (kMaxThreadsPerSm / kThreads);
}

// Workspace: per-unit arrival counters (epoch-tagged), then two partial
// slots (head piece, tail piece) per CTA.
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
inline size_t ws_count_bytes(long units) { return align256((size_t)units * 8); }
inline size_t ws_lse_bytes(long grid) { return align256((size_t)grid * 2 * kRowsPerTile * 4); }
inline size_t ws_o_bytes(long grid, int D) { return align256((size_t)grid * 2 * kRowsPerTile * D * 4); }
inline size_t workspace_bytes(long units, long grid, int D) {
  return ws_count_bytes(units) + ws_lse_bytes(grid) + ws_o_bytes(grid, D);
}

static_assert(kInitUnitsOff + 2 * sizeof(int) <= kBarrierBytes, "barrier area");
static_assert(sizeof(SegmentDesc) % 16 == 0 && sizeof(JobSlot) % 16 == 0, "alignment");
static_assert(2 * (smem_total(128) + kSmemReservedPerCta) <= (size_t)kSmemPerSm,
              "D = 128 layout must leave room for two CTAs per SM");
static_assert(2 * (smem_total(64) + kSmemReservedPerCta) <= (size_t)kSmemPerSm,
              "D = 64 layout must leave room for two CTAs per SM");
static_assert(smem_total(256) + kSmemReservedPerCta <= (size_t)kSmemPerSm && smem_total(256) <= 227 * 1024,
              "D = 256 layout must fit one CTA per SM");
static_assert(ctas_per_sm(64) == 2 && ctas_per_sm(128) == 2 && ctas_per_sm(256) == 1, "CTAs per SM");
static_assert((size_t)kMaxBalancedRows * 8 <= kStages * stage_bytes(64), "prologue scan fits the ring");

}  // namespace mxa
