// Tile and resource constants shared by the host planner and the kernels.
#pragma once

#include <stddef.h>

namespace mxa {

constexpr int kConsumerWarps = 4;                       // warps that do the math
constexpr int kThreads = 32 * (kConsumerWarps + 1);     // + one producer (TMA) warp
constexpr int kRowsPerTile = 16;                        // packed query rows per tile (mma M)
constexpr int kStages = 3;                              // depth of the K/V shared-memory ring
constexpr int kSmemPerSm = 228 * 1024;                  // B200 shared memory per SM
constexpr int kSmemReservedPerCta = 1024;               // driver-reserved shared memory per CTA
constexpr int kMaxThreadsPerSm = 2048;
constexpr int kMaxBalancedRows = 16384;                 // balanced schedule scans B rows in smem

// KV tokens per pipeline stage: every stage carries T x D elements of K and
// of V (16 KiB each in 16-bit types), so T = 8192 / D.
constexpr int block_tokens(int D) { return 8192 / D; }

constexpr size_t stage_bytes(int D) { return (size_t)2 * block_tokens(D) * D * 2; }
constexpr int q_row_pitch(int D) { return D * 2; }
constexpr size_t q_tile_bytes(int D) { return (size_t)kRowsPerTile * q_row_pitch(D); }
// fp32 scratch in which consumer warps 1..3 hand 8 rows of their output to warp 0
constexpr size_t merge_bytes(int D) { return (size_t)(kConsumerWarps - 1) * 8 * D * 4; }

struct SegmentDesc {
  int b, h, rt;          // batch row, KV head, row tile
  int blk_beg, blk_end;  // KV blocks [blk_beg, blk_end) of this unit
  int L;                 // valid keys of row b
  int kind;              // 0 = whole unit (final output), 1 = head partial (slot 0),
                         // 2 = tail partial (slot 1), -1 = end of work
  int pad;
};

constexpr size_t kBarrierBytes = 128;   // full[kStages], empty[kStages], qfull, qempty
constexpr size_t kDescBytes = sizeof(SegmentDesc);
constexpr size_t kMlBytes = (size_t)kConsumerWarps * kRowsPerTile * 2 * 4;

// Offsets inside the dynamic shared memory (base aligned to 1024 bytes).
constexpr size_t smem_ring_off() { return 0; }
constexpr size_t smem_q_off(int D) { return smem_ring_off() + kStages * stage_bytes(D); }
constexpr size_t smem_merge_off(int D) { return smem_q_off(D) + q_tile_bytes(D); }
constexpr size_t smem_ml_off(int D) { return smem_merge_off(D) + merge_bytes(D); }
constexpr size_t smem_desc_off(int D) { return smem_ml_off(D) + kMlBytes; }
constexpr size_t smem_bar_off(int D) { return smem_desc_off(D) + kDescBytes; }
constexpr size_t smem_total(int D) { return smem_bar_off(D) + kBarrierBytes; }

// Two CTAs per SM must fit: the ring, one Q tile, the merge scratch and the
// barriers of each, plus the driver's per-CTA reservation.

constexpr int ctas_per_sm(int D) {
  return (int)(kSmemPerSm / (smem_total(D) + kSmemReservedPerCta)) < (kMaxThreadsPerSm / kThreads)
             ? (int)(kSmemPerSm / (smem_total(D) + kSmemReservedPerCta))
             : (kMaxThreadsPerSm / kThreads);
}

// Workspace: per-unit merge metadata, then two partial slots per CTA.
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
inline size_t ws_meta_bytes(long units) { return align256((size_t)units * 8); }
inline size_t ws_lse_bytes(long grid) { return align256((size_t)grid * 2 * kRowsPerTile * 4); }
inline size_t ws_o_bytes(long grid, int D) { return align256((size_t)grid * 2 * kRowsPerTile * D * 4); }
inline size_t workspace_bytes(long units, long grid, int D) {
  return ws_meta_bytes(units) + ws_lse_bytes(grid) + ws_o_bytes(grid, D);
}

}  // namespace mxa

namespace mxa {
static_assert(2 * (smem_total(128) + kSmemReservedPerCta) <= (size_t)kSmemPerSm,
              "D = 128 layout must leave room for two CTAs per SM");
static_assert(2 * (smem_total(64) + kSmemReservedPerCta) <= (size_t)kSmemPerSm,
              "D = 64 layout must leave room for two CTAs per SM");
static_assert(smem_desc_off(128) % 16 == 0 && smem_bar_off(128) % 8 == 0, "alignment");
}  // namespace mxa
