// kda_internal.h -- plan format and shared host/device definitions of libkda.so (internal).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

constexpr int kD = 128;      // head dim (Dk = Dv), fixed by the FlashKDA constraints
constexpr int kChunk = KDA_CHUNK;

// ---- plan: int32 header followed by one record per (sequence, value head) unit ----
// PH_SEG_CHUNKS > 0 selects the chunk-parallel (segmented) schedule: every unit's chunks are cut
// into segments of that many chunks, run as independent work items in three passes (segment
// summaries, a prefix combine of the segment start states, outputs).  PR_SEG_BASE is then the
// number of segments after the first over all earlier units (the unit's first state slot).
constexpr int32_t kPlanMagic = 0x4B444131;  // "KDA1"
constexpr int32_t kPlanVersion = 2;
constexpr int kPlanHeader = 16;
constexpr int kPlanRecord = 8;

enum PlanHeader : int {
  PH_MAGIC = 0, PH_VERSION, PH_HEADER_WORDS, PH_RECORD_WORDS, PH_UNITS, PH_LAYOUT, PH_B, PH_NQK,
  PH_NV, PH_S, PH_D, PH_TOTAL_CHUNKS, PH_MAX_CHUNKS, PH_NUM_SMS, PH_SEG_CHUNKS, PH_CHECKSUM
};
enum PlanRecord : int {
  PR_B = 0, PR_H, PR_HQ, PR_TOK_START, PR_LEN, PR_CHUNKS, PR_CHUNK_OFFSET, PR_SEG_BASE
};

// ---- segmented schedule: per state slot (a segment after a unit's first) three fp32 128x128
// matrices in the workspace after its header: M (the segment's state transition), R (its
// state from a zero start), and the segment's start state. ----
constexpr size_t kSlotFloats = (size_t)3 * kD * kD;
constexpr size_t kSlotBytes = kSlotFloats * 4;
enum SlotPart : int { SLOT_M = 0, SLOT_R = 1, SLOT_START = 2 };

// Segments of a unit with `chunks` chunks under segment length `seg` (>= 1).
inline int32_t unit_segments(int32_t chunks, int32_t seg) { return (chunks + seg - 1) / seg; }
// Work items of the two kernel passes of the segmented schedule, and state slots.
struct SegCounts {
  long long items_a, items_c, slots;
};
SegCounts seg_counts(const int32_t* plan);

// ---- workspace ----
constexpr size_t kWsHeaderBytes = 256;  // int32 status word at offset 0, item counter at 4
enum DeviceStatus : int32_t { DS_OK = 0, DS_PLAN = 1, DS_TIMEOUT = 2 };

// Per-chunk intermediates of the two-kernel path (fp32):
//   W [64][128], U [64][128], Qt [64][128], Kh [64][128], Aqk [64][64], gC [128]
constexpr size_t kWsW = 0;
constexpr size_t kWsU = kWsW + (size_t)kChunk * kD * 4;
constexpr size_t kWsQt = kWsU + (size_t)kChunk * kD * 4;
constexpr size_t kWsKh = kWsQt + (size_t)kChunk * kD * 4;
constexpr size_t kWsAqk = kWsKh + (size_t)kChunk * kD * 4;
constexpr size_t kWsGc = kWsAqk + (size_t)kChunk * kChunk * 4;
constexpr size_t kWsChunkBytes = kWsGc + (size_t)kD * 4 + 128 * 4;  // padded to 256 B
static_assert(kWsChunkBytes % 256 == 0, "chunk slots stay 256-byte aligned");

int32_t plan_checksum(const int32_t* plan, size_t n);

// Host-side validation shared by the entry points; returns KDA_OK or an error code.
kda_status_t validate_shape(const kda_shape_t* s);
kda_status_t validate_plan(const int32_t* plan, size_t n, const kda_shape_t* s);
// Workspace bytes of kda_forward for a validated plan.
size_t fused_workspace_bytes(const int32_t* plan);

}  // namespace kda
