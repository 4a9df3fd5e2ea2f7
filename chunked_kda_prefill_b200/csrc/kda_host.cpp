// kda_host.cpp -- host side of libkda.so: status strings, argument validation and the planner.
//
// The planner is the counterpart of flash_kda_metadata (FlashKDA README, 功能说明): an int32
// schedule computed from shapes, layout, valid lengths and the device's core count, reading no
// tensor values, reusable across calls with the same schedule.  The checks follow the FlashKDA
// README 约束说明 (D = 128, B >= 1, S > 0, 1 <= Nqk <= Nv with Nv % Nqk == 0, lower_bound in
// [-5, 0], TND cu_seqlens a strictly increasing prefix sum from 0 to T, BNSD/BSND valid lengths
// in [1, S]).  The Ascend-only capacity limit on Nv is not inherited.
#include <algorithm>
#include <cmath>
#include <climits>
#include <cstring>
#include <vector>

#include "kda_internal.h"

namespace kda {

int32_t plan_checksum(const int32_t* plan, size_t n) {
  uint32_t h = 2166136261u;
  for (size_t i = 0; i < n; ++i) {
    if (i == PH_CHECKSUM) continue;
    h = (h ^ (uint32_t)plan[i]) * 16777619u;
  }
  return (int32_t)(h & 0x7fffffff);
}

kda_status_t validate_shape(const kda_shape_t* s) {
  if (!s) return KDA_ERR_NULL;
  if (s->layout < KDA_LAYOUT_BNSD || s->layout > KDA_LAYOUT_TND) return KDA_ERR_LAYOUT;
  if (s->D != kD && s->D != 64) return KDA_ERR_DIM;
  if (s->B < 1 || s->S < 1) return KDA_ERR_SHAPE;
  if (s->Nqk < 1 || s->Nv < s->Nqk || s->Nv % s->Nqk != 0) return KDA_ERR_HEADS;
  // index ranges: units fit int32; every tensor's element count fits int64 comfortably
  const long long units = (long long)s->B * s->Nv;
  if (units > INT_MAX / 2) return KDA_ERR_SHAPE;
  const long long rows = (s->layout == KDA_LAYOUT_TND) ? (long long)s->S : (long long)s->B * s->S;
  if (rows * (long long)s->Nv * s->D > (1LL << 46)) return KDA_ERR_SHAPE;
  return KDA_OK;
}

SegCounts seg_counts(const int32_t* p) {
  SegCounts c{0, 0, 0};
  const int32_t seg = p[PH_SEG_CHUNKS];
  if (seg <= 0) return c;
  for (int u = 0; u < p[PH_UNITS]; ++u) {
    const int32_t nseg = unit_segments(p[kPlanHeader + u * kPlanRecord + PR_CHUNKS], seg);
    c.items_a += 2LL * nseg - 1;  // the first segment from the true state; R and M runs after
    c.items_c += nseg - 1;        // outputs of every segment after the first
  }
  c.slots = c.items_c;
  return c;
}

size_t fused_workspace_bytes(const int32_t* p) {
  return kWsHeaderBytes + (size_t)seg_counts(p).slots * kSlotBytes;
}

kda_status_t validate_plan(const int32_t* p, size_t n, const kda_shape_t* s) {
  if (!p) return KDA_ERR_NULL;
  if (n < (size_t)kPlanHeader) return KDA_ERR_PLAN;
  if (p[PH_MAGIC] != kPlanMagic || p[PH_VERSION] != kPlanVersion ||
      p[PH_HEADER_WORDS] != kPlanHeader || p[PH_RECORD_WORDS] != kPlanRecord)
    return KDA_ERR_PLAN;
  const long long need = kPlanHeader + (long long)p[PH_UNITS] * kPlanRecord;
  if (p[PH_UNITS] < 1 || (long long)n < need) return KDA_ERR_PLAN;
  if (plan_checksum(p, (size_t)need) != p[PH_CHECKSUM]) return KDA_ERR_PLAN;
  if (p[PH_SEG_CHUNKS] < 0) return KDA_ERR_PLAN;
  if (s) {
    if (p[PH_LAYOUT] != s->layout || p[PH_B] != s->B || p[PH_NQK] != s->Nqk ||
        p[PH_NV] != s->Nv || p[PH_S] != s->S || p[PH_D] != s->D ||
        (long long)p[PH_UNITS] != (long long)s->B * s->Nv)
      return KDA_ERR_PLAN;
  }
  return KDA_OK;
}

}  // namespace kda

using namespace kda;

extern "C" const char* kda_status_string(kda_status_t st) {
  switch (st) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_NULL: return "KDA_ERR_NULL: a required pointer is NULL";
    case KDA_ERR_LAYOUT: return "KDA_ERR_LAYOUT: layout must be BNSD, BSND or TND";
    case KDA_ERR_SHAPE: return "KDA_ERR_SHAPE: B and S must be >= 1 and sizes must fit";
    case KDA_ERR_HEADS: return "KDA_ERR_HEADS: need 1 <= Nqk <= Nv and Nv % Nqk == 0";
    case KDA_ERR_DIM: return "KDA_ERR_DIM: head dim D must be 64 or 128";
    case KDA_ERR_LOWER_BOUND:
      return "KDA_ERR_LOWER_BOUND: lower_bound must be in [-5, 0] and scale finite";
    case KDA_ERR_SEQLENS: return "KDA_ERR_SEQLENS: cu_seqlens malformed";
    case KDA_ERR_PLAN: return "KDA_ERR_PLAN: plan too small, corrupt or built for another shape";
    case KDA_ERR_ALIAS: return "KDA_ERR_ALIAS: output buffer overlaps an input";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace NULL, too small or misaligned";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: CUDA runtime or launch failure";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a bounded device-side wait gave up";
    case KDA_ERR_DEVICE: return "KDA_ERR_DEVICE: current device is not an sm_100 GPU";
    case KDA_ERR_ALIGN: return "KDA_ERR_ALIGN: tensor base pointers must be 16-byte aligned";
    case KDA_ERR_CAPACITY:
      return "KDA_ERR_CAPACITY: problem needs more scratch than kda_forward_noalloc's fixed "
             "KDA_NOALLOC_SCRATCH_BYTES; use kda_forward with a workspace";
  }
  return "KDA_ERR_UNKNOWN";
}

extern "C" kda_status_t kda_plan_size(const kda_shape_t* shape, size_t* n_int32) {
  if (!n_int32) return KDA_ERR_NULL;
  kda_status_t st = validate_shape(shape);
  if (st != KDA_OK) return st;
  *n_int32 = (size_t)kPlanHeader + (size_t)shape->B * shape->Nv * kPlanRecord;
  return KDA_OK;
}

namespace {

// The segment length the default schedule picks, from a cost model in units of one chunk's
// time on one SM (measured on B200: starting a work item costs about 0.9 chunk, one step of the
// segment start-state chain about 0.26).  With segments of n chunks, unit u has
// nseg_u = ceil(chunks_u / n); the first pass runs sum(2 nseg_u - 1) items and the last
// sum(nseg_u - 1), each in ceil(items / SMs) waves of n + 0.9; the chain takes
// max(nseg_u) - 2 steps.  Whole units take one wave of the longest unit.  Splitting is only
// considered when the units leave more than half the SMs idle (otherwise the extra passes
// cannot pay), and the cheapest n >= 2 is taken if it beats whole units.
int32_t auto_segment_chunks(const std::vector<int32_t>& chunks, int32_t num_sms) {
  const long long units = (long long)chunks.size();
  int32_t max_chunks = 0;
  for (int32_t c : chunks) max_chunks = std::max(max_chunks, c);
  if (units * 2 > num_sms || max_chunks < 4) return 0;
  constexpr double kItem = 0.9, kStep = 0.26;
  const double sms = (double)num_sms;
  double best = (double)max_chunks + kItem;  // whole units: one wave
  int32_t best_n = 0;
  for (int32_t n = 2; n < max_chunks; ++n) {
    long long items1 = 0, items3 = 0, max_seg = 0;
    for (int32_t c : chunks) {
      const long long nseg = (c + n - 1) / n;
      items1 += 2 * nseg - 1;
      items3 += nseg - 1;
      max_seg = std::max(max_seg, nseg);
    }
    const double wave = (double)n + kItem;
    const double t = std::ceil((double)items1 / sms) * wave +
                     std::ceil((double)items3 / sms) * wave +
                     (double)std::max(0LL, max_seg - 2) * kStep;
    if (t < best) {
      best = t;
      best_n = n;
    }
  }
  return best_n;
}

kda_status_t plan_impl(const kda_shape_t* shape, const int32_t* cu, int32_t num_sms,
                       int32_t seg_request, int32_t* plan, size_t n_int32) {
  kda_status_t st = validate_shape(shape);
  if (st != KDA_OK) return st;
  if (!plan) return KDA_ERR_NULL;
  if (num_sms < 1) return KDA_ERR_SHAPE;
  const size_t need = (size_t)kPlanHeader + (size_t)shape->B * shape->Nv * kPlanRecord;
  if (n_int32 < need) return KDA_ERR_PLAN;

  const int B = shape->B, Nv = shape->Nv, S = shape->S;
  std::vector<int32_t> len(B), start(B);
  if (shape->layout == KDA_LAYOUT_TND) {
    if (!cu) return KDA_ERR_SEQLENS;
    if (cu[0] != 0 || cu[B] != S) return KDA_ERR_SEQLENS;
    for (int b = 0; b < B; ++b) {
      if (cu[b + 1] <= cu[b]) return KDA_ERR_SEQLENS;
      len[b] = cu[b + 1] - cu[b];
      start[b] = cu[b];
    }
  } else {
    for (int b = 0; b < B; ++b) {
      if (cu) {
        if (cu[0] != 0) return KDA_ERR_SEQLENS;
        const long long L = (long long)cu[b + 1] - cu[b];
        if (L < 1 || L > S) return KDA_ERR_SEQLENS;
        len[b] = (int32_t)L;
      } else {
        len[b] = S;
      }
      start[b] = 0;
    }
  }

  struct Unit { int32_t b, h, L, chunks; };
  std::vector<Unit> units;
  units.reserve((size_t)B * Nv);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Nv; ++h)
      units.push_back({b, h, len[b], (len[b] + kChunk - 1) / kChunk});
  // longest first, ties in (b, h) order: the persistent scan takes units from the front
  std::stable_sort(units.begin(), units.end(),
                   [](const Unit& a, const Unit& c) { return a.chunks > c.chunks; });

  std::memset(plan, 0, need * sizeof(int32_t));
  long long total = 0;
  int32_t maxc = 0;
  const int G = Nv / shape->Nqk;
  for (size_t i = 0; i < units.size(); ++i) {
    int32_t* r = plan + kPlanHeader + i * kPlanRecord;
    r[PR_B] = units[i].b;
    r[PR_H] = units[i].h;
    r[PR_HQ] = units[i].h / G;
    r[PR_TOK_START] = start[units[i].b];
    r[PR_LEN] = units[i].L;
    r[PR_CHUNKS] = units[i].chunks;
    if (total > INT_MAX) return KDA_ERR_SHAPE;
    r[PR_CHUNK_OFFSET] = (int32_t)total;
    total += units[i].chunks;
    maxc = std::max(maxc, units[i].chunks);
  }
  if (total > INT_MAX) return KDA_ERR_SHAPE;
  // segment length: explicit request (> 0), none (0), or the default policy (< 0)
  std::vector<int32_t> unit_chunks(units.size());
  for (size_t i = 0; i < units.size(); ++i) unit_chunks[i] = units[i].chunks;
  const int32_t seg = seg_request >= 0 ? seg_request : auto_segment_chunks(unit_chunks, num_sms);
  long long seg_base = 0;
  for (size_t i = 0; i < units.size(); ++i) {
    int32_t* r = plan + kPlanHeader + i * kPlanRecord;
    r[PR_SEG_BASE] = (int32_t)seg_base;
    if (seg > 0) seg_base += unit_segments(units[i].chunks, seg) - 1;
    if (seg_base > INT_MAX / 4) return KDA_ERR_SHAPE;
  }
  plan[PH_SEG_CHUNKS] = seg;
  plan[PH_MAGIC] = kPlanMagic;
  plan[PH_VERSION] = kPlanVersion;
  plan[PH_HEADER_WORDS] = kPlanHeader;
  plan[PH_RECORD_WORDS] = kPlanRecord;
  plan[PH_UNITS] = (int32_t)units.size();
  plan[PH_LAYOUT] = shape->layout;
  plan[PH_B] = B;
  plan[PH_NQK] = shape->Nqk;
  plan[PH_NV] = Nv;
  plan[PH_S] = S;
  plan[PH_D] = shape->D;
  plan[PH_TOTAL_CHUNKS] = (int32_t)total;
  plan[PH_MAX_CHUNKS] = maxc;
  plan[PH_NUM_SMS] = num_sms;
  plan[PH_CHECKSUM] = plan_checksum(plan, need);
  return KDA_OK;
}

}  // namespace

extern "C" kda_status_t kda_plan(const kda_shape_t* shape, const int32_t* cu, int32_t num_sms,
                                 int32_t* plan, size_t n_int32) {
  return plan_impl(shape, cu, num_sms, -1, plan, n_int32);
}

extern "C" kda_status_t kda_plan_segmented(const kda_shape_t* shape, const int32_t* cu,
                                           int32_t num_sms, int32_t segment_chunks,
                                           int32_t* plan, size_t n_int32) {
  if (segment_chunks < 0) return KDA_ERR_SHAPE;
  return plan_impl(shape, cu, num_sms, segment_chunks, plan, n_int32);
}

extern "C" kda_status_t kda_workspace_size(const int32_t* plan, size_t n, size_t* bytes) {
  if (!bytes) return KDA_ERR_NULL;
  kda_status_t st = validate_plan(plan, n, nullptr);
  if (st != KDA_OK) return st;
  // the status word, plus the state slots of a segmented schedule
  *bytes = fused_workspace_bytes(plan);
  return KDA_OK;
}
