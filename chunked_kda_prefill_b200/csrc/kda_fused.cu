// kda_fused.cu -- fused chunked KDA prefill for sm_100a: one persistent CTA of 16 warps per SM,
// one (sequence, value head) unit at a time, tcgen05 tensor cores for every contraction, the
// 128x128 fp32 state kept in TMEM for the whole sequence.
//
// Per 64-token chunk (the chunk equations of the FlashKDA README, 功能说明), eight phases:
//   1 prologue (CUDA cores): gate activation g = lb*sigmoid(e^A_log*(g_raw+dt_bias)) in log2
//     units, chunk-local cumulative sum G, q/k row L2-normalise, beta = sigmoid(logit); then the
//     bf16 operand tiles, each row factored through a reference row of its 16-row block so that
//     no factor overflows (the sub-chunk reference point b_gn of vLLM PR 43195's excerpt):
//       Aop = [k^ 2^(G-ref_I) ; scale q^ 2^(G-ref_I)],  B^(I) rows = k^ 2^(ref_I - G)  (s < 16(I+1)),
//       K~ = k^ 2^G, Q~ = scale q^ 2^G, K^ = k^ 2^(G_last - G)   (written over the raw q/k/g tiles)
//   2 MMA  D_I = Aop B^(I)^T, I = 0..3 (M=128, N=160 for all four blocks, K=128): rows 0-63 give
//     T = stril(diag(beta) K~ K-^T), rows 64-127 give Aqk = tril(Q~ K-^T); meanwhile K^ lo is
//     stored and the state left by the previous chunk becomes the bf16 hi/lo state operand
//   3 solve (fp32): X = (I+T)^-1 by 32x32 blocks (diagonal inverses by forward substitution in
//     registers, then the off-diagonal block by two 32x32x32 products on warp-level bf16 MMAs
//     with a three-term hi/lo split);
//     Xsol = X diag(beta) -> bf16 hi and lo parts stacked as one 128-row operand
//   4 MMA  W^T = K~^T [Xsol_hi; Xsol_lo]^T and U^T = V^T [Xsol_hi; Xsol_lo]^T (one N=128 chain
//          each, hi and lo parts side by side); S <- S Diag(2^G_last)
//     meanwhile.  Then -W -> bf16 hi and lo, stored token-major over the K~ and V tiles
//   5 MMA  [O^T | Da | Db] = S_hi [Q~ | -W_hi | -W_lo]^T (N=192) and [O^T | Da] += S_lo [Q~ | -W_hi]^T
//     (A operand = bf16 state in TMEM), Da and Db accumulating onto U's two parts; Delta^T = Da + Db
//   6 Delta^T -> bf16 hi and lo in TMEM
//   7 MMA  S += Delta^T K^ (hi/lo),  O^T += Delta^T Aqk^T   (then TMA for the chunk after next)
//   8 O^T -> bf16 out (TMA store); fp32 final_state after the item's last chunk
// Operands that feed the state recurrence (Xsol, W, S, Delta, K^) are split into bf16 hi + lo
// parts and multiplied as hi*hi + lo*hi + hi*lo, so the state path keeps ~16 significant bits
// instead of bf16's 8: without that, rounding errors pile up when the gate does not decay.
// A tcgen05 MMA costs about the same for every N up to 128, so operands are stacked along N
// wherever their products land in adjacent accumulator columns.
// TMA brings q/k/v/g of the next chunk into the other half of a two-slot ring while a chunk is
// processed.  Every wait is bounded; a time-out sets the workspace status to DS_TIMEOUT and the
// CTA drains its copies, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "kda_internal.h"
#include "kda_layout.cuh"
#include "kda_once.h"
#include "kda_sm100.cuh"
#include "kda_tmap.h"

namespace kda {

namespace {

using namespace sm100;

constexpr int kThreads = 512;

// The state operand of phase 5: a bf16 hi/lo pair (1, default) or the bf16 hi part alone (0: no
// lo conversion and 8 fewer MMAs per chunk, at a lower precision of W S^T and Q~ S^T; a variant
// for precision/speed experiments, built with -DKDA_STATE_LO=0).
#ifndef KDA_STATE_LO
#define KDA_STATE_LO 1
#endif
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kWaitLimit = 1u << 26;

// TMEM columns (512 allocated).  Lane = output row of every accumulator (dv for the state path).
constexpr uint32_t TC_S = 0;      // state S, fp32 [Dv lanes][Dk cols]
constexpr uint32_t TC_D = 128;    // phases 2-3: intra D_0..D_3 (160 cols)
constexpr uint32_t TC_W = 128;    // phase 4: W^T partial products, Xsol_hi part | Xsol_lo part
constexpr uint32_t TC_U = 256;    // phase 4: U^T partial products, Xsol_hi part | Xsol_lo part
constexpr uint32_t TC_O = 192;    // phases 5-8: O^T [Dv][64 tokens] (zeroed after phase 4)
constexpr uint32_t TC_DA = 256;   // phase 5: U_hi part + S_hi (-W_hi)^T + S_lo (-W_hi)^T
constexpr uint32_t TC_DB = 320;   // phase 5: U_lo part + S_hi (-W_lo)^T;  Delta^T = DA + DB
constexpr uint32_t TC_SHI = 384;  // bf16 state operand hi (64 cols = 128 bf16 per lane)
constexpr uint32_t TC_SLO = 448;  // bf16 state operand lo
constexpr uint32_t TC_DHI = 384;  // phases 6-7: bf16 Delta^T operand hi (32 cols), over TC_SHI
constexpr uint32_t TC_DLO = 416;  //              and its lo part

// Shared memory (offsets from a 1024-byte aligned base).  A ring slot holds one chunk's raw
// tiles as 64-row x 64-column atoms (8 KB, 128-byte swizzled):
//   q0 | g0 | v0 | q1 | g1 | v1 | k0 | k1      (x0 = columns 0-63, x1 = columns 64-127)
// so that after phase 4 the 192 rows [Q~ ; -W_hi ; -W_lo] of each column half are contiguous:
// one K-major N=192 operand for phase 5.
constexpr uint32_t SLOT_BYTES = 65536;
constexpr uint32_t OFF_Q = 0, OFF_G = 8192, OFF_V = 16384, OFF_K = 49152;
constexpr uint32_t QGV_ATOM = 24576;  // distance between the two column halves of q, g, v
constexpr uint32_t K_ATOM = 8192;
constexpr uint32_t SM_AOP = 131072;   // [128 rows][128] bf16, 2 atoms of 16 KB; after phase 2:
constexpr uint32_t SM_XSOL = SM_AOP;  //   [Xsol hi ; Xsol lo] 128 rows x 64 cols (16 KB)
constexpr uint32_t SM_BT = 163840;    // [B^(0); B^(1); B^(2); B^(3)]: one 160-row tile; the solve
constexpr uint32_t BT_ROWS = 160;     //   scratch in phase 3; from phase 5 the next chunk's
constexpr uint32_t SM_WTOT = SM_BT;   //   warp totals / prefixes fp32 [16][128] and
constexpr uint32_t SM_CST = SM_BT + 8192;  // reference constants fp32 [7][4 blocks][128]
constexpr uint32_t SM_KLO = 204800;   // K^ lo part [64][128] (phases 2-7); phase 8 until the
constexpr uint32_t SM_OSTG = SM_KLO;  //   next chunk's phase 2: the out tile for the TMA store
constexpr uint32_t SM_AQK = 221184;   // [64][64] bf16 (phases 3-7)
constexpr uint32_t SM_GC = 229376;    // fp32 [128]: 2^G_last
constexpr uint32_t SM_BETA = 229888;  // fp32 [64]
constexpr uint32_t SM_BAR = 230144;   // raw_full[2], mma, mma_u (the U MMAs of phase 4)
constexpr uint32_t SM_TSLOT = 230176;
constexpr uint32_t SM_FLAG = 230180;
constexpr uint32_t SM_PROD = 230184;  // the TMA producer's state (thread 0 only), 120 bytes
constexpr uint32_t SM_BAR_P1 = 230304;  // one arrival per warp once its phase-1 loads are done
constexpr uint32_t SM_END = 230312;
constexpr size_t kFusedSmemBytes = SM_END + 1024;

// per-(block, column) constants of the operand factorisation, indices into SM_CST
// (CST_NREF holds the reference row's cumulative gate negated, so that phase 1 adds it)
enum : int { CST_NREF = 0, CST_GE, CST_P2REF, CST_KFAC, CST_CDIAG, CST_C2, CST_C3, CST_N };

// Phase timestamps for performance analysis (CTA 0, thread 0, first 64 chunks), compiled in
// only for a profiling build (-DKDA_PHASE_TIMING=1): every thread would otherwise evaluate the
// check at each of the ~20 phase boundaries of every chunk.
#ifndef KDA_PHASE_TIMING
#define KDA_PHASE_TIMING 0
#endif
#if KDA_PHASE_TIMING
#define KDA_TS(slot_)                                                        \
  do {                                                                       \
    if (tprof_on) p.tprof[(size_t)gidx * 32 + (slot_)] = clock64();          \
  } while (0)
#else
#define KDA_TS(slot_) \
  do {                \
  } while (0)
#endif

__device__ __forceinline__ uint32_t dcol(int I) { return 8u * I * (I + 1); }

// Byte offset of element (row, col) of a 64-row tile stored as two 64-column atoms `atom` bytes
// apart (128-byte swizzle inside each atom).
__device__ __forceinline__ uint32_t atom_off(uint32_t atom, uint32_t row, uint32_t col) {
  return (col >> 6) * atom + row * 128u + ((((col & 63u) >> 3) ^ (row & 7u)) << 4) + (col & 7u) * 2u;
}

__device__ __forceinline__ bool plan_ok(const Params& p) {
  return p.plan[PH_MAGIC] == kPlanMagic && p.plan[PH_CHECKSUM] == p.plan_checksum &&
         p.plan[PH_UNITS] == p.n_units;
}

__device__ __forceinline__ void unpack4(const uint2 v, float (&f)[4]) {
  f[0] = __uint_as_float(v.x << 16);
  f[1] = __uint_as_float(v.x & 0xFFFF0000u);
  f[2] = __uint_as_float(v.y << 16);
  f[3] = __uint_as_float(v.y & 0xFFFF0000u);
}
__device__ __forceinline__ uint2 pack4(float a, float b, float c, float d) {
  return make_uint2(pack_bf16(a, b), pack_bf16(c, d));
}
// the two floats of a packed bf16 pair (low half = first element)
__device__ __forceinline__ float bf16_lo_of(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_of(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
// bf16 hi part of (a, b) packed, and the packed bf16 of the remainders (a, b) - hi
__device__ __forceinline__ uint32_t split_lo(float a, float b, uint32_t hi) {
  return pack_bf16(a - bf16_lo_of(hi), b - bf16_hi_of(hi));
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                    pack_bf16(f[6], f[7]));
}

// d += a b for one 16x8x16 tile on the warp-level tensor-core path (bf16 inputs, fp32 d), with the
// PTX fragment layouts, g = lane / 4 and t = lane % 4: a = A(g, 2t..2t+1), A(g+8, 2t..), A(g, 2t+8..),
// A(g+8, 2t+8..) (bf16 pairs, first element in the low half); b = B(2t..2t+1, g), B(2t+8..2t+9, g);
// d = D(g, 2t), D(g, 2t+1), D(g+8, 2t), D(g+8, 2t+1).
__device__ __forceinline__ void mma_bf16_m16n8k16(float (&d)[4], const uint32_t (&a)[4],
                                                  const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

struct Maps {
  CUtensorMap q, k, v, g, o;
};

// A work item: a range of chunks of one (sequence, value head) unit, the state it starts from
// and where its final state goes.  Mode 0 runs units whole.  Under a segmented plan, mode 1 runs
// per unit its first segment from the true initial state (outputs written) and, for every later
// segment s, an R run (from S = 0) and an M run (from S = I with v = 0) that leave the segment's
// affine map S -> S M_s + R_s in state slot s; mode 2 runs every later segment from its start
// state (computed in between by the combine kernel), writing outputs and the final state.
// Mode 3 (the summary of kda_forward_summary) runs every unit twice, item 2u from S = 0 (its
// final state is R, to p.sum_r) and item 2u + 1 from S = I with v = 0 (M, to p.sum_m), writing
// no outputs: the unit's affine map S -> S M + R over all its tokens.  Under a segmented plan
// it runs every segment's pair instead (segments after the first into the state slots), and
// kda_combine.cu composes them into the unit's maps.
struct Item {
  int b, h, hq, tok0, L;  // the sequence, its first packed row and its length
  int c_begin, c_end;     // chunks of the sequence this item runs
  int coff;               // the unit's chunk offset (debug dump)
  int ident;              // start from the identity (M run)
  const float* s_in;      // start state (null: zero; ignored for the identity)
  float* s_out;           // where the final state goes (null: nowhere)
  int write_out, zero_v, pad;  // write outputs; treat v as zero; zero-fill rows past L
};

__device__ __forceinline__ float* slot_ptr(const Params& p, int slot, int part) {
  return p.states + (size_t)slot * kSlotFloats + (size_t)part * kD * kD;
}

// Item i of this launch (every argument comes from the plan; see the Item comment).
template <int DIM, bool SUMMARY>
__device__ Item item_of(const Params& p, int i) {
  const int32_t* R = p.plan + kPlanHeader;
  const bool seg_summary = SUMMARY && p.seg_chunks > 0;  // mode 3 under a segmented plan
  int u = SUMMARY ? (i >> 1) : i;
  if ((!SUMMARY && p.mode != 0) || seg_summary) {
    // the unit whose item range holds i (item offsets increase along the plan)
    int lo = 0, hi = p.n_units - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      const int base = R[mid * kPlanRecord + PR_SEG_BASE];
      const int off = seg_summary ? 2 * (mid + base) : (p.mode == 1) ? mid + 2 * base : base;
      if (off <= i) lo = mid; else hi = mid - 1;
    }
    u = lo;
  }
  const int32_t* rec = R + u * kPlanRecord;
  Item it;
  it.b = rec[PR_B];
  it.h = rec[PR_H];
  it.hq = rec[PR_HQ];
  it.tok0 = rec[PR_TOK_START];
  it.L = rec[PR_LEN];
  it.coff = rec[PR_CHUNK_OFFSET];
  const int nch = rec[PR_CHUNKS];
  const size_t bh = ((size_t)it.b * p.Nv + it.h) * DIM * DIM;
  const float* s0 = p.S0 ? p.S0 + bh : nullptr;
  it.ident = 0;
  it.zero_v = 0;
  if (SUMMARY) {  // mode 3
    it.s_in = nullptr;
    it.write_out = 0;
    it.pad = 0;
    // whole units: item 2u + (0: R, 1: M).  Segmented plan: items 2 (u + base) + 2 s + (0, 1)
    // for every segment s of unit u; segment 0's maps go to sum_r / sum_m, later ones to the
    // state slots (base + s - 1), and the combine kernel composes them afterwards.
    int sgm = 0, c0 = 0, c1 = nch;
    if (seg_summary) {
      const int base = rec[PR_SEG_BASE];
      sgm = (i - 2 * (u + base)) >> 1;
      c0 = sgm * p.seg_chunks;
      c1 = min(nch, c0 + p.seg_chunks);
    }
    it.c_begin = c0;
    it.c_end = c1;
    const bool m_run = i & 1;
    if (m_run) {
      it.ident = 1;
      it.zero_v = 1;
    }
    if (sgm == 0) {
      it.s_out = (m_run ? p.sum_m : p.sum_r) + bh;
    } else {
      it.s_out = slot_ptr(p, rec[PR_SEG_BASE] + sgm - 1, m_run ? SLOT_M : SLOT_R);
    }
    return it;
  }
  if (p.mode == 0) {
    it.c_begin = 0;
    it.c_end = nch;
    it.s_in = s0;
    it.s_out = p.Sf + bh;
    it.write_out = 1;
    it.pad = 1;
    return it;
  }
  const int seg = p.seg_chunks, nseg = (nch + seg - 1) / seg;
  const int base = rec[PR_SEG_BASE];
  int sgm;
  if (p.mode == 1) {
    const int j = i - (u + 2 * base);
    sgm = (j + 1) >> 1;
    if (j == 0) {  // the first segment, from the true initial state
      it.s_in = s0;
      it.s_out = (nseg == 1) ? p.Sf + bh : slot_ptr(p, base, SLOT_START);
      it.write_out = 1;
      it.pad = (nseg == 1);
    } else {
      it.s_in = nullptr;
      it.write_out = 0;
      it.pad = 0;
      if (j & 1) {
        it.s_out = slot_ptr(p, base + sgm - 1, SLOT_R);
      } else {
        it.ident = 1;
        it.zero_v = 1;
        it.s_out = slot_ptr(p, base + sgm - 1, SLOT_M);
      }
    }
  } else {
    sgm = i - base + 1;
    it.s_in = slot_ptr(p, base + sgm - 1, SLOT_START);
    it.s_out = (sgm == nseg - 1) ? p.Sf + bh : nullptr;
    it.write_out = 1;
    it.pad = (sgm == nseg - 1);
  }
  it.c_begin = sgm * seg;
  it.c_end = min(nch, it.c_begin + seg);
  return it;
}

// The part of an item the TMA producer needs.
struct LoadRec {
  int b, h, hq, tok0, c_begin, c_end;
};
template <int DIM, bool SUMMARY>
__device__ __forceinline__ LoadRec load_rec(const Params& p, int i) {
  LoadRec r{0, 0, 0, 0, 0, 0};
  if (i < p.n_items) {
    const Item it = item_of<DIM, SUMMARY>(p, i);
    r = LoadRec{it.b, it.h, it.hq, it.tok0, it.c_begin, it.c_end};
  }
  return r;
}

// The load schedule, kept in shared memory: the cursor (next (item, chunk) of this CTA's stream,
// chunks planned so far, the current and next item, read one item ahead so no global load sits
// on the issue path), written by thread 0 only; the chunk whose tiles go out during the current
// chunk, which ten warps read to issue one TMA box each; and, in the dynamically scheduled
// instance, the CTA's item sequence.  There a CTA's first item is its blockIdx.x and thread 0
// claims each later one from the launch's item counter when its loads reach the item before
// (items go out in plan order, longest first, to whichever CTA frees up first); the consumer
// loop reads the sequence from a ring of four, as the loads run at most two chunks, so at most
// three items, ahead of it.  The other instances take every gridDim.x-th item.
struct Producer {
  int pu, pc;
  uint32_t issued;
  LoadRec cur, next;
  int ld_valid, ld_c, ld_slot;
  LoadRec ld_rec;
  int next_item, n_seq;
  int seq[4];
};
static_assert(sizeof(Producer) <= SM_BAR_P1 - SM_PROD, "producer state overflows its region");

// Tensor coordinates of chunk c of unit `ur` for the q/k maps (qc) and the v/g/out maps (vc).
__device__ __forceinline__ void chunk_coords(const Params& p, const LoadRec& ur, int c, int& qc1,
                                             int& qc2, int& vc1, int& vc2) {
  const int t = c * kChunk;
  if (p.layout == KDA_LAYOUT_BNSD) {
    qc1 = t; qc2 = ur.b * p.Nqk + ur.hq; vc1 = t; vc2 = ur.b * p.Nv + ur.h;
  } else {
    const int row = (p.layout == KDA_LAYOUT_BSND ? ur.b * p.S : ur.tok0) + t;
    qc1 = ur.hq; qc2 = row; vc1 = ur.h; vc2 = row;
  }
}

// TMA of one 64x64 box of chunk c into ring slot `slot`: box 0-1 q (column halves), 2-3 g,
// 4-5 v, 6-7 k.  Every box arrives on the slot's barrier with its own byte count, so the eight
// boxes can be issued by eight threads (a TMA issue occupies its thread for tens of cycles).
__device__ __forceinline__ void issue_box(const Params& p, const Maps& m, uint32_t sbase,
                                          const LoadRec& ur, int c, int slot, int box) {
  int qc1, qc2, vc1, vc2;
  chunk_coords(p, ur, c, qc1, qc2, vc1, vc2);
  const uint32_t bar = sbase + SM_BAR + 8u * slot;
  const uint32_t dst = sbase + slot * SLOT_BYTES;
  const int half = box & 1;
  mbar_arrive_expect_tx(bar, 8192);
  switch (box >> 1) {
    case 0: tma_load_3d(dst + OFF_Q + half * QGV_ATOM, &m.q, bar, 64 * half, qc1, qc2); break;
    case 1: tma_load_3d(dst + OFF_G + half * QGV_ATOM, &m.g, bar, 64 * half, vc1, vc2); break;
    case 2: tma_load_3d(dst + OFF_V + half * QGV_ATOM, &m.v, bar, 64 * half, vc1, vc2); break;
    default: tma_load_3d(dst + OFF_K + half * K_ATOM, &m.k, bar, 64 * half, qc1, qc2); break;
  }
}

}  // namespace

// DIM: the tensors' head dim (128, or 64 with the upper channels zero-filled); every tile,
// TMEM accumulator and MMA is 128 channels wide either way.  KIND: KIND_FORWARD (modes 0-2),
// KIND_SUMMARY (mode 3), or KIND_DEBUG (mode 0 that also dumps every chunk's intermediates to
// `dbg`; a separate instance, so the dump code takes no registers from the others).
// KIND_FORWARD_DYN: mode 0 with dynamic item claims, for plans whose units differ in length and
// outnumber the CTAs.
enum : int { KIND_FORWARD = 0, KIND_SUMMARY = 1, KIND_DEBUG = 2, KIND_FORWARD_DYN = 3 };
template <int DIM, int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    kda_fused_kernel(const Params p, const __grid_constant__ Maps maps, float* dbg) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, by an offset into the shared array itself (not through an integer
  // round trip) so that the compiler keeps every access below in the shared state space
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // K steps of 16 over the head dim in the MMAs that contract it (phases 2 and 5): at D = 64 the
  // upper channels are zero and their steps are skipped
  constexpr int kDimSteps = DIM / 16;
  const uint32_t wq = (uint32_t)(warp & 3) * 32u;  // TMEM lane quarter of this warp
  const uint32_t wlane = wq << 16;
  const int wg = warp >> 2;  // warpgroup 0..3: each covers all 128 TMEM lanes

  if (!plan_ok(p)) {
    if (tid == 0) atomicExch(p.status, DS_PLAN);
    return;
  }
  const uint32_t bar_mma = sbase + SM_BAR + 16;
  const uint32_t bar_mma_u = sbase + SM_BAR + 24;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + SM_FLAG);
  float* wtot = reinterpret_cast<float*>(sm + SM_WTOT);
  float* cst = reinterpret_cast<float*>(sm + SM_CST);
  float* gcs = reinterpret_cast<float*>(sm + SM_GC);
  float* beta_s = reinterpret_cast<float*>(sm + SM_BETA);

  if (tid == 0) {
    mbar_init(sbase + SM_BAR, 8);  // one arrival per TMA box of the slot
    mbar_init(sbase + SM_BAR + 8, 8);
    mbar_init(bar_mma, 1);
    mbar_init(bar_mma_u, 1);
    mbar_init(sbase + SM_BAR_P1, kThreads / 32);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(sbase + SM_TSLOT, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(sm + SM_TSLOT);
  const uint32_t tl = tbase + wlane;  // this warp's TMEM lane quarter

  const int G_stride = gridDim.x;
  int32_t* const item_counter = reinterpret_cast<int32_t*>(p.ws + 4);  // (dynamic instance)
  // Thread 0 issues every MMA and plans the loads; the TMA boxes are issued by other warps so no
  // thread carries more than one or two.  Per chunk c (ring slot s): during the phase-2 MMAs
  // thread 0 picks chunk c+2 (slot s again); lane 0 of warps 1-6 issue its q/g/v boxes in phase 7
  // (q/g/v of slot s are free once the phase-5 MMAs are done), lane 0 of warps 7-8 its k boxes in
  // phase 8 (after the phase-7 MMAs); lane 0 of warps 9-10 store chunk c's out tile after phase 8.
  Producer* prod = reinterpret_cast<Producer*>(sm + SM_PROD);
  auto plan_load = [&]() {  // thread 0
    Producer& pr = *prod;
    if (pr.pu >= p.n_items) {
      pr.ld_valid = 0;
      return;
    }
    pr.ld_valid = 1;
    pr.ld_rec = pr.cur;
    pr.ld_c = pr.pc;
    pr.ld_slot = pr.issued & 1;
    ++pr.issued;
    if (++pr.pc == pr.cur.c_end) {
      if constexpr (KIND == KIND_FORWARD_DYN) {
        pr.pu = pr.next_item;
        pr.cur = pr.next;
        pr.pc = pr.cur.c_begin;
        pr.next_item = (pr.pu < p.n_items) ? (G_stride + atomicAdd(item_counter, 1)) : p.n_items;
        pr.next = load_rec<DIM, false>(p, pr.next_item);
        pr.seq[pr.n_seq & 3] = pr.next_item;
        ++pr.n_seq;
      } else {
        pr.pu += G_stride;
        pr.cur = pr.next;
        pr.pc = pr.cur.c_begin;
        pr.next = load_rec<DIM, KIND == KIND_SUMMARY>(p, pr.pu + G_stride);
      }
    }
  };
  auto issue_planned = [&](int box) {
    const Producer& pr = *prod;
    if (pr.ld_valid) issue_box(p, maps, sbase, pr.ld_rec, pr.ld_c, pr.ld_slot, box);
  };
  const bool st_thread = lane == 0 && (warp == 9 || warp == 10);  // out-tile store issuers
  if (tid == 0) {
    prod->pu = blockIdx.x;
    prod->issued = 0;
    prod->cur = load_rec<DIM, KIND == KIND_SUMMARY>(p, blockIdx.x);
    prod->pc = prod->cur.c_begin;
    if constexpr (KIND == KIND_FORWARD_DYN) {
      prod->next_item = G_stride + atomicAdd(item_counter, 1);
      prod->next = load_rec<DIM, false>(p, prod->next_item);
      prod->seq[0] = blockIdx.x;
      prod->seq[1] = prod->next_item;
      prod->n_seq = 2;
    } else {
      prod->next = load_rec<DIM, KIND == KIND_SUMMARY>(p, blockIdx.x + G_stride);
    }
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.k);
    tma_prefetch_desc(&maps.v);
    tma_prefetch_desc(&maps.g);
    tma_prefetch_desc(&maps.o);
    for (int i = 0; i < 2; ++i) {  // chunks 0 and 1 of the stream
      plan_load();
      for (int box = 0; box < 8; ++box) issue_planned(box);
    }
    prod->ld_valid = 0;
  }
  if constexpr (KIND == KIND_FORWARD_DYN) __syncthreads();  // the sequence's first entries

  uint32_t gidx = 0;       // chunks consumed by this CTA
  uint32_t mma_phase = 0;    // parity of the next MMA-barrier completion
  uint32_t mma_u_phase = 0;  // and of the phase-4 U MMAs' barrier
  uint32_t p1_phase = 0;     // and of the phase-1 load barrier
  bool aborted = false;

  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(p.status, DS_TIMEOUT);
  };
  auto wait_mma = [&]() {
    if (!mbar_wait_bounded(bar_mma, mma_phase, kWaitLimit)) fail();
    mma_phase ^= 1u;
  };

  // phase-1 thread map: warp w owns rows 4w..4w+3 (16-row block w/4), lane owns columns 4l..4l+3
  const int r0 = 4 * warp, j0 = 4 * lane, Jb = warp >> 2;
  // Byte offset of (row r0 + i, columns j0..j0+3) inside a 64-column atom.  The 128-byte swizzle
  // depends only on the row mod 8, so the same offset serves every tile whose rows start at a
  // multiple of 8 (the slot tiles, Aop rows r and 64 + r, the B staircase blocks, K^ lo); a tile
  // adds its base and, for columns 64-127 (lanes 16-31), its atom stride.
  uint32_t io[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t r = (uint32_t)(r0 + i);
    io[i] = r * 128u + (((((uint32_t)j0 & 63u) >> 3) ^ (r & 7u)) << 4) + ((uint32_t)j0 & 7u) * 2u;
  }
  const uint32_t colhalf = (uint32_t)(j0 >> 6);

  for (int k_item = 0, ii = blockIdx.x; ii < p.n_items && !aborted;
       ++k_item, ii = (KIND == KIND_FORWARD_DYN) ? prod->seq[k_item & 3] : ii + G_stride) {
    const Item it = item_of<DIM, KIND == KIND_SUMMARY>(p, ii);
    const int b = it.b, h = it.h, tok0 = it.tok0, L = it.L, coff = it.coff;
    const float a_h = expf(p.A_log[h]);
    const float lbl2 = p.lower_bound * kLog2e;
    float dtb[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) dtb[e] = (j0 < DIM) ? p.dt_bias[h * DIM + j0 + e] : 0.f;

    // ---- start state (the item's: initial_state, a state slot, zeros or the identity):
    //      fp32 -> TMEM S, bf16 hi/lo -> TMEM state operand ----
    {
      const int i = wq + lane;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const int col0 = wg * 32 + half * 16;
        uint32_t fv[16], hi[8];
#if KDA_STATE_LO
        uint32_t lo[8];
#endif
#pragma unroll
        for (int c = 0; c < 16; c += 4) {
          float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
          if (it.ident) {
            const int d = i - (col0 + c);
            x = make_float4(d == 0 ? 1.f : 0.f, d == 1 ? 1.f : 0.f, d == 2 ? 1.f : 0.f,
                            d == 3 ? 1.f : 0.f);
          } else if (it.s_in && i < DIM && col0 + c < DIM) {
            x = *reinterpret_cast<const float4*>(it.s_in + (size_t)i * DIM + col0 + c);
          }
          fv[c] = __float_as_uint(x.x);
          fv[c + 1] = __float_as_uint(x.y);
          fv[c + 2] = __float_as_uint(x.z);
          fv[c + 3] = __float_as_uint(x.w);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float x0 = __uint_as_float(fv[2 * c]), x1 = __uint_as_float(fv[2 * c + 1]);
          hi[c] = pack_bf16(x0, x1);
#if KDA_STATE_LO
          lo[c] = split_lo(x0, x1, hi[c]);
#endif
        }
        tmem_st16(tl + TC_S + col0, fv);
        tmem_st8(tl + TC_SHI + col0 / 2, hi);
#if KDA_STATE_LO
        tmem_st8(tl + TC_SLO + col0 / 2, lo);
#endif
      }
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();

    // The front of phase 1 of chunk cc (ring slot of the gi-th chunk of this CTA): wait for its
    // tiles; gate activation and the in-thread cumsum of this thread's 4 rows (kept in registers
    // until that phase 1), warp totals -> wtot; beta.  For every chunk after an item's first it
    // runs under the previous chunk's phase-5 MMAs (warp 0 after issuing them; the wtot region is
    // free from then on).
    float4 gnext[4];  // this thread's rows of the next chunk's in-warp cumsums (front_gate -> phase 1)
    auto front_gate = [&](int cc, uint32_t gi, __nv_bfloat16 blog) {
      const int nn = min(kChunk, L - cc * kChunk);
      const uint8_t* sg_tile = sm + (gi & 1) * SLOT_BYTES + OFF_G;
      if (!mbar_wait_bounded(sbase + SM_BAR + 8u * (gi & 1), (gi >> 1) & 1u, kWaitLimit)) fail();
      // g_act * log2(e) = lb log2(e) / (1 + 2^(-log2(e) e^A_log (g_raw + dt_bias)))
      const float ca = -a_h * kLog2e;
      // this thread's rows 4 warp .. 4 warp + 3 and columns j0 .. j0 + 3 (the phase-1 map), kept in
      // registers until phase 1; the warp totals go to wtot for the column scan
      {
        const int grp = warp;
        float2 G[4][2];  // rows x column pairs (packed fp32x2 arithmetic)
        const float2 ca2 = make_float2(ca, ca), one2 = make_float2(1.f, 1.f);
        const float2 lb2 = make_float2(lbl2, lbl2);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = 4 * grp + i;
          // (row 4 grp + i has the swizzle of row r0 + i: grp and warp have the same parity)
          const int off = (int)(colhalf * QGV_ATOM + io[i]);
          const uint2 w = *reinterpret_cast<const uint2*>(sg_tile + off);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t wh = h ? w.y : w.x;
            const float2 x = __fmul2_rn(
                __fadd2_rn(make_float2(bf16_lo_of(wh), bf16_hi_of(wh)),
                           make_float2(dtb[2 * h], dtb[2 * h + 1])), ca2);
            const float2 den = __fadd2_rn(make_float2(ex2(x.x), ex2(x.y)), one2);
            const float2 sgm = __fmul2_rn(make_float2(__fdividef(1.0f, den.x),
                                                      __fdividef(1.0f, den.y)), lb2);
            G[i][h] = (r < nn) ? sgm : make_float2(0.f, 0.f);
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (i > 0) {
            G[i][0] = __fadd2_rn(G[i][0], G[i - 1][0]);
            G[i][1] = __fadd2_rn(G[i][1], G[i - 1][1]);
          }
          gnext[i] = make_float4(G[i][0].x, G[i][0].y, G[i][1].x, G[i][1].y);
        }
        *reinterpret_cast<float4*>(wtot + grp * kD + j0) =
            make_float4(G[3][0].x, G[3][0].y, G[3][1].x, G[3][1].y);
      }
      if (tid >= kChunk && tid < 2 * kChunk)  // (beta: threads 64-127, not warp 0)
        beta_s[tid - kChunk] =
            (tid - kChunk < nn) ? __fdividef(1.0f, 1.0f + __expf(-__bfloat162float(blog))) : 0.0f;
    };
    // Column j (threads 128-255, clear of the MMA-issuing warp 0): exclusive prefix of the 16
    // warp totals (in place); the block reference rows (G at rows 15, 31, 47, 63) and from them
    // the per-block constants of the factorisation; 2^G_last.  Runs under the previous chunk's
    // phase-7 MMAs (after an item's first chunk).
    auto front_scan = [&]() {
      if (tid < kD || tid >= 2 * kD) return;
      const int j = tid - kD;
      float run = 0.f, ref[4];
#pragma unroll
      for (int w2 = 0; w2 < 16; ++w2) {
        const float t = wtot[w2 * kD + j];
        wtot[w2 * kD + j] = run;
        run += t;
        if ((w2 & 3) == 3) ref[w2 >> 2] = run;
      }
#pragma unroll
      for (int I = 0; I < 4; ++I) {
        const float refI = (I == 0) ? 0.f : ref[I - 1];
        const float ge = ref[I];
        cst[(CST_NREF * 4 + I) * kD + j] = -refI;
        cst[(CST_GE * 4 + I) * kD + j] = ge;
        cst[(CST_P2REF * 4 + I) * kD + j] = ex2(refI);
        cst[(CST_KFAC * 4 + I) * kD + j] = ex2(ref[3] - ge);
        cst[(CST_CDIAG * 4 + I) * kD + j] = ex2(refI - ge);
        cst[(CST_C2 * 4 + I) * kD + j] = (I <= 1) ? ex2(ref[I + 1] - ge) : 0.f;
        cst[(CST_C3 * 4 + I) * kD + j] = (I == 0) ? ex2(ref[2] - ge) : 0.f;
      }
      gcs[j] = ex2(ref[3]);
    };

    // beta logits (row tid): the item's first chunk now, each later chunk one chunk ahead
    __nv_bfloat16 bl_next = __float2bfloat16_rn(0.f);
    const bool beta_thread = tid >= kChunk && tid < 2 * kChunk;  // row tid - 64
    {
      const int t = it.c_begin * kChunk + tid - kChunk;
      __nv_bfloat16 bl_first = __float2bfloat16_rn(0.f);
      if (beta_thread && t < L) bl_first = p.beta[beta_offset(p.layout, p.Nv, p.S, b, h, tok0, t)];
      if (beta_thread && t + kChunk < L)
        bl_next = p.beta[beta_offset(p.layout, p.Nv, p.S, b, h, tok0, t + kChunk)];
      front_gate(it.c_begin, gidx, bl_first);
      __syncthreads();
      front_scan();
      __syncthreads();
    }

    for (int c = it.c_begin; c < it.c_end; ++c, ++gidx) {
      const int slot = gidx & 1;
      uint8_t* sq = sm + slot * SLOT_BYTES;  // slot base: q, g, v atoms at QGV_ATOM, k at K_ATOM
      const uint32_t as = sbase + slot * SLOT_BYTES;
      const int t0 = c * kChunk;
      const int n = min(kChunk, L - t0);
      const bool last = (c == it.c_end - 1);
#if KDA_PHASE_TIMING
      const bool tprof_on = p.tprof && blockIdx.x == 0 && tid == 0 && gidx < 64;
#endif
      KDA_TS(0);

      // =================== phase 1: operand tiles ===================
      float G[4][4];
      float k4[CST_N][4];
      {
        // this thread's rows of G (in-warp cumsum + the warp prefix) and its block's constants
        const float4 pre = *reinterpret_cast<const float4*>(wtot + warp * kD + j0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 x = gnext[i];
          G[i][0] = x.x + pre.x;
          G[i][1] = x.y + pre.y;
          G[i][2] = x.z + pre.z;
          G[i][3] = x.w + pre.w;
        }
#pragma unroll
        for (int v = 0; v < CST_N; ++v) {
          const float4 x = *reinterpret_cast<const float4*>(cst + (v * 4 + Jb) * kD + j0);
          k4[v][0] = x.x;
          k4[v][1] = x.y;
          k4[v][2] = x.z;
          k4[v][3] = x.w;
        }
      }
      // wtot and the constants (in the B-tile region) are overwritten below by the staircase:
      // each warp reports its loads done, and every thread waits for all sixteen reports only
      // before its first store into that region
      __syncwarp();
      if (lane == 0) mbar_arrive(sbase + SM_BAR_P1);
      KDA_TS(12);
      uint2 khlo[4];  // K^ lo parts of this thread's rows, stored under the intra MMAs
      {
        float rqv[4], rkv[4];
        uint2 qwv[4], kwv[4];  // raw q/k words, kept for the operand pass
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float qv[4], kv[4];
          const bool valid = r0 + i < n;
          const uint2 zero2 = make_uint2(0u, 0u);
          const uint2 qw = *reinterpret_cast<const uint2*>(sq + OFF_Q + colhalf * QGV_ATOM + io[i]);
          const uint2 kw = *reinterpret_cast<const uint2*>(sq + OFF_K + colhalf * K_ATOM + io[i]);
          qwv[i] = valid ? qw : zero2;
          kwv[i] = valid ? kw : zero2;
          unpack4(qwv[i], qv);
          unpack4(kwv[i], kv);
          float ssq = 0.f, ssk = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            ssq = fmaf(qv[e], qv[e], ssq);
            ssk = fmaf(kv[e], kv[e], ssk);
          }
          rqv[i] = ssq;
          rkv[i] = ssk;
        }
        {
          // reduce-scatter the 8 partial sums over the warp, then broadcast the 8 totals
          const bool u16 = lane & 16, u8 = lane & 8, u4 = lane & 4;
          float w4[4], x2[2];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float send = u16 ? rqv[k] : rkv[k];
            const float keep = u16 ? rkv[k] : rqv[k];
            w4[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const float send = u8 ? w4[k] : w4[2 + k];
            const float keep = u8 ? w4[2 + k] : w4[k];
            x2[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
          }
          float y = (u4 ? x2[1] : x2[0]) + __shfl_xor_sync(0xffffffffu, u4 ? x2[0] : x2[1], 4);
          y += __shfl_xor_sync(0xffffffffu, y, 2);
          y += __shfl_xor_sync(0xffffffffu, y, 1);
          // lane l holds the total of value (l >> 2) & 7: index k + 2 (u8) + 4 (u16) of rq (0-3),
          // rk (4-7); it turns its total into the row's factor (q rows carry the scale), and the
          // eight factors are broadcast
          y = rsqrtf(y + 1e-6f) * (u16 ? 1.0f : p.scale);
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            rqv[m] = __shfl_sync(0xffffffffu, y, 4 * (m & 1) + 8 * (m >> 1));
            rkv[m] = __shfl_sync(0xffffffffu, y, 16 + 4 * (m & 1) + 8 * (m >> 1));
          }
        }
        // this thread's 4 rows x 4 columns as two fp32 pairs per row (packed fp32x2 arithmetic);
        // the staircase copies B^(Jb..3) of the warp's 16-row block Jb (warp-uniform)
        auto f2 = [](float a, float b) { return make_float2(a, b); };
        const float2 m1 = f2(-1.f, -1.f);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = r0 + i;
          const bool valid = r < n;
          const float rq = rqv[i], rk = rkv[i];
          const float2 rq2 = f2(rq, rq), rk2 = f2(rk, rk);
          uint32_t pa[2], pq[2], pqt[2], pkh[2], pkt[2], pb0[2], pb1[2], pb2[2], pb3[2], pkl[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t kw = h ? kwv[i].y : kwv[i].x, qw = h ? qwv[i].y : qwv[i].x;
            const float2 kv2 = f2(bf16_lo_of(kw), bf16_hi_of(kw));
            const float2 qv2 = f2(bf16_lo_of(qw), bf16_hi_of(qw));
            const float2 g2 = f2(G[i][2 * h], G[i][2 * h + 1]);
            const float2 kn = __fmul2_rn(kv2, rk2), qn = __fmul2_rn(qv2, rq2);
            const float2 da = __fadd2_rn(g2, f2(k4[CST_NREF][2 * h], k4[CST_NREF][2 * h + 1]));
            const float2 db = __ffma2_rn(g2, m1, f2(k4[CST_GE][2 * h], k4[CST_GE][2 * h + 1]));
            const float2 fA = f2(ex2(da.x), ex2(da.y));
            const float2 kbe = __fmul2_rn(kn, f2(ex2(db.x), ex2(db.y)));
            const float2 ka = __fmul2_rn(kn, fA), qa = __fmul2_rn(qn, fA);
            const float2 p2r = f2(k4[CST_P2REF][2 * h], k4[CST_P2REF][2 * h + 1]);
            const float2 kt = __fmul2_rn(ka, p2r), qt = __fmul2_rn(qa, p2r);
            const float2 kh = __fmul2_rn(kbe, f2(k4[CST_KFAC][2 * h], k4[CST_KFAC][2 * h + 1]));
            const float2 b0 = __fmul2_rn(kbe, f2(k4[CST_CDIAG][2 * h], k4[CST_CDIAG][2 * h + 1]));
            const float2 b2 = __fmul2_rn(kbe, f2(k4[CST_C2][2 * h], k4[CST_C2][2 * h + 1]));
            const float2 b3 = __fmul2_rn(kbe, f2(k4[CST_C3][2 * h], k4[CST_C3][2 * h + 1]));
            pa[h] = pack_bf16(ka.x, ka.y);
            pq[h] = pack_bf16(qa.x, qa.y);
            pqt[h] = pack_bf16(qt.x, qt.y);
            pkt[h] = pack_bf16(kt.x, kt.y);
            pkh[h] = pack_bf16(kh.x, kh.y);
            const float2 rem = __fadd2_rn(kh, f2(-bf16_lo_of(pkh[h]), -bf16_hi_of(pkh[h])));
            pkl[h] = pack_bf16(rem.x, rem.y);
            pb0[h] = pack_bf16(b0.x, b0.y);
            pb1[h] = pack_bf16(kbe.x, kbe.y);  // B^(Jb+1): reference row is this block's last row
            pb2[h] = pack_bf16(b2.x, b2.y);
            pb3[h] = pack_bf16(b3.x, b3.y);
          }
          khlo[i] = make_uint2(pkl[0], pkl[1]);
          if (i == 0 && !mbar_wait_bounded(sbase + SM_BAR_P1, p1_phase, kWaitLimit)) fail();
          uint8_t* aop = sm + SM_AOP + colhalf * 16384u + io[i];
          uint8_t* bst = sm + SM_BT + colhalf * (BT_ROWS * 128u) + io[i];
          *reinterpret_cast<uint2*>(aop) = make_uint2(pa[0], pa[1]);
          *reinterpret_cast<uint2*>(aop + 8192) = make_uint2(pq[0], pq[1]);
          *reinterpret_cast<uint2*>(sq + OFF_Q + colhalf * QGV_ATOM + io[i]) = make_uint2(pqt[0], pqt[1]);
          *reinterpret_cast<uint2*>(sq + OFF_K + colhalf * K_ATOM + io[i]) = make_uint2(pkh[0], pkh[1]);
          *reinterpret_cast<uint2*>(sq + OFF_G + colhalf * QGV_ATOM + io[i]) = make_uint2(pkt[0], pkt[1]);
          *reinterpret_cast<uint2*>(bst + dcol(Jb) * 128u) = make_uint2(pb0[0], pb0[1]);  // diagonal
          if (Jb + 1 <= 3)
            *reinterpret_cast<uint2*>(bst + dcol(Jb + 1) * 128u) = make_uint2(pb1[0], pb1[1]);
          if (Jb + 2 <= 3)
            *reinterpret_cast<uint2*>(bst + dcol(Jb + 2) * 128u) = make_uint2(pb2[0], pb2[1]);
          if (Jb + 3 <= 3)
            *reinterpret_cast<uint2*>(bst + dcol(Jb + 3) * 128u) = make_uint2(pb3[0], pb3[1]);
          if (!valid || it.zero_v)  // an M run treats v as zero
            *reinterpret_cast<uint2*>(sq + OFF_V + colhalf * QGV_ATOM + io[i]) = make_uint2(0, 0);
        }
      }
      p1_phase ^= 1u;
      if (st_thread) tma_store_wait_read();  // the previous out tile (in the K^ lo region) was read
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      KDA_TS(2);
      if (*abort_flag) {
        aborted = true;
        break;
      }

      // =================== phase 2: intra MMAs ===================
      if (tid == 0) {
        tc_fence_after();
        // D[:, 0:160] = Aop [B^(0); B^(1); B^(2); B^(3)]^T in one N=160 chain: D_I = cols dcol(I)..
        const uint32_t idesc = idesc_bf16(128, BT_ROWS, 0, 0);
#pragma unroll
        for (int kk = 0; kk < kDimSteps; ++kk) {
          const uint64_t ad = smem_desc(sbase + SM_AOP + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd =
              smem_desc(sbase + SM_BT + (kk >> 2) * (BT_ROWS * 128) + (kk & 3) * 32, 16, 1024);
          mma_ss(tbase + TC_D, ad, bd, idesc, kk > 0);
        }
        mma_commit(bar_mma);
        plan_load();  // the chunk after next, whose boxes go out in phases 7 and 8
      }
      // K^ lo for the phase-7 MMAs (its region's previous out tile was read by the end of phase 1)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<uint2*>(sm + SM_KLO + colhalf * 8192u + io[i]) = khlo[i];
      if (c > it.c_begin) {
        // the state after the previous chunk -> this chunk's bf16 hi/lo operand (phase 5), under
        // the intra MMAs.  16 state columns at a time; warp 0 issues the MMAs, so warps 8 and
        // 12 (its TMEM lanes) take its columns.  (D = 64: columns past D stay out of every
        // product, phase 5 skipping their K steps.)
        auto conv16_of = [&](int c16, const uint32_t (&v)[16]) {
          uint32_t hi[8];
#if KDA_STATE_LO
          uint32_t lo[8];
#endif
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float a0 = __uint_as_float(v[2 * e]), a1 = __uint_as_float(v[2 * e + 1]);
            hi[e] = pack_bf16(a0, a1);
#if KDA_STATE_LO
            lo[e] = split_lo(a0, a1, hi[e]);
#endif
          }
          tmem_st8(tl + TC_SHI + c16 / 2, hi);
#if KDA_STATE_LO
          tmem_st8(tl + TC_SLO + c16 / 2, lo);
#endif
        };
        auto conv16 = [&](int c16) {
          uint32_t v[16];
          tmem_ld16(tl + TC_S + c16, v);
          tmem_wait_ld();
          conv16_of(c16, v);
        };
        if (warp != 0 && wg * 32 < DIM) {
          uint32_t va[16], vb[16];
          tmem_ld16(tl + TC_S + wg * 32, va);
          tmem_ld16(tl + TC_S + wg * 32 + 16, vb);
          tmem_wait_ld();
          conv16_of(wg * 32, va);
          conv16_of(wg * 32 + 16, vb);
        }
        if (warp == 8) conv16(0);
        if (warp == 12) conv16(16);
        tmem_wait_st();
      }
      wait_mma();
      KDA_TS(3);
      tc_fence_after();

      // =================== phase 3: T, Aqk, solve ===================
      // X = (I + T)^-1 by 32x32 blocks, A = rows/columns 0-31 and B = 32-63:
      //   X_AA = (I + T_AA)^-1 and X_BB = (I + T_BB)^-1, one warp each, as soon as that warp has its
      //     rows of T: two 16x16 diagonal inverses by column forward substitution (a half-warp
      //     each, lane c computing column c in registers) and the block below them,
      //     X_10 = -P_1 (T_10 P_0), by two 16x16x16 products;
      //   X_BA = -X_BB (T_BA X_AA), two 32x32x32 products on warps 0-7 (one 16x8 output tile a
      //     warp, on the warp-level tensor-core path);
      // Xsol = X diag(beta) goes out in bf16 hi and lo parts, the diagonal blocks by warps 8-15
      // while the products run.
      constexpr int TP = 68;                              // row pitch of T and X (floats)
      constexpr int YP = 36;                              // row pitch of Y (floats)
      float* Ts = reinterpret_cast<float*>(sm + SM_BT);   // T = stril(diag(beta) K~ K-^T) [64][TP]
      float* Xs = Ts + 64 * TP;                           // X_AA and X_BB               [64][TP]
      float* Ys = reinterpret_cast<float*>(sm + SM_AOP + 16384);  // Y = T_BA X_AA     [32][YP]
      // (Xs ends inside the B-tile region; Ys lies in Aop's upper half, free after the intra MMA)
      {
        // TMEM lane quarter q4 = warp & 3 holds rows 32 (q4 & 1) .. +31 of k (q4 < 2) or q (q4 >= 2),
        // i.e. row blocks bA = 2 (q4 & 1) and bA + 1.  Items are (16-row block, 16-column chunk);
        // chunks right of a block's diagonal are zero.  q rows (Aqk): the quarter's 8 items, 2 a
        // warp.  k rows (T): T_AA's three chunks (0,0) (1,0) (1,1) go to warps 0, 4 and 8, and T_BB's
        // (2,2) (3,2) (3,3) to warps 1, 5 and 9, one each and first, so that warps 0 and 1 (the
        // diagonal inverses) wait only for one extraction; T_BA's four chunks go to warps 5, 9 and 13.
        const int q4 = warp & 3;
        const int r = (q4 & 1) * 32 + lane;
        const bool krow = q4 < 2;
        const float br = krow ? beta_s[r] : 0.f;
        const int bA = 2 * (q4 & 1);
        auto item_at = [&](int it, int& blk, int& ch) -> bool {
          if (krow) {
            if (it == 0 && wg < 3) {  // the diagonal block pair: (bA,bA) (bA+1,bA) (bA+1,bA+1)
              blk = bA + (wg > 0 ? 1 : 0);
              ch = bA + (wg == 2 ? 1 : 0);
              return true;
            }
            // T_BA: warp 5 (2,1); warp 9 (3,1); warp 13 (2,0) (3,0)
            blk = (wg == 3) ? 2 + it : wg + 1;
            ch = (wg == 3) ? 0 : 1;
            return q4 == 1 && wg >= 1 && (wg == 3 || it == 1);
          }
          const int item = 2 * wg + it;
          blk = bA + (item >> 2);
          ch = item & 3;
          return it < 2;
        };
        // an item's 16 columns of its block's rows -> T (fp32, scaled by beta) or Aqk (bf16),
        // strictly lower / lower parts; chunks right of the diagonal of an Aqk block are zeroed
        auto put = [&](int blk, int ch, const uint32_t (&v)[16]) {
          const bool mine = (r >> 4) == blk;
          if (!mine) return;
          if (ch > blk) {
            if (!krow) {
              *reinterpret_cast<uint4*>(sm + SM_AQK + sw128_offset(64, r, 16 * ch)) = make_uint4(0, 0, 0, 0);
              *reinterpret_cast<uint4*>(sm + SM_AQK + sw128_offset(64, r, 16 * ch + 8)) = make_uint4(0, 0, 0, 0);
            }
          } else if (krow) {
#pragma unroll
            for (int s0 = 0; s0 < 16; s0 += 4) {
              float f[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                f[e] = (16 * ch + s0 + e < r) ? br * __uint_as_float(v[s0 + e]) : 0.f;
              *reinterpret_cast<float4*>(Ts + r * TP + 16 * ch + s0) = make_float4(f[0], f[1], f[2], f[3]);
            }
          } else {
#pragma unroll
            for (int s0 = 0; s0 < 16; s0 += 8) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                f[e] = (16 * ch + s0 + e <= r) ? __uint_as_float(v[s0 + e]) : 0.f;
              *reinterpret_cast<uint4*>(sm + SM_AQK + sw128_offset(64, r, 16 * ch + s0)) = pack8(f);
            }
          }
        };
        {
          // the items' TMEM loads in one round trip (an item without data reads its quarter's
          // first chunk, unused)
          int blk[2], ch[2];
          bool has[2];
          uint32_t v0[16], v1[16];
#pragma unroll
          for (int it = 0; it < 2; ++it) {
            has[it] = item_at(it, blk[it], ch[it]);
            if (!has[it] || ch[it] > blk[it]) { blk[it] = has[it] ? blk[it] : bA; ch[it] = has[it] ? ch[it] : 0; }
          }
          KDA_TS(24);
          tmem_ld16(tl + TC_D + dcol(blk[0]) + 16 * (ch[0] <= blk[0] ? ch[0] : 0), v0);
          tmem_ld16(tl + TC_D + dcol(blk[1]) + 16 * (ch[1] <= blk[1] ? ch[1] : 0), v1);
          tmem_wait_ld();
          KDA_TS(23);
          if (has[0]) put(blk[0], ch[0], v0);
          // the second and third chunk of T_AA / T_BB are in Ts: tell warp 0 / 1
          if (krow && (wg == 1 || wg == 2)) named_bar_arrive(3 + q4, 96);
          if (has[1]) put(blk[1], ch[1], v1);
        }
        // warp 12 extracts nothing: Xsol's upper right 32x32 block is zero
        if (warp == 12) {
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int t = 32 * k4 + lane;  // 0..127
            const int row = t >> 2, cq = 32 + 8 * (t & 3);
            *reinterpret_cast<uint4*>(sm + SM_XSOL + sw128_offset(128, row, cq)) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(sm + SM_XSOL + sw128_offset(128, 64 + row, cq)) = make_uint4(0, 0, 0, 0);
          }
        }
      }
      // X_AA (warp 0) and X_BB (warp 1), each from its two 16x16 diagonal blocks: half-warp h
      // computes P_h = (I + T_hh)^-1 (lane c: column c, rows by forward substitution), then the
      // warp forms the block below the diagonal, X_10 = -P_1 (T_10 P_0)
      float* Ws = reinterpret_cast<float*>(sm + SM_AOP + 16384 + 32 * YP * 4);  // 2 x [16][20]
      KDA_TS(19);
      if (warp < 2) {
        named_bar_sync(3 + warp, 96);  // this warp's rows of T are in Ts (its chunk and warps 4/8's or 5/9's)
        const int h = lane >> 4, c = lane & 15, base = 32 * warp + 16 * h;
        {
          float x[16];
          x[0] = (c == 0) ? 1.f : 0.f;
#pragma unroll
          for (int rr = 1; rr < 16; ++rr) {
            const float* trow = Ts + (base + rr) * TP + base;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int s0 = 0; s0 < rr; s0 += 4) {
              const float4 t4 = *reinterpret_cast<const float4*>(trow + s0);
              if (s0 + 0 < rr) a0 = fmaf(t4.x, x[s0], a0);
              if (s0 + 1 < rr) a1 = fmaf(t4.y, x[s0 + 1], a1);
              if (s0 + 2 < rr) a0 = fmaf(t4.z, x[s0 + 2], a0);
              if (s0 + 3 < rr) a1 = fmaf(t4.w, x[s0 + 3], a1);
            }
            x[rr] = (rr == c) ? 1.f : -(a0 + a1);
          }
#pragma unroll
          for (int rr = 0; rr < 16; ++rr) Xs[(base + rr) * TP + base + c] = x[rr];
        }
        __syncwarp();
        KDA_TS(20);
        // 16x16x16 products by the warp: lane = (row i, column half jh), 8 columns each
        const int b0 = 32 * warp, i = lane & 15, jh = 8 * (lane >> 4);
        auto prod16 = [&](const float* Lrow, const float* R, int ldr, float2 (&acc)[4]) {
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[e] = make_float2(0.f, 0.f);
#pragma unroll
          for (int k0 = 0; k0 < 16; k0 += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(Lrow + k0);
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const float4 ra = *reinterpret_cast<const float4*>(R + (k0 + kk) * ldr + jh);
              const float4 rb = *reinterpret_cast<const float4*>(R + (k0 + kk) * ldr + jh + 4);
              const float2 l2 = make_float2(lv[kk], lv[kk]);
              acc[0] = __ffma2_rn(l2, make_float2(ra.x, ra.y), acc[0]);
              acc[1] = __ffma2_rn(l2, make_float2(ra.z, ra.w), acc[1]);
              acc[2] = __ffma2_rn(l2, make_float2(rb.x, rb.y), acc[2]);
              acc[3] = __ffma2_rn(l2, make_float2(rb.z, rb.w), acc[3]);
            }
          }
        };
        float2 acc[4];
        float* W = Ws + warp * 16 * 20;
        prod16(Ts + (b0 + 16 + i) * TP + b0, Xs + b0 * TP + b0, TP, acc);  // T_10 P_0
        *reinterpret_cast<float4*>(W + i * 20 + jh) = make_float4(acc[0].x, acc[0].y, acc[1].x, acc[1].y);
        *reinterpret_cast<float4*>(W + i * 20 + jh + 4) = make_float4(acc[2].x, acc[2].y, acc[3].x, acc[3].y);
        __syncwarp();
        KDA_TS(21);
        prod16(Xs + (b0 + 16 + i) * TP + b0 + 16, W, 20, acc);  // P_1 (T_10 P_0)
        float* xo = Xs + (b0 + 16 + i) * TP + b0 + jh;
        *reinterpret_cast<float4*>(xo) = make_float4(-acc[0].x, -acc[0].y, -acc[1].x, -acc[1].y);
        *reinterpret_cast<float4*>(xo + 4) = make_float4(-acc[2].x, -acc[2].y, -acc[3].x, -acc[3].y);
        // (the block above the diagonal, rows 0-15 x columns 16-31, is zero)
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(Xs + (b0 + i) * TP + b0 + 16 + jh) = z4;
        *reinterpret_cast<float4*>(Xs + (b0 + i) * TP + b0 + 16 + jh + 4) = z4;
        KDA_TS(22);
      }
      __syncthreads();
      KDA_TS(13);
      // Xsol row `row`, columns c0 .. c0 + 3 from x[4] (bf16 hi in rows 0-63, lo in 64-127)
      auto put_xsol4 = [&](int row, int c0, float x0, float x1, float x2, float x3) {
        const float4 b4 = *reinterpret_cast<const float4*>(beta_s + c0);
        const float f0 = x0 * b4.x, f1 = x1 * b4.y, f2 = x2 * b4.z, f3 = x3 * b4.w;
        const uint2 hi = pack4(f0, f1, f2, f3);
        const uint2 lo = make_uint2(split_lo(f0, f1, hi.x), split_lo(f2, f3, hi.y));
        *reinterpret_cast<uint2*>(sm + SM_XSOL + sw128_offset(128, row, c0)) = hi;
        *reinterpret_cast<uint2*>(sm + SM_XSOL + sw128_offset(128, 64 + row, c0)) = lo;
      };
      if (warp < 8) {
        // d = L R for the warp's 16x8 tile (rows 16 mt.., columns 8 nt..) of a 32x32x32 product,
        // on the warp-level tensor-core path (mma.sync m16n8k16, bf16).  Each operand is split
        // into a bf16 high part and a bf16 remainder and multiplied as lo*hi + hi*lo + hi*hi
        // (about 16 significant bits, as the Xsol operand these blocks become; fp32
        // accumulation).  This reads a small fraction of the shared-memory wavefronts of the
        // FFMA form, where every lane needs a whole row of L and a broadcast of R, and issues
        // half the instructions of the tf32 m16n8k8 form.
        const int mt = warp >> 2, nt = warp & 3, g = lane >> 2, t = lane & 3;
        auto tprod = [&](const float* L, int ldl, const float* R, int ldr, float (&d)[4]) {
          d[0] = d[1] = d[2] = d[3] = 0.f;
          float2 av[2][4];
          float bv[2][4];
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const int k0 = 16 * ks + 2 * t;
            av[ks][0] = *reinterpret_cast<const float2*>(L + g * ldl + k0);
            av[ks][1] = *reinterpret_cast<const float2*>(L + (g + 8) * ldl + k0);
            av[ks][2] = *reinterpret_cast<const float2*>(L + g * ldl + k0 + 8);
            av[ks][3] = *reinterpret_cast<const float2*>(L + (g + 8) * ldl + k0 + 8);
            bv[ks][0] = R[k0 * ldr + g];
            bv[ks][1] = R[(k0 + 1) * ldr + g];
            bv[ks][2] = R[(k0 + 8) * ldr + g];
            bv[ks][3] = R[(k0 + 9) * ldr + g];
          }
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            uint32_t ah[4], al[4], bh[2], bl[2];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              ah[e] = pack_bf16(av[ks][e].x, av[ks][e].y);
              al[e] = split_lo(av[ks][e].x, av[ks][e].y, ah[e]);
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              bh[e] = pack_bf16(bv[ks][2 * e], bv[ks][2 * e + 1]);
              bl[e] = split_lo(bv[ks][2 * e], bv[ks][2 * e + 1], bh[e]);
            }
            mma_bf16_m16n8k16(d, al, bh);
            mma_bf16_m16n8k16(d, ah, bl);
            mma_bf16_m16n8k16(d, ah, bh);
          }
        };
        float d[4];
        tprod(Ts + (32 + 16 * mt) * TP, TP, Xs + 8 * nt, TP, d);  // Y = T_BA X_AA
        const int yr = 16 * mt + g, yc = 8 * nt + 2 * t;
        *reinterpret_cast<float2*>(Ys + yr * YP + yc) = make_float2(d[0], d[1]);
        *reinterpret_cast<float2*>(Ys + (yr + 8) * YP + yc) = make_float2(d[2], d[3]);
        named_bar_sync(2, 256);
        KDA_TS(14);
        tprod(Xs + (32 + 16 * mt) * TP + 32, TP, Ys + 8 * nt, YP, d);  // X_BA = -X_BB Y
        // Xsol rows 32 + yr and 40 + yr, columns yc and yc + 1 (bf16 hi in rows 0-63, lo in 64-127)
        const float2 b2 = *reinterpret_cast<const float2*>(beta_s + yc);
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const float f0 = -d[2 * hr] * b2.x, f1 = -d[2 * hr + 1] * b2.y;
          const uint32_t hi = pack_bf16(f0, f1);
          const int row = 32 + yr + 8 * hr;
          *reinterpret_cast<uint32_t*>(sm + SM_XSOL + sw128_offset(128, row, yc)) = hi;
          *reinterpret_cast<uint32_t*>(sm + SM_XSOL + sw128_offset(128, 64 + row, yc)) =
              split_lo(f0, f1, hi);
        }
        KDA_TS(15);
      } else {
        // the diagonal blocks' Xsol: 2 blocks x 32 rows x 4 column octets, one item a thread
        const int t = tid - 256;
        const int base = 32 * (t >> 7), row = (t >> 2) & 31, cq = 8 * (t & 3);
        const float* xr = Xs + (base + row) * TP + base + cq;
        const float4 xa = *reinterpret_cast<const float4*>(xr);
        const float4 xb = *reinterpret_cast<const float4*>(xr + 4);
        put_xsol4(base + row, base + cq, xa.x, xa.y, xa.z, xa.w);
        put_xsol4(base + row, base + cq + 4, xb.x, xb.y, xb.z, xb.w);
      }
      KDA_TS(16);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      KDA_TS(4);

      // =================== phase 4: W^T and U^T;  S <- S Diag(2^G_last) ===================
      if (tid == 0) {
        tc_fence_after();
        // K~ and V are MN-major A operands (rows = tokens s, the two column halves QGV_ATOM apart)
        // (W and U alike: B = [Xsol_hi ; Xsol_lo], one N=128 operand; the two halves of each
        // product are summed later, W in its epilogue, U by the phase-5 accumulation)
        const uint32_t idesc_w = idesc_bf16(128, 128, 1, 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t aw = smem_desc(as + OFF_G + kk * 2048, QGV_ATOM, 1024);
          mma_ss(tbase + TC_W, aw, smem_desc(sbase + SM_XSOL + kk * 32, 16, 1024), idesc_w, kk > 0);
        }
        mma_commit(bar_mma);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t av = smem_desc(as + OFF_V + kk * 2048, QGV_ATOM, 1024);
          mma_ss(tbase + TC_U, av, smem_desc(sbase + SM_XSOL + kk * 32, 16, 1024), idesc_w, kk > 0);
        }
        mma_commit(bar_mma_u);  // the U MMAs are waited for only before -W lo overwrites V
      }
      {
        // the state decay for this chunk (the phase-5 MMAs read the bf16 copies, not TC_S); warp 0
        // issues the MMAs it overlaps, so warp 4 (same TMEM lanes) takes its columns as well
        auto decay = [&](int col) {
          uint32_t v[16], w2[16];
          tmem_ld16(tl + TC_S + col, v);
          tmem_ld16(tl + TC_S + col + 16, w2);
          tmem_wait_ld();
#pragma unroll
          for (int e4 = 0; e4 < 16; e4 += 4) {
            const float4 ga = *reinterpret_cast<const float4*>(gcs + col + e4);
            const float4 gb = *reinterpret_cast<const float4*>(gcs + col + 16 + e4);
            v[e4] = __float_as_uint(__uint_as_float(v[e4]) * ga.x);
            v[e4 + 1] = __float_as_uint(__uint_as_float(v[e4 + 1]) * ga.y);
            v[e4 + 2] = __float_as_uint(__uint_as_float(v[e4 + 2]) * ga.z);
            v[e4 + 3] = __float_as_uint(__uint_as_float(v[e4 + 3]) * ga.w);
            w2[e4] = __float_as_uint(__uint_as_float(w2[e4]) * gb.x);
            w2[e4 + 1] = __float_as_uint(__uint_as_float(w2[e4 + 1]) * gb.y);
            w2[e4 + 2] = __float_as_uint(__uint_as_float(w2[e4 + 2]) * gb.z);
            w2[e4 + 3] = __float_as_uint(__uint_as_float(w2[e4 + 3]) * gb.w);
          }
          tmem_st16(tl + TC_S + col, v);
          tmem_st16(tl + TC_S + col + 16, w2);
        };
        if (warp != 0 && wg * 32 < DIM) decay(wg * 32);  // (D = 64: columns past D unused)
        if (warp == 4) decay(0);
        tmem_wait_st();
      }
      wait_mma();
      KDA_TS(5);
      tc_fence_after();
      {
        // W row r (r = 16 wg .. 16 wg + 15) at lane j: -W -> bf16 hi over the K~ tile, lo over the
        // V tile, token-major [r][j] (the K-major layout of the phase-5 B operand).  Lanes j and
        // j ^ 1 swap one value per row pair, so each writes two adjacent columns of one row.
        const int j = wq + lane;
        const bool odd = lane & 1;
        uint32_t va[16], vb[16], wlo[8];
        tmem_ld16(tl + TC_W + 16 * wg, va);
        tmem_ld16(tl + TC_W + 64 + 16 * wg, vb);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float w0 = -(__uint_as_float(va[2 * q]) + __uint_as_float(vb[2 * q]));
          const float w1 = -(__uint_as_float(va[2 * q + 1]) + __uint_as_float(vb[2 * q + 1]));
          const float recv = __shfl_xor_sync(0xffffffffu, odd ? w0 : w1, 1);
          const float x0 = odd ? recv : w0, x1 = odd ? w1 : recv;  // columns j & ~1 and j | 1
          const int r = 16 * wg + 2 * q + (odd ? 1 : 0);
          const uint32_t off = atom_off(QGV_ATOM, r, j & ~1);
          const uint32_t hi = pack_bf16(x0, x1);
          wlo[q] = pack_bf16(x0 - bf16_lo_of(hi), x1 - bf16_hi_of(hi));
          *reinterpret_cast<uint32_t*>(sq + OFF_G + off) = hi;  // K~ was read by the W MMAs
        }
        // the lo parts go over V, which the U MMAs read: wait for them first
        if (!mbar_wait_bounded(bar_mma_u, mma_u_phase, kWaitLimit)) fail();
        mma_u_phase ^= 1u;
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int r = 16 * wg + 2 * q + (odd ? 1 : 0);
          *reinterpret_cast<uint32_t*>(sq + OFF_V + atom_off(QGV_ATOM, r, j & ~1)) = wlo[q];
        }
      }
      if (KIND == KIND_DEBUG && dbg && !it.zero_v) {
        // per-chunk intermediates in the two-kernel workspace layout (fp32)
        float* dc = dbg + (size_t)(coff + c) * (kWsChunkBytes / 4);
        const int i = wq + lane;
        if (wg == 0) {
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t wa[16], wb[16], ua[16], ub[16];
            tmem_ld16(tl + TC_W + 16 * ch, wa);
            tmem_ld16(tl + TC_W + 64 + 16 * ch, wb);
            tmem_ld16(tl + TC_U + 16 * ch, ua);
            tmem_ld16(tl + TC_U + 64 + 16 * ch, ub);
            tmem_wait_ld();
            for (int e = 0; e < 16; ++e) {
              dc[kWsW / 4 + (16 * ch + e) * kD + i] = __uint_as_float(wa[e]) + __uint_as_float(wb[e]);
              dc[kWsU / 4 + (16 * ch + e) * kD + i] = __uint_as_float(ua[e]) + __uint_as_float(ub[e]);
            }
          }
        }
        for (int e = tid; e < kChunk * kD; e += kThreads) {
          const int r = e / kD, j = e % kD;
          dc[kWsQt / 4 + e] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sq + OFF_Q + atom_off(QGV_ATOM, r, j)));
          dc[kWsKh / 4 + e] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sq + OFF_K + atom_off(K_ATOM, r, j)));
        }
        for (int e = tid; e < kChunk * kChunk; e += kThreads) {
          const int r = e / kChunk, s = e % kChunk;
          dc[kWsAqk / 4 + e] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + SM_AQK + sw128_offset(64, r, s)));
        }
        if (tid < kD) dc[kWsGc / 4 + tid] = gcs[tid];
        __syncthreads();  // every read of W's lo half is done before it is zeroed below
      }
      {
        // O^T accumulates from zero in phase 5 (its MMAs add to DA and DB, which hold U): clear
        // this thread's 16 columns of it, the W lo half this thread has read
        tmem_st16_zero(tl + TC_O + 16 * wg);
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      KDA_TS(6);

      // ============ phase 5: [O^T | Da | Db] = S [Q~ | -W_hi | -W_lo]^T ============
      if (tid == 0) {
        tc_fence_after();
        // B rows: Q~ (0-63), -W_hi (64-127), -W_lo (128-191): one K-major tile per column half
        const uint32_t idesc_3 = idesc_bf16(128, 192, 0, 0);
#pragma unroll
        for (int kk = 0; kk < kDimSteps; ++kk) {
          const uint64_t bd = smem_desc(as + (kk >> 2) * QGV_ATOM + (kk & 3) * 32, 16, 1024);
          mma_ts(tbase + TC_O, tbase + TC_SHI + kk * 8, bd, idesc_3, 1);
        }
#if KDA_STATE_LO
        const uint32_t idesc_2 = idesc_bf16(128, 128, 0, 0);
#pragma unroll
        for (int kk = 0; kk < kDimSteps; ++kk) {
          const uint64_t bd = smem_desc(as + (kk >> 2) * QGV_ATOM + (kk & 3) * 32, 16, 1024);
          mma_ts(tbase + TC_O, tbase + TC_SLO + kk * 8, bd, idesc_2, 1);
        }
#endif
        KDA_TS(26);
        mma_commit(bar_mma);
      }
      if (c + 1 < it.c_end) {
        // the next chunk's gate and cumsum under these MMAs, then its successor's beta load
        front_gate(c + 1, gidx + 1, bl_next);
        const int t2 = t0 + 2 * kChunk + tid - kChunk;
        if (c + 2 < it.c_end && beta_thread && t2 < L)
          bl_next = p.beta[beta_offset(p.layout, p.Nv, p.S, b, h, tok0, t2)];
      }
      wait_mma();
      KDA_TS(7);
      tc_fence_after();

      // =================== phase 6: Delta^T = Da + Db (U^T included) -> bf16 hi and lo ===================
      {
        // warpgroup wg converts tokens 16 wg .. 16 wg + 15
        uint32_t va[16], vb[16], hi[8], lo[8];
        tmem_ld16(tl + TC_DA + 16 * wg, va);
        tmem_ld16(tl + TC_DB + 16 * wg, vb);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float d0 = __uint_as_float(va[2 * e]) + __uint_as_float(vb[2 * e]);
          const float d1 = __uint_as_float(va[2 * e + 1]) + __uint_as_float(vb[2 * e + 1]);
          hi[e] = pack_bf16(d0, d1);
          lo[e] = split_lo(d0, d1, hi[e]);
        }
        tmem_st8(tl + TC_DHI + 8 * wg, hi);
        tmem_st8(tl + TC_DLO + 8 * wg, lo);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncthreads();
      KDA_TS(8);

      // =================== phase 7: S += Delta^T K^,  O^T += Delta^T Aqk^T ===================
      if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc_s = idesc_bf16(128, 128, 0, 1);
        const uint32_t idesc_o = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bk = smem_desc(as + OFF_K + kk * 2048, K_ATOM, 1024);
          mma_ts(tbase + TC_S, tbase + TC_DHI + kk * 8, bk, idesc_s, 1);
          mma_ts(tbase + TC_S, tbase + TC_DLO + kk * 8, bk, idesc_s, 1);
          mma_ts(tbase + TC_S, tbase + TC_DHI + kk * 8, smem_desc(sbase + SM_KLO + kk * 2048, 8192, 1024),
                 idesc_s, 1);
          mma_ts(tbase + TC_O, tbase + TC_DHI + kk * 8, smem_desc(sbase + SM_AQK + kk * 32, 16, 1024),
                 idesc_o, 1);
        }
        KDA_TS(25);
        mma_commit(bar_mma);
      }
      if (lane == 0 && warp >= 1 && warp <= 6) issue_planned(warp - 1);  // q/g/v of this slot are free
      if (c + 1 < it.c_end) front_scan();  // the next chunk's column scan under these MMAs
      wait_mma();
      KDA_TS(9);
      tc_fence_after();
      if (lane == 0 && (warp == 7 || warp == 8)) issue_planned(warp - 1);  // and now its k tile

      // =================== phase 8: out rows;  S -> bf16 operand (and final_state) ===================
      {
        const int i = wq + lane;
        const int col = wg * 32;
        uint32_t vo[16];
        tmem_ld16(tl + TC_O + 16 * wg, vo);
        tmem_wait_ld();
        if (!it.write_out) {
          // a segment-summary run: only its final state is kept
        } else if (n == kChunk) {
          // full chunk: out tile [t][i] (128B-swizzled, as the out tensor map expects) in the free
          // K^ lo region, stored by TMA after the phase-8 barrier
          // (lanes i and i ^ 1 swap one value per token pair and write two adjacent columns)
          const bool odd = lane & 1;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float o0 = __uint_as_float(vo[2 * q]), o1 = __uint_as_float(vo[2 * q + 1]);
            const float recv = __shfl_xor_sync(0xffffffffu, odd ? o0 : o1, 1);
            const int t = 16 * wg + 2 * q + (odd ? 1 : 0);
            *reinterpret_cast<uint32_t*>(sm + SM_OSTG + sw128_offset(64, t, i & ~1)) =
                odd ? pack_bf16(recv, o1) : pack_bf16(o0, recv);
          }
        } else {
          // the sequence's last, partial chunk: plain stores of the valid rows
          const int64_t ostride = (p.layout == KDA_LAYOUT_BNSD) ? DIM : (int64_t)p.Nv * DIM;
          __nv_bfloat16* orow = p.out + row_offset(p.layout, p.Nv, p.S, b, h, tok0, t0, DIM) + i;
          if (i < DIM) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int t = 16 * wg + e;
              if (t < n) orow[t * ostride] = __float2bfloat16_rn(__uint_as_float(vo[e]));
            }
          }
        }
        KDA_TS(18);
        // (the state's bf16 operand for the next chunk is made in that chunk's phase 2)
        if (last && it.s_out && i < DIM && col < DIM) {
          uint32_t v0[16], v1[16];
          tmem_ld16(tl + TC_S + col, v0);
          tmem_ld16(tl + TC_S + col + 16, v1);
          tmem_wait_ld();
          float* dst = it.s_out + (size_t)i * DIM + col;
#pragma unroll
          for (int e = 0; e < 16; e += 4) {
            *reinterpret_cast<float4*>(dst + e) = make_float4(
                __uint_as_float(v0[e]), __uint_as_float(v0[e + 1]), __uint_as_float(v0[e + 2]),
                __uint_as_float(v0[e + 3]));
            *reinterpret_cast<float4*>(dst + 16 + e) = make_float4(
                __uint_as_float(v1[e]), __uint_as_float(v1[e + 1]), __uint_as_float(v1[e + 2]),
                __uint_as_float(v1[e + 3]));
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      KDA_TS(10);
      if (st_thread && n == kChunk && it.write_out) {
        int qc1, qc2, oc1, oc2;
        const LoadRec ur{b, h, 0, tok0, 0, 0};
        chunk_coords(p, ur, c, qc1, qc2, oc1, oc2);
        const int half = warp - 9;
        if (64 * half < DIM) {  // (D = 64: the upper half is padding)
          tma_store_3d(&maps.o, sbase + SM_OSTG + half * 8192, 64 * half, oc1, oc2);
          tma_store_commit();
        }
      }
      if (*abort_flag) {
        aborted = true;
        break;
      }
    }
    // rows past the valid length (BNSD/BSND storage padding) are defined as zero
    if (!aborted && it.pad && p.layout != KDA_LAYOUT_TND) {
      const int per_row = DIM / 8;  // 16-byte stores per row
      for (int e = tid; e < (p.S - L) * per_row; e += kThreads) {
        const int t = L + e / per_row, q8 = (e % per_row) * 8;
        *reinterpret_cast<uint4*>(p.out + row_offset(p.layout, p.Nv, p.S, b, h, tok0, t, DIM) +
                                  q8) = make_uint4(0, 0, 0, 0);
      }
    }
  }

  // drain: loads still in flight must land, and stores complete, before this CTA exits
  if (st_thread) tma_store_wait_all();
  if (tid == 0) {
    while (gidx < prod->issued) {
      if (!mbar_wait_bounded(sbase + SM_BAR + 8u * (gidx & 1), (gidx >> 1) & 1u, kWaitLimit)) {
        atomicExch(p.status, DS_TIMEOUT);
        break;
      }
      ++gidx;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

namespace {

// D = 64: the kernel still loads two 64-column boxes per tile; the second lies wholly past the
// tensor's D columns and reads as zeros, so the upper 64 channels of q, k, v, g are zero.
bool make_map(CUtensorMap* m, const void* base, int layout, int B, int NX, int S, int D) {
  uint64_t dims[3], strides[2];
  uint32_t box[3];
  if (layout == KDA_LAYOUT_BNSD) {
    dims[0] = (uint64_t)D; dims[1] = (uint64_t)S; dims[2] = (uint64_t)B * NX;
    strides[0] = (uint64_t)D * 2; strides[1] = (uint64_t)S * D * 2;
    box[0] = 64; box[1] = 64; box[2] = 1;
  } else {
    const uint64_t rows = (layout == KDA_LAYOUT_BSND) ? (uint64_t)B * S : (uint64_t)S;
    dims[0] = (uint64_t)D; dims[1] = (uint64_t)NX; dims[2] = rows;
    strides[0] = (uint64_t)D * 2; strides[1] = (uint64_t)NX * D * 2;
    box[0] = 64; box[1] = 1; box[2] = 64;
  }
  return encode_bf16_3d(m, base, dims, strides, box);
}

}  // namespace

cudaError_t launch_fused(const Params& p, float* dbg, cudaStream_t stream, bool dyn_items) {
  static PerDevice setup;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int num_sms = 0;
  e = once_per_device(setup, dev, &num_sms, [](int d, int* sms) {
    const void* fns[] = {(const void*)kda_fused_kernel<kD, KIND_FORWARD>,
                         (const void*)kda_fused_kernel<64, KIND_FORWARD>,
                         (const void*)kda_fused_kernel<kD, KIND_FORWARD_DYN>,
                         (const void*)kda_fused_kernel<64, KIND_FORWARD_DYN>,
                         (const void*)kda_fused_kernel<kD, KIND_SUMMARY>,
                         (const void*)kda_fused_kernel<64, KIND_SUMMARY>,
                         (const void*)kda_fused_kernel<kD, KIND_DEBUG>,
                         (const void*)kda_fused_kernel<64, KIND_DEBUG>};
    for (const void* f : fns) {
      const cudaError_t r = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)kFusedSmemBytes);
      if (r != cudaSuccess) return r;
    }
    return cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, d);
  });
  if (e != cudaSuccess) return e;
  if (num_sms < 1) return cudaErrorInvalidValue;
  Maps m;
  if (!make_map(&m.q, p.q, p.layout, p.B, p.Nqk, p.S, p.D) ||
      !make_map(&m.k, p.k, p.layout, p.B, p.Nqk, p.S, p.D) ||
      !make_map(&m.v, p.v, p.layout, p.B, p.Nv, p.S, p.D) ||
      !make_map(&m.g, p.g, p.layout, p.B, p.Nv, p.S, p.D) ||
      !make_map(&m.o, p.out, p.layout, p.B, p.Nv, p.S, p.D))
    return cudaErrorInvalidValue;
  if (p.n_items < 1) return cudaSuccess;
  const int grid = p.n_items < num_sms ? p.n_items : num_sms;
  const int kind = (p.mode == 3) ? KIND_SUMMARY
                   : dbg          ? KIND_DEBUG
                   : (p.mode == 0 && dyn_items && p.n_items > grid) ? KIND_FORWARD_DYN
                                                                      : KIND_FORWARD;
  const bool d128 = (p.D == kD);
#define KDA_LAUNCH_FUSED(DIM_, KIND_) \
  kda_fused_kernel<DIM_, KIND_><<<grid, kThreads, kFusedSmemBytes, stream>>>(p, m, dbg)
  if (kind == KIND_FORWARD) {
    if (d128) KDA_LAUNCH_FUSED(kD, KIND_FORWARD); else KDA_LAUNCH_FUSED(64, KIND_FORWARD);
  } else if (kind == KIND_FORWARD_DYN) {
    if (d128) KDA_LAUNCH_FUSED(kD, KIND_FORWARD_DYN); else KDA_LAUNCH_FUSED(64, KIND_FORWARD_DYN);
  } else if (kind == KIND_SUMMARY) {
    if (d128) KDA_LAUNCH_FUSED(kD, KIND_SUMMARY); else KDA_LAUNCH_FUSED(64, KIND_SUMMARY);
  } else {
    if (d128) KDA_LAUNCH_FUSED(kD, KIND_DEBUG); else KDA_LAUNCH_FUSED(64, KIND_DEBUG);
  }
#undef KDA_LAUNCH_FUSED
  return cudaGetLastError();
}

}  // namespace kda
