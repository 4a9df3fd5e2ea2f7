// kda_fused.cu -- fused chunked KDA prefill for sm_100a: one persistent CTA per (sequence, value
// head) unit at a time, tcgen05 tensor cores for every contraction, the 128x128 fp32 state kept in
// TMEM for the whole sequence.
//
// Per 64-token chunk (the chunk equations of the FlashKDA README, 功能说明), eight phases:
//   1 prologue (CUDA cores): gate activation g = lb*sigmoid(e^A_log*(g_raw+dt_bias)) in log2
//     units, chunk-local cumulative sum G, q/k row L2-normalise, beta = sigmoid(logit); then the
//     bf16 operand tiles, each row factored through a reference row of its 16-row block so that
//     no factor overflows (the sub-chunk reference point b_gn of vLLM PR 43195's excerpt):
//       Aop = [k^ 2^(G-ref_I) ; scale q^ 2^(G-ref_I)],  B^(I) rows = k^ 2^(ref_I - G)  (s < 16(I+1)),
//       K~ = k^ 2^G, Q~ = scale q^ 2^G, K^ = k^ 2^(G_last - G)   (written over the raw q/k/g tiles)
//   2 MMA  D_I = Aop B^(I)^T, I = 0..3 (M=128, N=16(I+1), K=128): rows 0-63 give
//     T = stril(diag(beta) K~ K-^T), rows 64-127 give Aqk = tril(Q~ K-^T)
//   3 solve (CUDA cores, fp32): X = (I+T)^-1 by 16x16 diagonal blocks and off-diagonal updates;
//     Xsol = X diag(beta) -> bf16
//   4 MMA  W^T = K~^T Xsol^T and U^T = V^T Xsol^T (M=128, N=64, K=64); W -> -W bf16
//   5 MMA  Delta^T = U^T + S0 (-W)^T and O^T = S0 Q~^T (A = bf16 state read from TMEM)
//   6 Delta^T -> bf16 in TMEM;  S <- S Diag(2^G_last)
//   7 MMA  S += Delta^T K^,  O^T += Delta^T Aqk^T   (then TMA for the chunk after next)
//   8 O^T -> bf16 out;  S -> bf16 state operand (and fp32 final_state after the last chunk)
// Operands that feed the state recurrence (Xsol, W, S0, Delta, K^) are split into bf16 hi + lo
// parts and multiplied as hi*hi + lo*hi + hi*lo, so the state path keeps ~16 significant bits
// instead of bf16's 8: without that, rounding errors pile up when the gate does not decay.
// TMA brings q/k/v/g of the next chunk into the other half of a two-slot ring while a chunk is
// processed.  Every wait is bounded; a time-out sets the workspace status to DS_TIMEOUT and the
// CTA drains its copies, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_internal.h"
#include "kda_layout.cuh"
#include "kda_sm100.cuh"
#include "kda_tmap.h"

namespace kda {

namespace {

using namespace sm100;

constexpr int kThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kWaitLimit = 1u << 26;

// TMEM columns (512 allocated)
constexpr uint32_t TC_S = 0;       // state S, fp32 [Dv lanes][Dk cols]
constexpr uint32_t TC_DELTA = 128; // U^T then Delta^T, fp32 [Dv][64 tokens]
constexpr uint32_t TC_O = 192;     // O^T, fp32 [Dv][64 tokens]
constexpr uint32_t TC_D = 256;     // intra D_0..D_3 (160 cols); later W^T (64 cols) and:
constexpr uint32_t TC_SLO = 320;   //   bf16 lo part of the state operand (64 cols), phases 4b-5
constexpr uint32_t TC_DLO = 384;   //   bf16 lo part of the Delta^T operand (32 cols), phases 6-7
constexpr uint32_t TC_S0 = 416;    // bf16 state operand, 64 cols = 128 bf16 per lane
constexpr uint32_t TC_DB = 480;    // bf16 Delta^T operand, 32 cols = 64 bf16 per lane

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t SLOT_BYTES = 65536;
constexpr uint32_t OFF_Q = 0, OFF_K = 16384, OFF_G = 32768, OFF_V = 49152;
constexpr uint32_t SM_AOP = 131072;   // [128 rows][128] bf16, 2 atoms of 16 KB; after phase 2:
constexpr uint32_t SM_KLO = SM_AOP;           //   K^ lo part [64][128] (16 KB)
constexpr uint32_t SM_XWLO = SM_AOP + 16384;  //   Xsol lo part [64][64], then -W lo part [64][128]
constexpr uint32_t SM_OSTG = SM_AOP;          //   phase 8: out tile [64 tokens][128] for the TMA store
constexpr uint32_t SM_BT = 163840;    // [B^(0); B^(1); B^(2); B^(3)]: one 160-row tile; then the solve
constexpr uint32_t BT_ROWS = 160;
constexpr uint32_t SM_XSOL = 204800;  // [64][64] bf16
constexpr uint32_t SM_AQK = 212992;   // [64][64] bf16
constexpr uint32_t SM_WTOT = 221184;  // fp32 [8][128] warp totals of the gate cumsum
constexpr uint32_t SM_REFG = 225280;  // fp32 [4][128]: G at rows 15, 31, 47, 63
constexpr uint32_t SM_GC = 227328;    // fp32 [128]: 2^G_last
constexpr uint32_t SM_BETA = 227840;  // fp32 [64]
constexpr uint32_t SM_BAR = 228096;   // raw_full[2], mma
constexpr uint32_t SM_TSLOT = 228128;
constexpr uint32_t SM_FLAG = 228132;
constexpr uint32_t SM_END = 228160;
constexpr size_t kFusedSmemBytes = SM_END + 1024;

// Phase timestamps for performance analysis (CTA 0, thread 0, first 64 chunks).
#define KDA_TS(slot_)                                                        \
  do {                                                                       \
    if (tprof_on) p.tprof[(size_t)gidx * 32 + (slot_)] = clock64();          \
  } while (0)

__device__ __forceinline__ uint32_t dcol(int I) { return 8u * I * (I + 1); }

__device__ __forceinline__ bool plan_ok(const Params& p) {
  return p.plan[PH_MAGIC] == kPlanMagic && p.plan[PH_CHECKSUM] == p.plan_checksum &&
         p.plan[PH_UNITS] == p.n_units;
}

__device__ __forceinline__ void unpack8(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                    pack_bf16(f[6], f[7]));
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

struct Maps {
  CUtensorMap q, k, v, g, o;
};

// A unit's plan record as the producer keeps it in registers.
struct UnitRec {
  int b, h, hq, tok0, nch;
};
__device__ __forceinline__ UnitRec read_rec(const Params& p, int u) {
  UnitRec r{0, 0, 0, 0, 0};
  if (u < p.n_units) {
    const int32_t* rec = p.plan + kPlanHeader + u * kPlanRecord;
    r.b = rec[PR_B];
    r.h = rec[PR_H];
    r.hq = rec[PR_HQ];
    r.tok0 = rec[PR_TOK_START];
    r.nch = rec[PR_CHUNKS];
  }
  return r;
}

// TMA of chunk c of unit `ur` into ring slot `slot` (all four tensors, two 64-column boxes each).
__device__ void issue_chunk_loads(const Params& p, const Maps& m, uint32_t sbase, const UnitRec& ur,
                                  int c, int slot) {
  const int b = ur.b, h = ur.h, hq = ur.hq, tok0 = ur.tok0;
  const uint32_t bar = sbase + SM_BAR + 8u * slot;
  const uint32_t dst = sbase + slot * SLOT_BYTES;
  mbar_arrive_expect_tx(bar, SLOT_BYTES);
  const int t = c * kChunk;
  int qc1, qc2, vc1, vc2;
  if (p.layout == KDA_LAYOUT_BNSD) {
    qc1 = t; qc2 = b * p.Nqk + hq; vc1 = t; vc2 = b * p.Nv + h;
  } else {
    const int row = (p.layout == KDA_LAYOUT_BSND ? b * p.S : tok0) + t;
    qc1 = hq; qc2 = row; vc1 = h; vc2 = row;
  }
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    tma_load_3d(dst + OFF_Q + a * 8192, &m.q, bar, 64 * a, qc1, qc2);
    tma_load_3d(dst + OFF_K + a * 8192, &m.k, bar, 64 * a, qc1, qc2);
    tma_load_3d(dst + OFF_G + a * 8192, &m.g, bar, 64 * a, vc1, vc2);
    tma_load_3d(dst + OFF_V + a * 8192, &m.v, bar, 64 * a, vc1, vc2);
  }
}

// Rows of D_BLK (row block BLK of the intra product) -> T (fp32, scaled by beta, strictly
// lower, into Ts with pitch 68) for k rows, or Aqk (bf16, lower with diagonal, K-major) for
// q rows.  The TMEM load is issued by the whole warp; only lanes in row block BLK write.
template <int BLK>
__device__ __forceinline__ void extract_block(uint32_t ta, int r, bool krow, float br, float* Ts,
                                              uint8_t* aqk) {
  constexpr int NC = BLK + 1;
  constexpr int TP = 68;
  uint32_t v[16 * NC];
#pragma unroll
  for (int ch = 0; ch < NC; ++ch)
    tmem_ld16(ta + 8u * BLK * (BLK + 1) + 16 * ch, *reinterpret_cast<uint32_t(*)[16]>(v + 16 * ch));
  tmem_wait_ld();
  if ((r >> 4) != BLK) return;
  if (krow) {
#pragma unroll
    for (int s0 = 0; s0 < 64; s0 += 4) {
      float f[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int s = s0 + e;
        f[e] = (s < 16 * NC && s < r) ? br * __uint_as_float(v[s < 16 * NC ? s : 0]) : 0.f;
      }
      *reinterpret_cast<float4*>(Ts + r * TP + s0) = make_float4(f[0], f[1], f[2], f[3]);
    }
  } else {
#pragma unroll
    for (int s0 = 0; s0 < 64; s0 += 8) {
      float f[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int s = s0 + e;
        f[e] = (s < 16 * NC && s <= r) ? __uint_as_float(v[s < 16 * NC ? s : 0]) : 0.f;
      }
      *reinterpret_cast<uint4*>(aqk + sw128_offset(64, r, s0)) = pack8(f);
    }
  }
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    kda_fused_kernel(const Params p, const __grid_constant__ Maps maps, float* dbg) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t wq = (uint32_t)(warp & 3) * 32u;  // TMEM lane quarter of this warp
  const uint32_t wlane = wq << 16;
  const int wg = warp >> 2;

  if (!plan_ok(p)) {
    if (tid == 0) atomicExch(p.status, DS_PLAN);
    return;
  }
  const uint32_t bar_mma = sbase + SM_BAR + 16;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + SM_FLAG);
  float* wtot = reinterpret_cast<float*>(sm + SM_WTOT);
  float* refg = reinterpret_cast<float*>(sm + SM_REFG);
  float* gcs = reinterpret_cast<float*>(sm + SM_GC);
  float* beta_s = reinterpret_cast<float*>(sm + SM_BETA);

  if (tid == 0) {
    mbar_init(sbase + SM_BAR, 1);
    mbar_init(sbase + SM_BAR + 8, 1);
    mbar_init(bar_mma, 1);
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

  const int G_stride = gridDim.x;
  // producer cursor (thread 0): next (unit, chunk) of this CTA's stream to load
  // (plan records are read one unit ahead so no global load sits on the issue path)
  int pu = blockIdx.x, pc = 0;
  uint32_t issued = 0;
  UnitRec prec{0, 0, 0, 0, 0}, nrec{0, 0, 0, 0, 0};
  auto produce = [&]() {
    if (pu >= p.n_units) return;
    issue_chunk_loads(p, maps, sbase, prec, pc, issued & 1);
    ++issued;
    if (++pc == prec.nch) {
      pc = 0;
      pu += G_stride;
      prec = nrec;
      nrec = read_rec(p, pu + G_stride);
    }
  };
  if (tid == 0) {
    prec = read_rec(p, pu);
    nrec = read_rec(p, pu + G_stride);
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.k);
    tma_prefetch_desc(&maps.v);
    tma_prefetch_desc(&maps.g);
    produce();
    produce();
  }

  uint32_t gidx = 0;       // chunks consumed by this CTA
  uint32_t mma_phase = 0;  // parity of the next MMA-barrier completion
  bool aborted = false;

  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(p.status, DS_TIMEOUT);
  };
  auto wait_mma = [&]() {
    if (!mbar_wait_bounded(bar_mma, mma_phase, kWaitLimit)) fail();
    mma_phase ^= 1u;
  };

  for (int u = blockIdx.x; u < p.n_units && !aborted; u += G_stride) {
    const int32_t* rec = p.plan + kPlanHeader + u * kPlanRecord;
    const int b = rec[PR_B], h = rec[PR_H], tok0 = rec[PR_TOK_START];
    const int L = rec[PR_LEN], nch = rec[PR_CHUNKS], coff = rec[PR_CHUNK_OFFSET];
    const size_t sbase_g = ((size_t)b * p.Nv + h) * kD * kD;
    const float a_h = expf(p.A_log[h]);
    const float lbl2 = p.lower_bound * kLog2e;
    const int cg = tid & 15, rg = tid >> 4;
    const int j0 = cg * 8, r0 = rg * 4, Jb = rg >> 2;
    float dtb[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) dtb[e] = p.dt_bias[h * kD + j0 + e];

    // ---- state from initial_state (fp32 -> TMEM S, bf16 -> TMEM S0) ----
    {
      const int i = wq + lane;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t fv[32];
        const int col0 = wg * 64 + half * 32;
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
          if (p.S0) x = __ldg(reinterpret_cast<const float4*>(p.S0 + sbase_g + (size_t)i * kD + col0 + c));
          fv[c] = __float_as_uint(x.x);
          fv[c + 1] = __float_as_uint(x.y);
          fv[c + 2] = __float_as_uint(x.z);
          fv[c + 3] = __float_as_uint(x.w);
        }
        uint32_t lo[16], hi[16], pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          lo[c] = fv[c];
          hi[c] = fv[16 + c];
        }
        tmem_st16(tbase + wlane + TC_S + col0, lo);
        tmem_st16(tbase + wlane + TC_S + col0 + 16, hi);
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[c] = pack_bf16(__uint_as_float(fv[2 * c]), __uint_as_float(fv[2 * c + 1]));
        tmem_st16(tbase + wlane + TC_S0 + col0 / 2, pk);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();

    float bl_next = 0.f;
    if (tid < kChunk && tid < L)
      bl_next = __bfloat162float(p.beta[beta_offset(p.layout, p.Nv, p.S, b, h, tok0, tid)]);

    for (int c = 0; c < nch; ++c, ++gidx) {
      const int slot = gidx & 1;
      uint8_t* sQ = sm + slot * SLOT_BYTES + OFF_Q;
      uint8_t* sK = sm + slot * SLOT_BYTES + OFF_K;
      uint8_t* sG = sm + slot * SLOT_BYTES + OFF_G;
      uint8_t* sV = sm + slot * SLOT_BYTES + OFF_V;
      const uint32_t aQ = sbase + slot * SLOT_BYTES + OFF_Q;
      const uint32_t aK = sbase + slot * SLOT_BYTES + OFF_K;
      const uint32_t aG = sbase + slot * SLOT_BYTES + OFF_G;
      const uint32_t aV = sbase + slot * SLOT_BYTES + OFF_V;
      const int t0 = c * kChunk;
      const int n = min(kChunk, L - t0);
      const bool last = (c == nch - 1);
      const bool tprof_on = p.tprof && blockIdx.x == 0 && tid == 0 && gidx < 64;
      KDA_TS(0);

      // =================== phase 1: prologue and operand tiles ===================
      const float blog = bl_next;  // this chunk's beta logit (row tid), loaded one chunk ahead
      if (c + 1 < nch && tid < kChunk && t0 + kChunk + tid < L)
        bl_next = __bfloat162float(
            p.beta[beta_offset(p.layout, p.Nv, p.S, b, h, tok0, t0 + kChunk + tid)]);
      if (!mbar_wait_bounded(sbase + SM_BAR + 8u * slot, (gidx >> 1) & 1u, kWaitLimit)) fail();
      if (tid == 0) tma_store_wait_read();  // the out tile staged in the Aop region was read
      KDA_TS(1);

      float G[4][8];
      uint4 khlo[4];  // K^ lo parts of this thread's rows, stored once the intra MMA is done
      {
        // g_act * log2(e) = lb log2(e) / (1 + 2^(-log2(e) e^A_log (g_raw + dt_bias)))
        const float ca = -a_h * kLog2e;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = r0 + i;
          float gv[8];
          unpack8(*reinterpret_cast<const uint4*>(sG + sw128_offset(64, r, j0)), gv);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float sg = __fdividef(lbl2, 1.0f + ex2(ca * (gv[e] + dtb[e])));
            G[i][e] = (r < n) ? sg : 0.0f;
          }
        }
#pragma unroll
        for (int i = 1; i < 4; ++i)
#pragma unroll
          for (int e = 0; e < 8; ++e) G[i][e] += G[i - 1][e];
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float t = __shfl_up_sync(0xffffffffu, G[3][e], 16);
        if (lane >= 16) {
#pragma unroll
          for (int i = 0; i < 4; ++i) G[i][e] += t;
        }
      }
      if (lane >= 16) {
        float4* dst = reinterpret_cast<float4*>(wtot + warp * kD + j0);
        dst[0] = make_float4(G[3][0], G[3][1], G[3][2], G[3][3]);
        dst[1] = make_float4(G[3][4], G[3][5], G[3][6], G[3][7]);
      }
      if (tid < kChunk) beta_s[tid] = (tid < n) ? __fdividef(1.0f, 1.0f + __expf(-blog)) : 0.0f;
      __syncthreads();
      KDA_TS(11);
      {
        float pre[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) pre[e] = 0.f;
        for (int w2 = 0; w2 < warp; ++w2) {
#pragma unroll
          for (int e = 0; e < 8; ++e) pre[e] += wtot[w2 * kD + j0 + e];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int e = 0; e < 8; ++e) G[i][e] += pre[e];
      }
      if ((rg & 3) == 3) {
        float4* dst = reinterpret_cast<float4*>(refg + Jb * kD + j0);
        dst[0] = make_float4(G[3][0], G[3][1], G[3][2], G[3][3]);
        dst[1] = make_float4(G[3][4], G[3][5], G[3][6], G[3][7]);
      }
      __syncthreads();
      KDA_TS(12);
      if (tid < kD) gcs[tid] = ex2(refg[3 * kD + tid]);
      {
        // reference rows of this thread's 16-row block Jb (read straight from shared memory so
        // no register array is indexed by the thread-dependent block number)
        const float* Rprev = refg + (Jb == 0 ? 0 : Jb - 1) * kD + j0;  // G at row 16 Jb - 1
        const float* Rown = refg + Jb * kD + j0;                       // G at row 16 Jb + 15
        const float* Rnext = refg + (Jb < 3 ? Jb + 1 : 3) * kD + j0;   // G at row 16 Jb + 31
        const float* Rlast = refg + 3 * kD + j0;                       // G at row 63 (= G_last)
        float refI[8], GeJ[8], p2ref[8], kfac[8], cdiag[8], c2[8], c3[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          refI[e] = (Jb == 0) ? 0.f : Rprev[e];
          GeJ[e] = Rown[e];
          p2ref[e] = ex2(refI[e]);
          kfac[e] = ex2(Rlast[e] - GeJ[e]);
          cdiag[e] = ex2(refI[e] - GeJ[e]);
          c2[e] = (Jb <= 1) ? ex2(Rnext[e] - GeJ[e]) : 0.f;
          c3[e] = (Jb == 0) ? ex2(refg[2 * kD + j0 + e] - GeJ[e]) : 0.f;
        }
        uint4 qraw[4], kraw[4];
        float rqv[4], rkv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          qraw[i] = *reinterpret_cast<const uint4*>(sQ + sw128_offset(64, r0 + i, j0));
          kraw[i] = *reinterpret_cast<const uint4*>(sK + sw128_offset(64, r0 + i, j0));
          float qv[8], kv[8];
          unpack8(qraw[i], qv);
          unpack8(kraw[i], kv);
          float ssq = 0.f, ssk = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            ssq = fmaf(qv[e], qv[e], ssq);
            ssk = fmaf(kv[e], kv[e], ssk);
          }
          rqv[i] = ssq;
          rkv[i] = ssk;
        }
#pragma unroll
        for (int o = 1; o < 16; o <<= 1)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            rqv[i] += __shfl_xor_sync(0xffffffffu, rqv[i], o);
            rkv[i] += __shfl_xor_sync(0xffffffffu, rkv[i], o);
          }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = r0 + i;
          const bool valid = r < n;
          float qv[8], kv[8];
          unpack8(qraw[i], qv);
          unpack8(kraw[i], kv);
          const float rq = rsqrtf(rqv[i] + 1e-6f) * p.scale;
          const float rk = rsqrtf(rkv[i] + 1e-6f);
          float ka[8], qa[8], kt[8], qt[8], kh[8], khl[8], b0[8], b1[8], b2[8], b3[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float Gv = G[i][e];
            const float kn = valid ? kv[e] * rk : 0.f;
            const float qn = valid ? qv[e] * rq : 0.f;
            const float fA = ex2(Gv - refI[e]);
            const float kbe = kn * ex2(GeJ[e] - Gv);
            ka[e] = kn * fA;
            qa[e] = qn * fA;
            kt[e] = ka[e] * p2ref[e];
            qt[e] = qa[e] * p2ref[e];
            kh[e] = kbe * kfac[e];
            khl[e] = kh[e] - bf16_round(kh[e]);
            b0[e] = kbe * cdiag[e];  // B^(Jb): diagonal block
            b1[e] = kbe;             // B^(Jb+1): reference row is this block's last row
            b2[e] = kbe * c2[e];     // B^(Jb+2)
            b3[e] = kbe * c3[e];     // B^(Jb+3)
          }
          *reinterpret_cast<uint4*>(sm + SM_AOP + sw128_offset(128, r, j0)) = pack8(ka);
          *reinterpret_cast<uint4*>(sm + SM_AOP + sw128_offset(128, 64 + r, j0)) = pack8(qa);
          *reinterpret_cast<uint4*>(sQ + sw128_offset(64, r, j0)) = pack8(qt);
          *reinterpret_cast<uint4*>(sK + sw128_offset(64, r, j0)) = pack8(kh);
          khlo[i] = pack8(khl);
          *reinterpret_cast<uint4*>(sG + sw128_offset(64, r, j0)) = pack8(kt);
          *reinterpret_cast<uint4*>(sm + SM_BT + sw128_offset(BT_ROWS, dcol(Jb) + r, j0)) =
              pack8(b0);
          if (Jb + 1 <= 3)
            *reinterpret_cast<uint4*>(sm + SM_BT + sw128_offset(BT_ROWS, dcol(Jb + 1) + r, j0)) = pack8(b1);
          if (Jb + 2 <= 3)
            *reinterpret_cast<uint4*>(sm + SM_BT + sw128_offset(BT_ROWS, dcol(Jb + 2) + r, j0)) = pack8(b2);
          if (Jb + 3 <= 3)
            *reinterpret_cast<uint4*>(sm + SM_BT + sw128_offset(BT_ROWS, dcol(Jb + 3) + r, j0)) = pack8(b3);
          if (!valid) *reinterpret_cast<uint4*>(sV + sw128_offset(64, r, j0)) = make_uint4(0, 0, 0, 0);
        }
      }
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
        // D[:, 0:160] = Aop [B^(0); B^(1); B^(2); B^(3)]^T in one N=160 MMA chain: D_I = cols dcol(I)..
        const uint32_t idesc = idesc_bf16(128, BT_ROWS, 0, 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = smem_desc(sbase + SM_AOP + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd =
              smem_desc(sbase + SM_BT + (kk >> 2) * (BT_ROWS * 128) + (kk & 3) * 32, 16, 1024);
          mma_ss(tbase + TC_D, ad, bd, idesc, kk > 0);
        }
        mma_commit(bar_mma);
      }
      wait_mma();
      KDA_TS(3);
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<uint4*>(sm + SM_KLO + sw128_offset(64, r0 + i, j0)) = khlo[i];

      // =================== phase 3: T, Aqk, solve ===================
      // fp32 scratch in the B-tile region (free once the intra MMA has completed)
      constexpr int TP = 68, YP = 36;                       // row pitches (floats)
      float* Ts = reinterpret_cast<float*>(sm + SM_BT);   // T = stril(diag(beta) K~ K-^T) [64][TP]
      float* Xs = Ts + 64 * TP;                           // X = (I + T)^-1            [64][TP]
      float* Ys = Xs + 64 * TP;                           // block products            [32][YP]
      {
        // warp w: lane quarter q = w & 3 (q < 2: k rows -> T; q >= 2: q rows -> Aqk), row block
        // blk = 2 (q & 1) + (w >> 2); one batched TMEM load of D_blk, then the 16 lanes of that
        // block write their rows.  X is cleared alongside.
        const int q4 = warp & 3;
        const int r = (q4 & 1) * 32 + lane;
        const int blk = 2 * (q4 & 1) + (warp >> 2);
        const bool krow = q4 < 2;
        const float br = krow ? beta_s[r] : 0.f;
        const uint32_t ta = tbase + wlane + TC_D;
        switch (blk) {
          case 0: extract_block<0>(ta, r, krow, br, Ts, sm + SM_AQK); break;
          case 1: extract_block<1>(ta, r, krow, br, Ts, sm + SM_AQK); break;
          case 2: extract_block<2>(ta, r, krow, br, Ts, sm + SM_AQK); break;
          default: extract_block<3>(ta, r, krow, br, Ts, sm + SM_AQK); break;
        }
        for (int e = tid; e < 64 * TP / 4; e += kThreads)
          reinterpret_cast<float4*>(Xs)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      __syncthreads();
      KDA_TS(13);
      // level 1: X_II = (I + T_II)^-1 for the four 16x16 diagonal blocks, one column per thread
      if (tid < 64) {
        const int I = tid >> 4, cc = tid & 15, base = 16 * I;
        float x[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) x[k] = (k == cc) ? 1.f : 0.f;
        // outer-product order: once x[k] is final, update every later row (independent FMAs)
#pragma unroll
        for (int k = 0; k < 15; ++k) {
#pragma unroll
          for (int rr = k + 1; rr < 16; ++rr) x[rr] = fmaf(-Ts[(base + rr) * TP + base + k], x[k], x[rr]);
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) Xs[(base + k) * TP + base + cc] = x[k];
      }
      __syncthreads();
      KDA_TS(14);
      // level 2: X_{I,I-1} = -X_II T_{I,I-1} X_{I-1,I-1} for I = 1, 3 (two 16x16 merges)
      {
        const int pI = tid >> 7, rr = (tid >> 3) & 15, c0 = (tid & 7) * 2;
        const int I = 2 * pI + 1, J = I - 1;
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float t = Ts[(16 * I + rr) * TP + 16 * J + k];
          const float2 xv = *reinterpret_cast<const float2*>(Xs + (16 * J + k) * TP + 16 * J + c0);
          y0 = fmaf(t, xv.x, y0);
          y1 = fmaf(t, xv.y, y1);
        }
        *reinterpret_cast<float2*>(Ys + (16 * pI + rr) * YP + c0) = make_float2(y0, y1);
        __syncthreads();
        float z0 = 0.f, z1 = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float xx = Xs[(16 * I + rr) * TP + 16 * I + k];
          const float2 yv = *reinterpret_cast<const float2*>(Ys + (16 * pI + k) * YP + c0);
          z0 = fmaf(xx, yv.x, z0);
          z1 = fmaf(xx, yv.y, z1);
        }
        *reinterpret_cast<float2*>(Xs + (16 * I + rr) * TP + 16 * J + c0) = make_float2(-z0, -z1);
      }
      __syncthreads();
      KDA_TS(15);
      // level 3: X_(32:64, 0:32) = -X_(32:64, 32:64) T_(32:64, 0:32) X_(0:32, 0:32) (32x32 merge);
      // each thread owns a 2x2 output tile (rows 2 tr, 2 tr + 1; columns 2 tc, 2 tc + 1)
      {
        const int tr = tid >> 4, tc = tid & 15;
        float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll
        for (int k0 = 0; k0 < 32; k0 += 4) {
          const float4 ta = *reinterpret_cast<const float4*>(Ts + (32 + 2 * tr) * TP + k0);
          const float4 tb = *reinterpret_cast<const float4*>(Ts + (33 + 2 * tr) * TP + k0);
          const float tav[4] = {ta.x, ta.y, ta.z, ta.w}, tbv[4] = {tb.x, tb.y, tb.z, tb.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 xv = *reinterpret_cast<const float2*>(Xs + (k0 + e) * TP + 2 * tc);
            y00 = fmaf(tav[e], xv.x, y00);
            y01 = fmaf(tav[e], xv.y, y01);
            y10 = fmaf(tbv[e], xv.x, y10);
            y11 = fmaf(tbv[e], xv.y, y11);
          }
        }
        *reinterpret_cast<float2*>(Ys + (2 * tr) * YP + 2 * tc) = make_float2(y00, y01);
        *reinterpret_cast<float2*>(Ys + (2 * tr + 1) * YP + 2 * tc) = make_float2(y10, y11);
        __syncthreads();
        float z00 = 0.f, z01 = 0.f, z10 = 0.f, z11 = 0.f;
#pragma unroll
        for (int k0 = 0; k0 < 32; k0 += 4) {
          const float4 xa = *reinterpret_cast<const float4*>(Xs + (32 + 2 * tr) * TP + 32 + k0);
          const float4 xb = *reinterpret_cast<const float4*>(Xs + (33 + 2 * tr) * TP + 32 + k0);
          const float xav[4] = {xa.x, xa.y, xa.z, xa.w}, xbv[4] = {xb.x, xb.y, xb.z, xb.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 yv = *reinterpret_cast<const float2*>(Ys + (k0 + e) * YP + 2 * tc);
            z00 = fmaf(xav[e], yv.x, z00);
            z01 = fmaf(xav[e], yv.y, z01);
            z10 = fmaf(xbv[e], yv.x, z10);
            z11 = fmaf(xbv[e], yv.y, z11);
          }
        }
        *reinterpret_cast<float2*>(Xs + (32 + 2 * tr) * TP + 2 * tc) = make_float2(-z00, -z01);
        *reinterpret_cast<float2*>(Xs + (33 + 2 * tr) * TP + 2 * tc) = make_float2(-z10, -z11);
      }
      __syncthreads();
      KDA_TS(16);
      // Xsol = X diag(beta) -> bf16 hi and lo parts, K-major [r][s]
      {
        const int r = tid >> 2, s0 = (tid & 3) * 16;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float f[8], fl[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int s = s0 + 8 * hh + e;
            f[e] = (s <= r) ? Xs[r * TP + s] * beta_s[s] : 0.f;
            fl[e] = f[e] - bf16_round(f[e]);
          }
          *reinterpret_cast<uint4*>(sm + SM_XSOL + sw128_offset(64, r, s0 + 8 * hh)) = pack8(f);
          *reinterpret_cast<uint4*>(sm + SM_XWLO + sw128_offset(64, r, s0 + 8 * hh)) = pack8(fl);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      KDA_TS(4);

      // =================== phase 4: W^T and U^T ===================
      if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 64, 1, 0);
        // W first (its epilogue waits on this commit), then U (consumed in order by phase 5)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t aw = smem_desc(aG + kk * 2048, 8192, 1024);
          mma_ss(tbase + TC_D, aw, smem_desc(sbase + SM_XSOL + kk * 32, 16, 1024), idesc, kk > 0);
          mma_ss(tbase + TC_D, aw, smem_desc(sbase + SM_XWLO + kk * 32, 16, 1024), idesc, 1);
        }
        if (!dbg) mma_commit(bar_mma);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t av = smem_desc(aV + kk * 2048, 8192, 1024);
          mma_ss(tbase + TC_DELTA, av, smem_desc(sbase + SM_XSOL + kk * 32, 16, 1024), idesc, kk > 0);
          mma_ss(tbase + TC_DELTA, av, smem_desc(sbase + SM_XWLO + kk * 32, 16, 1024), idesc, 1);
        }
        if (dbg) mma_commit(bar_mma);  // the debug dump reads U too
      }
      {
        // lo part of the bf16 state operand, S - bf16(S), built while the W/U MMAs run (they
        // touch neither TC_S nor TC_SLO)
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t v0[16], v1[16], pk[16];
          const int col = wg * 64 + 32 * ch;
          tmem_ld16(tbase + wlane + TC_S + col, v0);
          tmem_ld16(tbase + wlane + TC_S + col + 16, v1);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float a0 = __uint_as_float(v0[2 * e]), a1 = __uint_as_float(v0[2 * e + 1]);
            const float c0 = __uint_as_float(v1[2 * e]), c1 = __uint_as_float(v1[2 * e + 1]);
            pk[e] = pack_bf16(a0 - bf16_round(a0), a1 - bf16_round(a1));
            pk[8 + e] = pack_bf16(c0 - bf16_round(c0), c1 - bf16_round(c1));
          }
          tmem_st16(tbase + wlane + TC_SLO + col / 2, pk);
        }
        tmem_wait_st();
      }
      wait_mma();
      KDA_TS(5);
      tc_fence_after();
      {
        // W^T row j (tokens r = 32 wg .. 32 wg + 31) -> -W^T stored MN-major: tile [j][r], one atom
        const int j = wq + lane;
        uint32_t vw[2][16];
        tmem_ld16(tbase + wlane + TC_D + wg * 32, vw[0]);
        tmem_ld16(tbase + wlane + TC_D + wg * 32 + 16, vw[1]);
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const uint32_t* v = vw[ch];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float hi[8], lo[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float wv = -__uint_as_float(v[8 * hh + e]);
              hi[e] = wv;
              lo[e] = wv - bf16_round(wv);
            }
            const int rc = wg * 32 + 16 * ch + 8 * hh;  // first token of this 8-wide chunk
            *reinterpret_cast<uint4*>(sG + sw128_offset(128, j, rc)) = pack8(hi);
            *reinterpret_cast<uint4*>(sm + SM_XWLO + sw128_offset(128, j, rc)) = pack8(lo);
          }
        }
      }
      if (dbg) {  // per-chunk intermediates in the two-kernel workspace layout (fp32)
        float* dc = dbg + (size_t)(coff + c) * (kWsChunkBytes / 4);
        const int i = wq + lane;
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t v[16], w[16];
          tmem_ld16(tbase + wlane + TC_D + 16 * ch, w);
          tmem_ld16(tbase + wlane + TC_DELTA + 16 * ch, v);
          tmem_wait_ld();
          if (wg == 0)
            for (int e = 0; e < 16; ++e) {
              dc[kWsW / 4 + (16 * ch + e) * kD + i] = __uint_as_float(w[e]);
              dc[kWsU / 4 + (16 * ch + e) * kD + i] = __uint_as_float(v[e]);
            }
        }
        for (int e = tid; e < kChunk * kD; e += kThreads) {
          const int r = e / kD, j = e % kD;
          dc[kWsQt / 4 + e] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sQ + sw128_offset(64, r, j)));
          dc[kWsKh / 4 + e] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sK + sw128_offset(64, r, j)));
        }
        for (int e = tid; e < kChunk * kChunk; e += kThreads) {
          const int r = e / kChunk, s = e % kChunk;
          dc[kWsAqk / 4 + e] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + SM_AQK + sw128_offset(64, r, s)));
        }
        if (tid < kD) dc[kWsGc / 4 + tid] = gcs[tid];
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      KDA_TS(6);

      // =================== phase 5: Delta^T = U^T - S0 W^T,  O^T = S0 Q~^T ===================
      if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 64, 0, 0);
        const uint32_t idesc_w = idesc_bf16(128, 64, 0, 1);  // -W^T tiles are MN-major [j][r]
        // Delta first (phase 6 waits on this commit); O^T = S0 Q~^T after it, covered by the
        // commit of phase 7
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bw = smem_desc(aG + kk * 2048, 16384, 1024);
          mma_ts(tbase + TC_DELTA, tbase + TC_S0 + kk * 8, bw, idesc_w, 1);
          mma_ts(tbase + TC_DELTA, tbase + TC_SLO + kk * 8, bw, idesc_w, 1);
          mma_ts(tbase + TC_DELTA, tbase + TC_S0 + kk * 8,
                 smem_desc(sbase + SM_XWLO + kk * 2048, 16384, 1024), idesc_w, 1);
        }
        mma_commit(bar_mma);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;
          mma_ts(tbase + TC_O, tbase + TC_S0 + kk * 8, smem_desc(aQ + koff, 16, 1024), idesc, kk > 0);
        }
      }
      if (wg == 1) {
        // S <- S Diag(2^G_last) while the Delta/O MMAs run (they read the bf16 copies, not TC_S)
#pragma unroll
        for (int ch = 0; ch < 8; ch += 2) {
          uint32_t v[16], w2[16];
          tmem_ld16(tbase + wlane + TC_S + 16 * ch, v);
          tmem_ld16(tbase + wlane + TC_S + 16 * ch + 16, w2);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            v[e] = __float_as_uint(__uint_as_float(v[e]) * gcs[16 * ch + e]);
            w2[e] = __float_as_uint(__uint_as_float(w2[e]) * gcs[16 * ch + 16 + e]);
          }
          tmem_st16(tbase + wlane + TC_S + 16 * ch, v);
          tmem_st16(tbase + wlane + TC_S + 16 * ch + 16, w2);
        }
        tmem_wait_st();
      }
      wait_mma();
      KDA_TS(7);
      tc_fence_after();

      // =================== phase 6: Delta^T -> bf16 hi and lo ===================
      {
        // warpgroup wg converts tokens 32 wg .. 32 wg + 31 (one batched load of 32 columns)
        uint32_t v0[16], v1[16], hi[16], lo[16];
        tmem_ld16(tbase + wlane + TC_DELTA + 32 * wg, v0);
        tmem_ld16(tbase + wlane + TC_DELTA + 32 * wg + 16, v1);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float d0 = __uint_as_float(v0[2 * e]), d1 = __uint_as_float(v0[2 * e + 1]);
          const float d2 = __uint_as_float(v1[2 * e]), d3 = __uint_as_float(v1[2 * e + 1]);
          hi[e] = pack_bf16(d0, d1);
          hi[8 + e] = pack_bf16(d2, d3);
          lo[e] = pack_bf16(d0 - bf16_round(d0), d1 - bf16_round(d1));
          lo[8 + e] = pack_bf16(d2 - bf16_round(d2), d3 - bf16_round(d3));
        }
        tmem_st16(tbase + wlane + TC_DB + 16 * wg, hi);
        tmem_st16(tbase + wlane + TC_DLO + 16 * wg, lo);
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
          const uint64_t bk = smem_desc(aK + kk * 2048, 8192, 1024);
          mma_ts(tbase + TC_S, tbase + TC_DB + kk * 8, bk, idesc_s, 1);
          mma_ts(tbase + TC_S, tbase + TC_DLO + kk * 8, bk, idesc_s, 1);
          mma_ts(tbase + TC_S, tbase + TC_DB + kk * 8, smem_desc(sbase + SM_KLO + kk * 2048, 8192, 1024),
                 idesc_s, 1);
          mma_ts(tbase + TC_O, tbase + TC_DB + kk * 8, smem_desc(sbase + SM_AQK + kk * 32, 16, 1024),
                 idesc_o, 1);
        }
        mma_commit(bar_mma);
      }
      wait_mma();
      KDA_TS(9);
      if (tid == 0 && !*abort_flag) {
        fence_proxy_async_smem();
        produce();  // the slot of this chunk is free: bring in the chunk after next
      }
      KDA_TS(17);
      tc_fence_after();

      // =================== phase 8: out rows;  S -> bf16 operand (and final_state) ===================
      {
        const int i = wq + lane;
        uint32_t vo[2][16];
        tmem_ld16(tbase + wlane + TC_O + wg * 32, vo[0]);
        tmem_ld16(tbase + wlane + TC_O + wg * 32 + 16, vo[1]);
        tmem_wait_ld();
        if (n == kChunk) {
          // full chunk: out tile [t][i] (128B-swizzled, as the out tensor map expects) in the free
          // Aop region, then two TMA stores issued below
#pragma unroll
          for (int ch = 0; ch < 2; ++ch)
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int t = wg * 32 + 16 * ch + e;
              *reinterpret_cast<__nv_bfloat16*>(sm + SM_OSTG + sw128_offset(64, t, i)) =
                  __float2bfloat16_rn(__uint_as_float(vo[ch][e]));
            }
        } else {
          // the sequence's last, partial chunk: plain stores of the valid rows
          const int64_t ostride = (p.layout == KDA_LAYOUT_BNSD) ? kD : (int64_t)p.Nv * kD;
          __nv_bfloat16* orow = p.out + row_offset(p.layout, p.Nv, p.S, b, h, tok0, t0) + i;
#pragma unroll
          for (int ch = 0; ch < 2; ++ch)
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int t = wg * 32 + 16 * ch + e;
              if (t < n) orow[t * ostride] = __float2bfloat16_rn(__uint_as_float(vo[ch][e]));
            }
        }
        KDA_TS(18);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t v0[16], v1[16], pk[16];
          const int col = wg * 64 + 32 * ch;
          tmem_ld16(tbase + wlane + TC_S + col, v0);
          tmem_ld16(tbase + wlane + TC_S + col + 16, v1);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            pk[e] = pack_bf16(__uint_as_float(v0[2 * e]), __uint_as_float(v0[2 * e + 1]));
            pk[8 + e] = pack_bf16(__uint_as_float(v1[2 * e]), __uint_as_float(v1[2 * e + 1]));
          }
          tmem_st16(tbase + wlane + TC_S0 + col / 2, pk);
          if (last) {
            float* dst = p.Sf + sbase_g + (size_t)i * kD + col;
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
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      KDA_TS(10);
      if (tid == 0 && n == kChunk) {
        int oc1, oc2;
        if (p.layout == KDA_LAYOUT_BNSD) {
          oc1 = t0;
          oc2 = b * p.Nv + h;
        } else {
          oc1 = h;
          oc2 = (p.layout == KDA_LAYOUT_BSND ? b * p.S : tok0) + t0;
        }
        tma_store_3d(&maps.o, sbase + SM_OSTG, 0, oc1, oc2);
        tma_store_3d(&maps.o, sbase + SM_OSTG + 8192, 64, oc1, oc2);
        tma_store_commit();
      }
      if (*abort_flag) {
        aborted = true;
        break;
      }
    }
    // rows past the valid length (BNSD/BSND storage padding) are defined as zero
    if (!aborted && p.layout != KDA_LAYOUT_TND) {
      for (int e = tid; e < (p.S - L) * 16; e += kThreads) {
        const int t = L + (e >> 4), q8 = (e & 15) * 8;
        *reinterpret_cast<uint4*>(p.out + row_offset(p.layout, p.Nv, p.S, b, h, tok0, t) + q8) =
            make_uint4(0, 0, 0, 0);
      }
    }
  }

  // drain: loads still in flight must land, and stores complete, before this CTA exits
  if (tid == 0) {
    tma_store_wait_all();
    while (gidx < issued) {
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

bool make_map(CUtensorMap* m, const void* base, int layout, int B, int NX, int S) {
  uint64_t dims[3], strides[2];
  uint32_t box[3];
  if (layout == KDA_LAYOUT_BNSD) {
    dims[0] = kD; dims[1] = (uint64_t)S; dims[2] = (uint64_t)B * NX;
    strides[0] = kD * 2; strides[1] = (uint64_t)S * kD * 2;
    box[0] = 64; box[1] = 64; box[2] = 1;
  } else {
    const uint64_t rows = (layout == KDA_LAYOUT_BSND) ? (uint64_t)B * S : (uint64_t)S;
    dims[0] = kD; dims[1] = (uint64_t)NX; dims[2] = rows;
    strides[0] = kD * 2; strides[1] = (uint64_t)NX * kD * 2;
    box[0] = 64; box[1] = 1; box[2] = 64;
  }
  return encode_bf16_3d(m, base, dims, strides, box);
}

}  // namespace

cudaError_t launch_fused(const Params& p, float* dbg, cudaStream_t stream) {
  static int configured_device = -1;
  static int num_sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(kda_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kFusedSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  Maps m;
  if (!make_map(&m.q, p.q, p.layout, p.B, p.Nqk, p.S) ||
      !make_map(&m.k, p.k, p.layout, p.B, p.Nqk, p.S) ||
      !make_map(&m.v, p.v, p.layout, p.B, p.Nv, p.S) ||
      !make_map(&m.g, p.g, p.layout, p.B, p.Nv, p.S) ||
      !make_map(&m.o, p.out, p.layout, p.B, p.Nv, p.S))
    return cudaErrorInvalidValue;
  const int grid = p.n_units < num_sms ? p.n_units : num_sms;
  kda_fused_kernel<<<grid, kThreads, kFusedSmemBytes, stream>>>(p, m, dbg);
  return cudaGetLastError();
}

}  // namespace kda
