// kda_simt.cu -- two-kernel fp32 CUDA-core path of chunked KDA prefill (sm_100a).
//
// Kernel 1 (kda_chunk_simt_kernel), one CTA per (unit, chunk), all chunks in parallel:
//   prologue  : q/k row L2-normalise, beta = sigmoid(logit), gate activation and the chunk-local
//               cumulative sum of the log-decay in log2 units (vLLM PR 43195: decay via exp2 of
//               the cumsum scaled by 1/ln 2);
//   intra     : T = stril(diag(beta) K~ K-^T) and Aqk = tril(Q~ K-^T), each pair factored through
//               a reference row of its 16-row block so no factor overflows (the sub-chunk
//               reference point b_gn of the FLA intra kernels, vLLM PR 43195 code excerpt);
//   solve     : W = (I+T)^-1 diag(beta) K~ and U = (I+T)^-1 diag(beta) V by forward substitution
//               (FlashKDA README 功能说明);
//   and writes W, U, Q~, K^ = K- * gamma_last, Aqk and gamma_last to the workspace.
// Kernel 2 (kda_scan_simt_kernel), one CTA per (unit, 16 value rows of the state): the
//   sequential pass over the chunks with the state tile in shared memory:
//     Delta = U - W S^T,  O = Q~ S^T + Aqk Delta,  S <- S Diag(gamma_last) + Delta^T K^.
// Everything is fp32; out is rounded to bf16 (nearest even).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_internal.h"
#include "kda_layout.cuh"
#include "kda_once.h"

namespace kda {

namespace {

constexpr int kP = kD + 1;  // padded pitch of fp32 [64][128] tiles in shared memory
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

// Find the unit whose chunk range [offset, offset + chunks) holds global chunk `gc`.
__device__ __forceinline__ int unit_of_chunk(const int32_t* plan, int n_units, int gc) {
  int lo = 0, hi = n_units - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (plan[kPlanHeader + mid * kPlanRecord + PR_CHUNK_OFFSET] <= gc) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ bool plan_ok(const Params& p) {
  return p.plan[PH_MAGIC] == kPlanMagic && p.plan[PH_CHECKSUM] == p.plan_checksum &&
         p.plan[PH_UNITS] == p.n_units;
}

}  // namespace

constexpr int kSimtChunkSmemFloats = 4 * kChunk * kP + kChunk * (kChunk + 1) + kChunk +
                                     2 * 16 * kP + kChunk * kP;
constexpr size_t kSimtChunkSmemBytes = (size_t)kSimtChunkSmemFloats * 4;

__global__ void __launch_bounds__(256, 1) kda_chunk_simt_kernel(Params p) {
  if (!plan_ok(p)) {
    if (threadIdx.x == 0) atomicExch(p.status, DS_PLAN);
    return;
  }
  extern __shared__ float sm[];
  float* Kn = sm;                          // [64][kP]  normalised k
  float* QW = Kn + kChunk * kP;            // [64][kP]  normalised q, later K~ then W
  float* Gs = QW + kChunk * kP;            // [64][kP]  log2 cumulative decay
  float* VU = Gs + kChunk * kP;            // [64][kP]  v, later U
  float* T = VU + kChunk * kP;             // [64][65]  T = stril(diag(beta) K~ K-^T)
  float* bet = T + kChunk * (kChunk + 1);  // [64]
  float* Ak = bet + kChunk;                // [16][kP]  k rows of block I scaled to the ref row
  float* Aq = Ak + 16 * kP;                // [16][kP]  q rows of block I scaled to the ref row
  float* Bk = Aq + 16 * kP;                // [64][kP]  k rows s scaled from the ref row

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gc = blockIdx.x;
  const int u = unit_of_chunk(p.plan, p.n_units, gc);
  const int32_t* rec = p.plan + kPlanHeader + u * kPlanRecord;
  const int b = rec[PR_B], h = rec[PR_H], hq = rec[PR_HQ], tok0 = rec[PR_TOK_START];
  const int L = rec[PR_LEN];
  const int c = gc - rec[PR_CHUNK_OFFSET];
  const int t0 = c * kChunk;
  const int n = min(kChunk, L - t0);

  // ---- q/k normalise, v load (warp per row, 4 elements per lane) ----
  for (int r = warp; r < kChunk; r += 8) {
    float kx[4] = {0, 0, 0, 0}, qx[4] = {0, 0, 0, 0}, vx[4] = {0, 0, 0, 0};
    if (r < n) {
      const int64_t oq = row_offset(p.layout, p.Nqk, p.S, b, hq, tok0, t0 + r);
      const int64_t ov = row_offset(p.layout, p.Nv, p.S, b, h, tok0, t0 + r);
      load4_bf16(p.k + oq + lane * 4, kx);
      load4_bf16(p.q + oq + lane * 4, qx);
      load4_bf16(p.v + ov + lane * 4, vx);
    }
    float sk = kx[0] * kx[0] + kx[1] * kx[1] + kx[2] * kx[2] + kx[3] * kx[3];
    float sq = qx[0] * qx[0] + qx[1] * qx[1] + qx[2] * qx[2] + qx[3] * qx[3];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sk += __shfl_xor_sync(0xffffffffu, sk, o);
      sq += __shfl_xor_sync(0xffffffffu, sq, o);
    }
    const float ik = 1.0f / sqrtf(sk + 1e-6f), iq = 1.0f / sqrtf(sq + 1e-6f);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      Kn[r * kP + lane * 4 + e] = kx[e] * ik;
      QW[r * kP + lane * 4 + e] = qx[e] * iq;
      VU[r * kP + lane * 4 + e] = vx[e];
    }
  }
  // ---- gate and log2-space chunk-local cumulative sum (thread per channel) ----
  if (tid < kD) {
    const int j = tid;
    const float a = expf(p.A_log[h]);
    const float db = p.dt_bias[h * kD + j];
    float acc = 0.0f;
    for (int r = 0; r < kChunk; ++r) {
      if (r < n) {
        const int64_t ov = row_offset(p.layout, p.Nv, p.S, b, h, tok0, t0 + r);
        const float x = __bfloat162float(p.g[ov + j]) + db;
        acc += p.lower_bound * sigmoidf_(a * x) * kLog2e;
      }
      Gs[r * kP + j] = acc;
    }
  } else if (tid < kD + kChunk) {
    const int r = tid - kD;
    float bv = 0.0f;
    if (r < n) bv = sigmoidf_(__bfloat162float(p.beta[beta_offset(p.layout, p.Nv, p.S, b, h, tok0, t0 + r)]));
    bet[r] = bv;
  }
  __syncthreads();

  float* wsc = reinterpret_cast<float*>(p.ws + kWsHeaderBytes + (size_t)gc * kWsChunkBytes);
  float* gW = wsc + kWsW / 4;
  float* gU = wsc + kWsU / 4;
  float* gQt = wsc + kWsQt / 4;
  float* gKh = wsc + kWsKh / 4;
  float* gAqk = wsc + kWsAqk / 4;
  float* gGc = wsc + kWsGc / 4;

  // ---- intra: per 16-row block I with reference row p0 = 16 I ----
  for (int I = 0; I < 4; ++I) {
    const int p0 = 16 * I;
    // A side (rows of block I): k_r 2^(G_r - G_p0) and q_r 2^(G_r - G_p0), both <= 1 in magnitude
    for (int e = tid; e < 16 * kD; e += 256) {
      const int rr = e / kD, j = e % kD;
      const int r = p0 + rr;
      const float f = exp2f(Gs[r * kP + j] - Gs[p0 * kP + j]);
      Ak[rr * kP + j] = Kn[r * kP + j] * f;
      Aq[rr * kP + j] = QW[r * kP + j] * f;
    }
    // B side (rows s < 16(I+1)): k_s 2^(G_p0 - G_s); <= 1 for s < p0, <= 2^(16*5/ln2) inside block
    for (int e = tid; e < 16 * (I + 1) * kD; e += 256) {
      const int s = e / kD, j = e % kD;
      Bk[s * kP + j] = Kn[s * kP + j] * exp2f(Gs[p0 * kP + j] - Gs[s * kP + j]);
    }
    __syncthreads();
    for (int m = 0; m <= I; ++m) {
      const int rr = tid & 15;
      const int s = (tid >> 4) + 16 * m;
      const int r = p0 + rr;
      float dk = 0.0f, dq = 0.0f;
#pragma unroll 8
      for (int j = 0; j < kD; ++j) {
        const float bs = Bk[s * kP + j];
        dk = fmaf(Ak[rr * kP + j], bs, dk);
        dq = fmaf(Aq[rr * kP + j], bs, dq);
      }
      T[r * (kChunk + 1) + s] = (s < r) ? bet[r] * dk : 0.0f;
      gAqk[r * kChunk + s] = (s <= r && r < n) ? p.scale * dq : 0.0f;
    }
    __syncthreads();
  }
  // upper part of T and Aqk (s >= 16(I+1)) is zero
  for (int e = tid; e < kChunk * kChunk; e += 256) {
    const int r = e / kChunk, s = e % kChunk;
    if (s >= 16 * (r / 16 + 1)) {
      T[r * (kChunk + 1) + s] = 0.0f;
      gAqk[r * kChunk + s] = 0.0f;
    }
  }
  // ---- Q~ = scale q 2^G,  K^ = k 2^(G_last - G),  gamma_last;  K~ = k 2^G into QW ----
  for (int e = tid; e < kChunk * kD; e += 256) {
    const int r = e / kD, j = e % kD;
    const float G = Gs[r * kP + j];
    const float Gl = Gs[(n - 1) * kP + j];
    const bool valid = r < n;
    gQt[e] = valid ? p.scale * QW[r * kP + j] * exp2f(G) : 0.0f;
    gKh[e] = valid ? Kn[r * kP + j] * exp2f(Gl - G) : 0.0f;
  }
  if (tid < kD) gGc[tid] = exp2f(Gs[(n - 1) * kP + tid]);
  __syncthreads();
  for (int e = tid; e < kChunk * kD; e += 256) {
    const int r = e / kD, j = e % kD;
    QW[r * kP + j] = (r < n) ? Kn[r * kP + j] * exp2f(Gs[r * kP + j]) : 0.0f;
  }
  __syncthreads();
  // ---- forward substitution: X_r = beta_r R_r - sum_{s<r} T[r][s] X_s (thread per column) ----
  {
    float* X = (tid < kD) ? QW : VU;
    const int col = tid & (kD - 1);
    for (int r = 0; r < n; ++r) {
      float acc = bet[r] * X[r * kP + col];
      for (int s = 0; s < r; ++s) acc = fmaf(-T[r * (kChunk + 1) + s], X[s * kP + col], acc);
      X[r * kP + col] = acc;
    }
  }
  __syncthreads();
  for (int e = tid; e < kChunk * kD; e += 256) {
    const int r = e / kD, j = e % kD;
    gW[e] = (r < n) ? QW[r * kP + j] : 0.0f;
    gU[e] = (r < n) ? VU[r * kP + j] : 0.0f;
  }
}

constexpr int kScanRows = 16;  // state rows (value dim) per scan CTA
constexpr size_t kSimtScanSmemBytes = (size_t)(kScanRows * kP + kChunk * (kScanRows + 1)) * 4;

__global__ void __launch_bounds__(256) kda_scan_simt_kernel(Params p) {
  if (!plan_ok(p)) {
    if (threadIdx.x == 0) atomicExch(p.status, DS_PLAN);
    return;
  }
  extern __shared__ float sm[];
  float* St = sm;                    // [16][kP] state rows i0..i0+15, all 128 key columns
  float* Dl = St + kScanRows * kP;   // [64][17] Delta for the 16 value columns of this tile
  const int tid = threadIdx.x;
  const int u = blockIdx.y;
  const int i0 = blockIdx.x * kScanRows;
  const int32_t* rec = p.plan + kPlanHeader + u * kPlanRecord;
  const int b = rec[PR_B], h = rec[PR_H], tok0 = rec[PR_TOK_START], L = rec[PR_LEN];
  const int nch = rec[PR_CHUNKS], off = rec[PR_CHUNK_OFFSET];
  const size_t sbase = ((size_t)b * p.Nv + h) * kD * kD;

  for (int e = tid; e < kScanRows * kD; e += 256) {
    const int ii = e / kD, j = e % kD;
    St[ii * kP + j] = p.S0 ? p.S0[sbase + (size_t)(i0 + ii) * kD + j] : 0.0f;
  }
  __syncthreads();

  const int r_a = tid >> 2;         // row for Delta / O (0..63)
  const int q_a = (tid & 3) * 4;    // first of 4 value columns (within the tile)
  const int j_c = tid & (kD - 1);   // key column for the state update
  const int ii_c = (tid >> 7) * 8;  // first of 8 state rows for the state update

  for (int c = 0; c < nch; ++c) {
    const float* wsc = reinterpret_cast<const float*>(p.ws + kWsHeaderBytes +
                                                      (size_t)(off + c) * kWsChunkBytes);
    const float* gW = wsc + kWsW / 4;
    const float* gU = wsc + kWsU / 4;
    const float* gQt = wsc + kWsQt / 4;
    const float* gKh = wsc + kWsKh / 4;
    const float* gAqk = wsc + kWsAqk / 4;
    const float* gGc = wsc + kWsGc / 4;
    const int n = min(kChunk, L - c * kChunk);

    // Delta = U - W S^T  and  O0 = Q~ S^T
    float dacc[4], oacc[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      dacc[e] = gU[r_a * kD + i0 + q_a + e];
      oacc[e] = 0.0f;
    }
    const float4* wrow = reinterpret_cast<const float4*>(gW + r_a * kD);
    const float4* qrow = reinterpret_cast<const float4*>(gQt + r_a * kD);
    for (int j4 = 0; j4 < kD / 4; ++j4) {
      const float4 w = __ldg(wrow + j4);
      const float4 qq = __ldg(qrow + j4);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float* srow = St + (q_a + e) * kP + j4 * 4;
        dacc[e] -= w.x * srow[0] + w.y * srow[1] + w.z * srow[2] + w.w * srow[3];
        oacc[e] += qq.x * srow[0] + qq.y * srow[1] + qq.z * srow[2] + qq.w * srow[3];
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) Dl[r_a * (kScanRows + 1) + q_a + e] = dacc[e];
    __syncthreads();
    // O += Aqk Delta  (Aqk is lower triangular with its diagonal)
    for (int s = 0; s <= r_a; ++s) {
      const float a = __ldg(gAqk + r_a * kChunk + s);
#pragma unroll
      for (int e = 0; e < 4; ++e) oacc[e] = fmaf(a, Dl[s * (kScanRows + 1) + q_a + e], oacc[e]);
    }
    if (r_a < n) {
      const int64_t oo = row_offset(p.layout, p.Nv, p.S, b, h, tok0, c * kChunk + r_a);
#pragma unroll
      for (int e = 0; e < 4; ++e) p.out[oo + i0 + q_a + e] = __float2bfloat16_rn(oacc[e]);
    }
    // S <- S Diag(gamma_last) + Delta^T K^
    float sacc[8];
    const float gl = __ldg(gGc + j_c);
#pragma unroll
    for (int e = 0; e < 8; ++e) sacc[e] = St[(ii_c + e) * kP + j_c] * gl;
    for (int r = 0; r < kChunk; ++r) {
      const float kh = __ldg(gKh + r * kD + j_c);
#pragma unroll
      for (int e = 0; e < 8; ++e) sacc[e] = fmaf(Dl[r * (kScanRows + 1) + ii_c + e], kh, sacc[e]);
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 8; ++e) St[(ii_c + e) * kP + j_c] = sacc[e];
    __syncthreads();
  }
  for (int e = tid; e < kScanRows * kD; e += 256) {
    const int ii = e / kD, j = e % kD;
    p.Sf[sbase + (size_t)(i0 + ii) * kD + j] = St[ii * kP + j];
  }
  // rows past the valid length (BNSD/BSND storage padding) are defined as zero
  if (p.layout != KDA_LAYOUT_TND) {
    for (int e = tid; e < (p.S - L) * kScanRows; e += 256) {
      const int t = L + e / kScanRows, ii = e % kScanRows;
      p.out[row_offset(p.layout, p.Nv, p.S, b, h, tok0, t) + i0 + ii] = __float2bfloat16_rn(0.0f);
    }
  }
}

cudaError_t launch_simt(const Params& p, int total_chunks, cudaStream_t stream) {
  static PerDevice setup;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int unused = 0;
  e = once_per_device(setup, dev, &unused, [](int, int*) {
    const cudaError_t r = cudaFuncSetAttribute(
        kda_chunk_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
        (int)kSimtChunkSmemBytes);
    if (r != cudaSuccess) return r;
    return cudaFuncSetAttribute(kda_scan_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kSimtScanSmemBytes);
  });
  if (e != cudaSuccess) return e;
  kda_chunk_simt_kernel<<<total_chunks, 256, kSimtChunkSmemBytes, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid(kD / kScanRows, p.n_units);
  kda_scan_simt_kernel<<<grid, 256, kSimtScanSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace kda
