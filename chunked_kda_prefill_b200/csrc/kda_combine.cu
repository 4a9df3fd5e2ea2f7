// kda_combine.cu -- the middle kernel of the segmented (chunk-parallel) schedule: every unit's
// segment start states from the segment summaries.
//
// Per chunk the state update is affine in the start state (FlashKDA README chunk equations,
// 功能说明): S_next = S Diag(gamma_C) + (U - W S^T)^T K^ = S M + R with M = Diag(gamma_C) - W^T K^
// and R = U^T K^, so a segment of chunks maps S to S M_s + R_s.  The first pass leaves M_s and
// R_s of every segment s >= 1 in its state slot, and the true start state of segment 1 (the end
// state of segment 0).  Here, per unit and in segment order,
//     S_{s+1} = S_s M_s + R_s        (fp32, 128 x 128 x 128 per step)
// for s = 1 .. nseg-2.  Rows of S are independent, so a unit's 128 rows are split over 8 CTAs
// of 16 rows; each CTA streams M_s through shared memory in 16-row slices.
#include <cuda_runtime.h>

#include "kda_internal.h"
#include "kda_layout.cuh"

namespace kda {
namespace {

constexpr int kRows = 16;      // state rows per CTA
constexpr int kKSlice = 16;    // rows of M per shared-memory slice
constexpr int kThreadsC = 256;  // thread = (row, 8-column group)

__global__ void __launch_bounds__(kThreadsC) kda_combine_kernel(const Params p) {
  __shared__ __align__(16) float sS[kRows][kD];
  __shared__ __align__(16) float sM[kKSlice][kD];
  const int u = blockIdx.x, r0 = blockIdx.y * kRows;
  const int32_t* rec = p.plan + kPlanHeader + u * kPlanRecord;
  const int seg = p.seg_chunks;
  const int nseg = (rec[PR_CHUNKS] + seg - 1) / seg;
  const int base = rec[PR_SEG_BASE];
  if (nseg < 3) return;  // S_1 comes from the first pass; nothing to chain
  const int tid = threadIdx.x, r = tid >> 4, c0 = (tid & 15) * 8;
  auto slot = [&](int sl, int part) {
    return p.states + (size_t)sl * kSlotFloats + (size_t)part * kD * kD;
  };
  // S_1 rows
  for (int e = tid; e < kRows * kD / 4; e += kThreadsC) {
    const int rr = e / (kD / 4), cc = (e % (kD / 4)) * 4;
    *reinterpret_cast<float4*>(&sS[rr][cc]) =
        *reinterpret_cast<const float4*>(slot(base, SLOT_START) + (size_t)(r0 + rr) * kD + cc);
  }
  __syncthreads();
  for (int s = 1; s <= nseg - 2; ++s) {
    const float* M = slot(base + s - 1, SLOT_M);
    const float* R = slot(base + s - 1, SLOT_R) + (size_t)(r0 + r) * kD + c0;
    float acc[8];
    {
      const float4 a = *reinterpret_cast<const float4*>(R);
      const float4 b = *reinterpret_cast<const float4*>(R + 4);
      acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w;
      acc[4] = b.x; acc[5] = b.y; acc[6] = b.z; acc[7] = b.w;
    }
    for (int k0 = 0; k0 < kD; k0 += kKSlice) {
      for (int e = tid; e < kKSlice * kD / 4; e += kThreadsC) {
        const int kk = e / (kD / 4), cc = (e % (kD / 4)) * 4;
        *reinterpret_cast<float4*>(&sM[kk][cc]) =
            *reinterpret_cast<const float4*>(M + (size_t)(k0 + kk) * kD + cc);
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kKSlice; ++kk) {
        const float sv = sS[r][k0 + kk];
        const float4 a = *reinterpret_cast<const float4*>(&sM[kk][c0]);
        const float4 b = *reinterpret_cast<const float4*>(&sM[kk][c0 + 4]);
        acc[0] = fmaf(sv, a.x, acc[0]);
        acc[1] = fmaf(sv, a.y, acc[1]);
        acc[2] = fmaf(sv, a.z, acc[2]);
        acc[3] = fmaf(sv, a.w, acc[3]);
        acc[4] = fmaf(sv, b.x, acc[4]);
        acc[5] = fmaf(sv, b.y, acc[5]);
        acc[6] = fmaf(sv, b.z, acc[6]);
        acc[7] = fmaf(sv, b.w, acc[7]);
      }
      __syncthreads();
    }
    // S_{s+1}: to its slot, and to shared memory for the next step
    float* dst = slot(base + s, SLOT_START) + (size_t)(r0 + r) * kD + c0;
    *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    *reinterpret_cast<float4*>(&sS[r][c0]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4*>(&sS[r][c0 + 4]) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_combine(const Params& p, cudaStream_t stream) {
  const dim3 grid((unsigned)p.n_units, kD / kRows);
  kda_combine_kernel<<<grid, kThreadsC, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace kda
