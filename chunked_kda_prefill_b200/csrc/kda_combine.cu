// kda_combine.cu -- the middle kernel of the segmented (chunk-parallel) schedule: every unit's
// segment start states from the segment summaries.
//
// Per chunk the state update is affine in the start state (FlashKDA README chunk equations,
// 功能说明): S_next = S Diag(gamma_C) + (U - W S^T)^T K^ = S M + R with M = Diag(gamma_C) - W^T K^
// and R = U^T K^, so a segment of chunks maps S to S M_s + R_s.  The first pass leaves M_s and
// R_s of every segment s >= 1 in its state slot, and the true start state of segment 1 (the end
// state of segment 0).  Here, per unit and in segment order,
//     S_{s+1} = S_s M_s + R_s        (fp32, D x D x D per step, D = 128 or 64)
// for s = 1 .. nseg-2.  Rows of S are independent, so a unit's D rows are split over D/8 CTAs
// of 8 rows.  Every M_s is known before the kernel starts, so M_{s+1} streams into shared memory
// (cp.async, double-buffered) while step s computes; only S_s is carried from step to step.
// A slot part holds a D x D matrix with row length D (the first D*D floats of its 128 x 128
// space), as the fused kernel writes it.
#include <cuda_runtime.h>

#include "kda_internal.h"
#include "kda_layout.cuh"

namespace kda {
namespace {

constexpr int kRowsC = 8;  // state rows per CTA; 2 D threads = (4-row group, column)
template <int D>
constexpr size_t combine_smem() { return (2 * D * D + kRowsC * D) * sizeof(float); }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_one() {  // all but the newest group complete
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

template <int D>
__global__ void __launch_bounds__(2 * D) kda_combine_kernel(const Params p) {
  constexpr int kThreadsC = 2 * D;
  extern __shared__ __align__(16) float csm[];
  float* sM = csm;               // [2][D][D]: M of the current and the next step
  float* sS = csm + 2 * D * D;   // [8][D]: this CTA's rows of S_s
  const int u = blockIdx.x, r0 = blockIdx.y * kRowsC;
  const int32_t* rec = p.plan + kPlanHeader + u * kPlanRecord;
  const int seg = p.seg_chunks;
  const int nseg = (rec[PR_CHUNKS] + seg - 1) / seg;
  const int base = rec[PR_SEG_BASE];
  if (nseg < 3) return;  // S_1 comes from the first pass; nothing to chain
  const int tid = threadIdx.x, rg = tid / D, col = tid % D;
  auto slot = [&](int sl, int part) {
    return p.states + (size_t)sl * kSlotFloats + (size_t)part * kD * kD;
  };
  auto load_m = [&](int s) {  // M_s -> buffer (s - 1) & 1, D/8 x 16 bytes per thread
    const float* src = slot(base + s - 1, SLOT_M);
    float* dst = sM + (size_t)((s - 1) & 1) * D * D;
    for (int e = tid; e < D * D / 4; e += kThreadsC) cp_async16(dst + 4 * e, src + 4 * e);
  };
  auto load_r = [&](int s, float (&r)[4]) {  // this thread's 4 entries of R_s
    const float* src = slot(base + s - 1, SLOT_R);
#pragma unroll
    for (int i = 0; i < 4; ++i) r[i] = src[(size_t)(r0 + 4 * rg + i) * D + col];
  };

  for (int e = tid; e < kRowsC * D / 4; e += kThreadsC)
    *reinterpret_cast<float4*>(sS + 4 * e) =
        *reinterpret_cast<const float4*>(slot(base, SLOT_START) + (size_t)r0 * D + 4 * e);
  load_m(1);
  cp_async_commit();
  float r_cur[4];
  load_r(1, r_cur);

  for (int s = 1; s <= nseg - 2; ++s) {
    if (s + 1 <= nseg - 2) load_m(s + 1);
    cp_async_commit();  // (an empty group on the last step keeps the wait count uniform)
    float r_next[4] = {0.f, 0.f, 0.f, 0.f};
    if (s + 1 <= nseg - 2) load_r(s + 1, r_next);
    cp_async_wait_one();
    __syncthreads();  // M_s (everyone's copies) and S_s are in shared memory
    const float* M = sM + (size_t)((s - 1) & 1) * D * D;
    float acc[4] = {r_cur[0], r_cur[1], r_cur[2], r_cur[3]};
#pragma unroll 4
    for (int k = 0; k < D; k += 4) {
      const float m0 = M[(k + 0) * D + col], m1 = M[(k + 1) * D + col];
      const float m2 = M[(k + 2) * D + col], m3 = M[(k + 3) * D + col];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 sv = *reinterpret_cast<const float4*>(sS + (4 * rg + i) * D + k);
        acc[i] = fmaf(sv.x, m0, fmaf(sv.y, m1, fmaf(sv.z, m2, fmaf(sv.w, m3, acc[i]))));
      }
    }
    __syncthreads();  // every read of S_s and of this M buffer is done
    float* dst = slot(base + s, SLOT_START);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      dst[(size_t)(r0 + 4 * rg + i) * D + col] = acc[i];
      sS[(4 * rg + i) * D + col] = acc[i];
      r_cur[i] = r_next[i];
    }
  }
}

}  // namespace

cudaError_t launch_combine(const Params& p, cudaStream_t stream) {
  static int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(kda_combine_kernel<kD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)combine_smem<kD>());
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kda_combine_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)combine_smem<64>());
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  if (p.D == kD) {
    const dim3 grid((unsigned)p.n_units, kD / kRowsC);
    kda_combine_kernel<kD><<<grid, 2 * kD, combine_smem<kD>(), stream>>>(p);
  } else {
    const dim3 grid((unsigned)p.n_units, 64 / kRowsC);
    kda_combine_kernel<64><<<grid, 2 * 64, combine_smem<64>(), stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace kda
