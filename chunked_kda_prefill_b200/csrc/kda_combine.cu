// kda_combine.cu -- state chaining through per-span affine maps: the middle kernel of the
// segmented (chunk-parallel) schedule (every unit's segment start states from the segment
// summaries), and kda_state_chain (the same fold over maps laid out step-major, the start-state
// step of context parallelism).
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
#include "kda_once.h"

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

// The chain S <- S M_j + R_j for j = 0 .. n-1 over this CTA's rows r0 .. r0+7 of a D x D state
// (row length D), starting from S_start (null: zeros; R_j null: zero).  After step j the rows go to dst_at(j)
// when that is not null.  M_{j+1} streams into shared memory while step j computes (cp.async,
// double-buffered), R_{j+1} into registers; only S is carried from step to step.  2 D threads:
// thread = (4-row group rg, column col).
template <int D, class MF, class RF, class DF>
__device__ __forceinline__ void chain_rows(float* sM, float* sS, const float* S_start, int n,
                                           int r0, MF m_at, RF r_at, DF dst_at) {
  constexpr int kThreadsC = 2 * D;
  const int tid = threadIdx.x, rg = tid / D, col = tid % D;
  auto load_m = [&](int j) {  // M_j -> buffer j & 1, D/8 x 16 bytes per thread
    const float* src = m_at(j);
    float* dst = sM + (size_t)(j & 1) * D * D;
    for (int e = tid; e < D * D / 4; e += kThreadsC) cp_async16(dst + 4 * e, src + 4 * e);
  };
  auto load_r = [&](int j, float (&r)[4]) {  // this thread's 4 entries of R_j (null: zero)
    const float* src = r_at(j);
#pragma unroll
    for (int i = 0; i < 4; ++i) r[i] = src ? src[(size_t)(r0 + 4 * rg + i) * D + col] : 0.f;
  };

  for (int e = tid; e < kRowsC * D / 4; e += kThreadsC)
    *reinterpret_cast<float4*>(sS + 4 * e) =
        S_start ? *reinterpret_cast<const float4*>(S_start + (size_t)r0 * D + 4 * e)
                : make_float4(0.f, 0.f, 0.f, 0.f);
  if (n <= 0) return;
  load_m(0);
  cp_async_commit();
  float r_cur[4];
  load_r(0, r_cur);

  for (int j = 0; j < n; ++j) {
    if (j + 1 < n) load_m(j + 1);
    cp_async_commit();  // (an empty group on the last step keeps the wait count uniform)
    float r_next[4] = {0.f, 0.f, 0.f, 0.f};
    if (j + 1 < n) load_r(j + 1, r_next);
    cp_async_wait_one();
    __syncthreads();  // M_j (everyone's copies) and S are in shared memory
    const float* M = sM + (size_t)(j & 1) * D * D;
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
    __syncthreads();  // every read of S and of this M buffer is done
    float* dst = dst_at(j);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (dst) dst[(size_t)(r0 + 4 * rg + i) * D + col] = acc[i];
      sS[(4 * rg + i) * D + col] = acc[i];
      r_cur[i] = r_next[i];
    }
  }
}

// Segmented schedule: S_{s+1} = S_s M_s + R_s for s = 1 .. nseg-2 from the state slots.
template <int D>
__global__ void __launch_bounds__(2 * D) kda_combine_kernel(const Params p) {
  extern __shared__ __align__(16) float csm[];
  const int u = blockIdx.x, r0 = blockIdx.y * kRowsC;
  const int32_t* rec = p.plan + kPlanHeader + u * kPlanRecord;
  const int seg = p.seg_chunks;
  const int nseg = (rec[PR_CHUNKS] + seg - 1) / seg;
  const int base = rec[PR_SEG_BASE];
  if (nseg < 3) return;  // S_1 comes from the first pass; nothing to chain
  auto slot = [&](int sl, int part) {
    return p.states + (size_t)sl * kSlotFloats + (size_t)part * kD * kD;
  };
  // step j = s - 1 uses segment s's map (slot base + s - 1) and writes segment s+1's start
  chain_rows<D>(csm, csm + 2 * D * D, slot(base, SLOT_START), nseg - 2, r0,
                [&](int j) { return (const float*)slot(base + j, SLOT_M); },
                [&](int j) { return (const float*)slot(base + j, SLOT_R); },
                [&](int j) { return slot(base + j + 1, SLOT_START); });
}

// kda_forward_summary under a segmented plan: unit u's maps from its segments' maps,
//     M = M_0 M_1 ... M_{n-1},   R = (((R_0 M_1 + R_1) M_2 + R_2) ...) M_{n-1} + R_{n-1},
// composed in place in sum_m / sum_r (which hold segment 0's maps) through the state slots of
// segments 1 .. n-1.  blockIdx.z: 0 composes M, 1 composes R.
template <int D>
__global__ void __launch_bounds__(2 * D) kda_summary_combine_kernel(const Params p) {
  extern __shared__ __align__(16) float csm[];
  const int u = blockIdx.x, r0 = blockIdx.y * kRowsC;
  const bool r_side = blockIdx.z == 1;
  const int32_t* rec = p.plan + kPlanHeader + u * kPlanRecord;
  const int seg = p.seg_chunks;
  const int nseg = (rec[PR_CHUNKS] + seg - 1) / seg;
  const int base = rec[PR_SEG_BASE];
  if (nseg < 2) return;  // one segment: its maps are the unit's
  float* buf = (r_side ? p.sum_r : p.sum_m) + ((size_t)rec[PR_B] * p.Nv + rec[PR_H]) * D * D;
  auto slot = [&](int sl, int part) {
    return p.states + (size_t)sl * kSlotFloats + (size_t)part * kD * kD;
  };
  chain_rows<D>(csm, csm + 2 * D * D, buf, nseg - 1, r0,
                [&](int j) { return (const float*)slot(base + j, SLOT_M); },
                [&](int j) { return r_side ? (const float*)slot(base + j, SLOT_R) : nullptr; },
                [&](int j) { return j == nseg - 2 ? buf : (float*)nullptr; });
}

// kda_state_chain: S_out[u] = fold of S <- S M_j[u] + R_j[u], j = 0 .. n-1, from S_in[u].
struct ChainParams {
  int units, n_steps;
  size_t step_stride;  // floats from step j's maps to step j+1's
  const float* S_in;   // [units][D][D] or null (zeros)
  const float* M;      // step j: [units][D][D] at M + j * step_stride
  const float* R;      // likewise
  float* S_out;        // [units][D][D]
};

template <int D>
__global__ void __launch_bounds__(2 * D) kda_chain_kernel(const ChainParams c) {
  extern __shared__ __align__(16) float csm[];
  const int u = blockIdx.x, r0 = blockIdx.y * kRowsC;
  const size_t mat = (size_t)D * D;
  const float* start = c.S_in ? c.S_in + u * mat : nullptr;
  float* out = c.S_out + u * mat;
  float* sS = csm + 2 * D * D;
  chain_rows<D>(csm, sS, start, c.n_steps, r0,
                [&](int j) { return c.M + (size_t)j * c.step_stride + u * mat; },
                [&](int j) { return c.R + (size_t)j * c.step_stride + u * mat; },
                [&](int j) { return j == c.n_steps - 1 ? out : (float*)nullptr; });
  if (c.n_steps <= 0) {  // no step: S_out = S_in (or zeros)
    __syncthreads();
    for (int e = threadIdx.x; e < kRowsC * D; e += 2 * D)
      out[(size_t)r0 * D + e] = sS[e];
  }
}

}  // namespace

cudaError_t launch_combine(const Params& p, cudaStream_t stream) {
  static PerDevice setup;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int unused = 0;
  e = once_per_device(setup, dev, &unused, [](int, int*) {
    const cudaError_t r = cudaFuncSetAttribute(kda_combine_kernel<kD>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)combine_smem<kD>());
    if (r != cudaSuccess) return r;
    return cudaFuncSetAttribute(kda_combine_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)combine_smem<64>());
  });
  if (e != cudaSuccess) return e;
  if (p.D == kD) {
    const dim3 grid((unsigned)p.n_units, kD / kRowsC);
    kda_combine_kernel<kD><<<grid, 2 * kD, combine_smem<kD>(), stream>>>(p);
  } else {
    const dim3 grid((unsigned)p.n_units, 64 / kRowsC);
    kda_combine_kernel<64><<<grid, 2 * 64, combine_smem<64>(), stream>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_summary_combine(const Params& p, cudaStream_t stream) {
  static PerDevice setup;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int unused = 0;
  e = once_per_device(setup, dev, &unused, [](int, int*) {
    const cudaError_t r = cudaFuncSetAttribute(kda_summary_combine_kernel<kD>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)combine_smem<kD>());
    if (r != cudaSuccess) return r;
    return cudaFuncSetAttribute(kda_summary_combine_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)combine_smem<64>());
  });
  if (e != cudaSuccess) return e;
  if (p.D == kD) {
    kda_summary_combine_kernel<kD><<<dim3((unsigned)p.n_units, kD / kRowsC, 2), 2 * kD,
                                     combine_smem<kD>(), stream>>>(p);
  } else {
    kda_summary_combine_kernel<64><<<dim3((unsigned)p.n_units, 64 / kRowsC, 2), 2 * 64,
                                     combine_smem<64>(), stream>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_chain(int units, int D, int n_steps, const float* S_in, const float* M,
                         const float* R, size_t step_stride, float* S_out, cudaStream_t stream) {
  static PerDevice setup;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int unused = 0;
  e = once_per_device(setup, dev, &unused, [](int, int*) {
    const cudaError_t r = cudaFuncSetAttribute(kda_chain_kernel<kD>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)combine_smem<kD>());
    if (r != cudaSuccess) return r;
    return cudaFuncSetAttribute(kda_chain_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)combine_smem<64>());
  });
  if (e != cudaSuccess) return e;
  const ChainParams c{units, n_steps, step_stride, S_in, M, R, S_out};
  if (D == kD) {
    kda_chain_kernel<kD><<<dim3((unsigned)units, kD / kRowsC), 2 * kD, combine_smem<kD>(),
                           stream>>>(c);
  } else {
    kda_chain_kernel<64><<<dim3((unsigned)units, 64 / kRowsC), 2 * 64, combine_smem<64>(),
                           stream>>>(c);
  }
  return cudaGetLastError();
}

}  // namespace kda
