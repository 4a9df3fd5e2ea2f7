// kda_layout.cuh -- kernel parameters and tensor addressing for the three FlashKDA layouts.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "kda_internal.h"

namespace kda {

struct Params {
  int layout, B, Nqk, Nv, S;
  int D;  // head dim of the tensors (64 or 128); the kernels compute at kD = 128 channels
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* g;
  const __nv_bfloat16* beta;
  float scale;
  const float* S0;  // may be null (zero initial state)
  const float* A_log;
  const float* dt_bias;
  float lower_bound;
  const int32_t* plan;  // device copy
  int32_t plan_checksum;
  int n_units;
  uint8_t* ws;
  int32_t* status;
  __nv_bfloat16* out;
  float* Sf;
  unsigned long long* tprof;  // optional: CTA 0 records clock64() at phase boundaries
  // work items of this launch: mode 0 = whole units; under a segmented plan (seg_chunks > 0)
  // mode 1 = the segment-summary pass, mode 2 = the output pass (see kda_plan_segmented)
  // mode 3 = the per-unit affine summary (M, R) of kda_forward_summary
  int mode, seg_chunks, n_items;
  float* states;  // the segmented schedule's state slots (workspace after its header)
  float* sum_m;   // mode 3: every unit's M and R, fp32 [B, Nv, D, D] each
  float* sum_r;
};

// Element offset of the D-vector of (sequence b, head hx of NX heads, token t of the sequence).
// BNSD [B,NX,S,D], BSND [B,S,NX,D], TND [T,NX,D] with the sequence starting at packed row tok0.
__device__ __forceinline__ int64_t row_offset(int layout, int NX, int S, int b, int hx, int tok0,
                                              int t, int D = kD) {
  if (layout == KDA_LAYOUT_BNSD) return (((int64_t)b * NX + hx) * S + t) * D;
  if (layout == KDA_LAYOUT_BSND) return (((int64_t)b * S + t) * NX + hx) * D;
  return ((int64_t)(tok0 + t) * NX + hx) * D;
}

// Offset of beta for (b, value head h, token t): BNSD [B,Nv,S], BSND [B,S,Nv], TND [T,Nv].
__device__ __forceinline__ int64_t beta_offset(int layout, int Nv, int S, int b, int h, int tok0,
                                               int t) {
  if (layout == KDA_LAYOUT_BNSD) return ((int64_t)b * Nv + h) * S + t;
  if (layout == KDA_LAYOUT_BSND) return ((int64_t)b * S + t) * Nv + h;
  return (int64_t)(tok0 + t) * Nv + h;
}

__device__ __forceinline__ void load4_bf16(const __nv_bfloat16* p, float x[4]) {
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(p));
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
  const __nv_bfloat162 c = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
  x[0] = __low2float(a);
  x[1] = __high2float(a);
  x[2] = __low2float(c);
  x[3] = __high2float(c);
}

// The two-kernel fp32 CUDA-core path (kda_simt.cu): needs kWsHeaderBytes + total_chunks *
// kWsChunkBytes of workspace.
cudaError_t launch_simt(const Params& p, int total_chunks, cudaStream_t stream);
// The fused tcgen05 path (kda_fused.cu): needs kWsHeaderBytes of workspace.  A non-null `dbg`
// receives every chunk's intermediates in the two-kernel workspace layout (test aid).
// dyn_items (mode 0 only): units are claimed dynamically, longest first, from an item counter at
// workspace offset 4, which must be zero at the launch
cudaError_t launch_fused(const Params& p, float* dbg, cudaStream_t stream, bool dyn_items = false);
// The segmented schedule's middle kernel: every unit's segment start states from the segment
// summaries (S_{s+1} = S_s M_s + R_s, fp32).
cudaError_t launch_combine(const Params& p, cudaStream_t stream);
// kda_forward_summary under a segmented plan: composes every unit's segment maps into sum_m /
// sum_r (which hold segment 0's).
cudaError_t launch_summary_combine(const Params& p, cudaStream_t stream);
// kda_state_chain's kernel: S_out[u] = fold of S <- S M_j[u] + R_j[u] from S_in[u] (null: 0);
// step j's maps start step_stride floats after step j-1's.
cudaError_t launch_chain(int units, int D, int n_steps, const float* S_in, const float* M,
                         const float* R, size_t step_stride, float* S_out, cudaStream_t stream);

enum ForwardPath : int { PATH_FUSED = 0, PATH_SIMT = 1, PATH_SUMMARY = 2 };

// Shared body of the forward entry points: every host check, then the launches of `path`.
kda_status_t forward_impl(int path, const kda_shape_t* shape, const int32_t* plan_host,
                          const int32_t* plan_dev, size_t n_int32, const void* q, const void* k,
                          const void* v, const void* g, const void* beta, float scale,
                          const float* initial_state, const float* A_log, const float* dt_bias,
                          float lower_bound, void* workspace, size_t workspace_bytes, void* out,
                          float* final_state, cudaStream_t stream, float* dbg,
                          unsigned long long* tprof = nullptr, float* sum_m = nullptr);

// Workspace bytes of the two-kernel path for a validated plan.
size_t simt_workspace_bytes(const int32_t* plan);

}  // namespace kda
