// kda_api.cu -- kda_forward / kda_device_status: argument checks, then the kernel launches.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>

#include "kda_internal.h"
#include "kda_layout.cuh"
#include "kda_once.h"

namespace kda {
namespace {

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};

bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

Range range_of(const void* p, size_t bytes) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return {lo, lo + bytes};
}

// Checks that the current device is an sm_100 part; the compute capability is cached per device
// ordinal.
kda_status_t check_device() {
  static PerDevice major_of;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
  int major = 0;
  if (once_per_device(major_of, dev, &major, [](int d, int* m) {
        return cudaDeviceGetAttribute(m, cudaDevAttrComputeCapabilityMajor, d);
      }) != cudaSuccess)
    return KDA_ERR_CUDA;
  return major == 10 ? KDA_OK : KDA_ERR_DEVICE;
}

}  // namespace

size_t simt_workspace_bytes(const int32_t* plan) {
  return kWsHeaderBytes + (size_t)plan[PH_TOTAL_CHUNKS] * kWsChunkBytes;
}

kda_status_t forward_impl(int path, const kda_shape_t* shape, const int32_t* plan_host,
                          const int32_t* plan_dev, size_t n_int32, const void* q, const void* k,
                          const void* v, const void* g, const void* beta, float scale,
                          const float* initial_state, const float* A_log, const float* dt_bias,
                          float lower_bound, void* workspace, size_t workspace_bytes, void* out,
                          float* final_state, cudaStream_t stream, float* dbg,
                          unsigned long long* tprof, float* sum_m) {
  kda_status_t st = validate_shape(shape);
  if (st != KDA_OK) return st;
  const bool summary = (path == PATH_SUMMARY);  // final_state receives R, sum_m M; no out
  if (!plan_host || !plan_dev || !q || !k || !v || !g || !beta || !A_log || !dt_bias ||
      !workspace || (!out && !summary) || !final_state || (summary && !sum_m))
    return KDA_ERR_NULL;
  st = validate_plan(plan_host, n_int32, shape);
  if (st != KDA_OK) return st;
  if (path == PATH_SIMT && shape->D != kD) return KDA_ERR_DIM;  // the fp32 path is D = 128 only
  if (!std::isfinite(scale)) return KDA_ERR_LOWER_BOUND;
  if (!(lower_bound >= -5.0f && lower_bound <= 0.0f)) return KDA_ERR_LOWER_BOUND;
  {
    const void* a16[] = {q, k, v, g, out, final_state, A_log, dt_bias, plan_dev, initial_state,
                         sum_m};
    for (const void* ptr : a16)
      if (reinterpret_cast<uintptr_t>(ptr) & 15u) return KDA_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(beta) & 1u) return KDA_ERR_ALIGN;
  }
  const size_t need =
      (path == PATH_SIMT) ? simt_workspace_bytes(plan_host) : fused_workspace_bytes(plan_host);
  if (workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return KDA_ERR_WORKSPACE;

  // aliasing: outputs must not overlap any input or each other
  const long long rows =
      shape->layout == KDA_LAYOUT_TND ? (long long)shape->S : (long long)shape->B * shape->S;
  const size_t D = (size_t)shape->D;
  const size_t qk_bytes = (size_t)rows * shape->Nqk * D * 2;
  const size_t vg_bytes = (size_t)rows * shape->Nv * D * 2;
  const size_t beta_bytes = (size_t)rows * shape->Nv * 2;
  const size_t st_bytes = (size_t)shape->B * shape->Nv * D * D * 4;
  const Range r_out = summary ? Range{0, 0} : range_of(out, vg_bytes);
  const Range r_fs = range_of(final_state, st_bytes);
  const Range r_m = summary ? range_of(sum_m, st_bytes) : Range{0, 0};
  const Range ins[] = {range_of(q, qk_bytes), range_of(k, qk_bytes), range_of(v, vg_bytes),
                       range_of(g, vg_bytes), range_of(beta, beta_bytes),
                       range_of(workspace, need), range_of(plan_dev, n_int32 * 4),
                       initial_state ? range_of(initial_state, st_bytes) : Range{0, 0}};
  for (const Range& r : ins) {
    if (r.hi == 0) continue;
    if (overlaps(r, r_out) || overlaps(r, r_fs) || overlaps(r, r_m)) return KDA_ERR_ALIAS;
  }
  if (overlaps(r_out, r_fs) || overlaps(r_m, r_fs)) return KDA_ERR_ALIAS;

  st = check_device();
  if (st != KDA_OK) return st;

  Params p{};
  p.layout = shape->layout;
  p.B = shape->B;
  p.Nqk = shape->Nqk;
  p.Nv = shape->Nv;
  p.S = shape->S;
  p.D = shape->D;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.g = static_cast<const __nv_bfloat16*>(g);
  p.beta = static_cast<const __nv_bfloat16*>(beta);
  p.scale = scale;
  p.S0 = initial_state;
  p.A_log = A_log;
  p.dt_bias = dt_bias;
  p.lower_bound = lower_bound;
  p.plan = plan_dev;
  p.plan_checksum = plan_host[PH_CHECKSUM];
  p.n_units = plan_host[PH_UNITS];
  p.ws = static_cast<uint8_t*>(workspace);
  p.status = static_cast<int32_t*>(workspace);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.Sf = final_state;
  p.tprof = tprof;

  p.seg_chunks = plan_host[PH_SEG_CHUNKS];
  p.states = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWsHeaderBytes);

  // the status word and the item counter of a dynamically scheduled launch
  if (cudaMemsetAsync(workspace, 0, 8, stream) != cudaSuccess) return KDA_ERR_CUDA;
  cudaError_t e;
  if (path == PATH_SIMT) {
    e = launch_simt(p, plan_host[PH_TOTAL_CHUNKS], stream);
  } else if (summary) {
    // every unit (or, under a segmented plan, every segment) twice: from S = 0 (R) and from
    // S = I with v = 0 (M); segment maps are then composed into the unit's
    const long long items =
        2LL * (p.seg_chunks > 0 ? seg_counts(plan_host).slots + p.n_units : p.n_units);
    if (items > INT_MAX) return KDA_ERR_SHAPE;
    p.mode = 3;
    p.n_items = (int)items;
    p.S0 = nullptr;
    p.sum_m = sum_m;
    p.sum_r = final_state;
    e = launch_fused(p, dbg, stream);
    if (e == cudaSuccess && p.seg_chunks > 0) e = launch_summary_combine(p, stream);
  } else if (p.seg_chunks <= 0) {
    p.mode = 0;
    p.n_items = p.n_units;
    // units of different lengths are claimed dynamically, longest first (the plan's order), by
    // whichever CTA frees up first; equal units keep the fixed stride
    const int32_t* R = plan_host + kPlanHeader;
    int lo = INT_MAX, hi = 0;
    for (int u = 0; u < p.n_units; ++u) {
      lo = std::min(lo, (int)R[u * kPlanRecord + PR_CHUNKS]);
      hi = std::max(hi, (int)R[u * kPlanRecord + PR_CHUNKS]);
    }
    e = launch_fused(p, dbg, stream, hi > lo);
  } else {
    // segmented schedule: segment summaries, start states, outputs
    const SegCounts sc = seg_counts(plan_host);
    if (sc.items_a > INT_MAX) return KDA_ERR_SHAPE;
    p.mode = 1;
    p.n_items = (int)sc.items_a;
    e = launch_fused(p, dbg, stream);
    if (e == cudaSuccess) e = launch_combine(p, stream);
    if (e == cudaSuccess && sc.items_c > 0) {
      p.mode = 2;
      p.n_items = (int)sc.items_c;
      e = launch_fused(p, dbg, stream);
    }
  }
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace kda

using namespace kda;

extern "C" kda_status_t kda_forward(const kda_shape_t* shape, const int32_t* plan_host,
                                    const int32_t* plan_dev, size_t n_int32, const void* q,
                                    const void* k, const void* v, const void* g, const void* beta,
                                    float scale, const float* initial_state, const float* A_log,
                                    const float* dt_bias, float lower_bound, void* workspace,
                                    size_t workspace_bytes, void* out, float* final_state,
                                    kda_stream_t stream) {
  return forward_impl(PATH_FUSED, shape, plan_host, plan_dev, n_int32, q, k, v, g, beta, scale,
                      initial_state, A_log, dt_bias, lower_bound, workspace, workspace_bytes, out,
                      final_state, reinterpret_cast<cudaStream_t>(stream), nullptr);
}

extern "C" kda_status_t kda_forward_summary(const kda_shape_t* shape, const int32_t* plan_host,
                                            const int32_t* plan_dev, size_t n_int32,
                                            const void* q, const void* k, const void* v,
                                            const void* g, const void* beta, const float* A_log,
                                            const float* dt_bias, float lower_bound,
                                            void* workspace, size_t workspace_bytes,
                                            float* M_out, float* R_out, kda_stream_t stream) {
  // scale only weights the outputs, which a summary does not write
  return forward_impl(PATH_SUMMARY, shape, plan_host, plan_dev, n_int32, q, k, v, g, beta, 1.0f,
                      nullptr, A_log, dt_bias, lower_bound, workspace, workspace_bytes, nullptr,
                      R_out, reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr, M_out);
}

extern "C" kda_status_t kda_state_chain(int32_t units, int32_t D, int32_t n_steps,
                                        const float* S_in, const float* M, const float* R,
                                        int64_t step_stride, float* S_out, kda_stream_t stream) {
  if (D != kD && D != 64) return KDA_ERR_DIM;
  if (units < 1 || n_steps < 0 || (long long)units > INT_MAX / 2) return KDA_ERR_SHAPE;
  const long long mat_floats = (long long)units * D * D;
  if (step_stride == 0) step_stride = mat_floats;
  if (step_stride < mat_floats || (step_stride & 3)) return KDA_ERR_SHAPE;
  if (!S_out || (n_steps > 0 && (!M || !R))) return KDA_ERR_NULL;
  const void* a16[] = {S_in, M, R, S_out};
  for (const void* ptr : a16)
    if (reinterpret_cast<uintptr_t>(ptr) & 15u) return KDA_ERR_ALIGN;
  const size_t st_bytes = (size_t)units * D * D * 4;
  const size_t maps_bytes =
      n_steps > 0 ? ((size_t)(n_steps - 1) * (size_t)step_stride) * 4 + st_bytes : 0;
  const Range r_out = range_of(S_out, st_bytes);
  // S_out may be S_in itself (each CTA reads its rows before it writes them), no other overlap
  if (S_in && S_in != S_out && overlaps(range_of(S_in, st_bytes), r_out)) return KDA_ERR_ALIAS;
  if (n_steps > 0 && (overlaps(range_of(M, maps_bytes), r_out) ||
                      overlaps(range_of(R, maps_bytes), r_out)))
    return KDA_ERR_ALIAS;
  kda_status_t st = check_device();
  if (st != KDA_OK) return st;
  return launch_chain(units, D, n_steps, S_in, M, R, (size_t)step_stride, S_out,
                      reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KDA_OK
             : KDA_ERR_CUDA;
}

// ---- internal entry points for the GPU tests (not part of include/kda.h) ----

// The two-kernel fp32 CUDA-core path, with a caller workspace of kda_simt_workspace_size bytes.
extern "C" __attribute__((visibility("default"))) kda_status_t kda_forward_simt(
    const kda_shape_t* shape, const int32_t* plan_host, const int32_t* plan_dev, size_t n_int32,
    const void* q, const void* k, const void* v, const void* g, const void* beta, float scale,
    const float* initial_state, const float* A_log, const float* dt_bias, float lower_bound,
    void* workspace, size_t workspace_bytes, void* out, float* final_state, kda_stream_t stream) {
  return forward_impl(PATH_SIMT, shape, plan_host, plan_dev, n_int32, q, k, v, g, beta, scale,
                      initial_state, A_log, dt_bias, lower_bound, workspace, workspace_bytes, out,
                      final_state, reinterpret_cast<cudaStream_t>(stream), nullptr);
}

extern "C" __attribute__((visibility("default"))) kda_status_t kda_simt_workspace_size(
    const int32_t* plan_host, size_t n_int32, size_t* bytes) {
  if (!bytes) return KDA_ERR_NULL;
  const kda_status_t st = validate_plan(plan_host, n_int32, nullptr);
  if (st != KDA_OK) return st;
  *bytes = simt_workspace_bytes(plan_host);
  return KDA_OK;
}

// The fused path with every chunk's intermediates (W, U, Q~, K^, Aqk, gamma_last; fp32, the
// two-kernel workspace layout after its 256-byte header) written to `dump` (if not NULL).  In a
// library built with -DKDA_PHASE_TIMING=1, CTA 0 also writes clock64() at each phase boundary of
// its first 64 chunks to `tprof` (32 words per chunk, if not NULL); the default build ignores it.
extern "C" __attribute__((visibility("default"))) kda_status_t kda_forward_debug(
    const kda_shape_t* shape, const int32_t* plan_host, const int32_t* plan_dev, size_t n_int32,
    const void* q, const void* k, const void* v, const void* g, const void* beta, float scale,
    const float* initial_state, const float* A_log, const float* dt_bias, float lower_bound,
    void* workspace, size_t workspace_bytes, void* out, float* final_state, float* dump,
    unsigned long long* tprof, kda_stream_t stream) {
  return forward_impl(PATH_FUSED, shape, plan_host, plan_dev, n_int32, q, k, v, g, beta, scale,
                      initial_state, A_log, dt_bias, lower_bound, workspace, workspace_bytes, out,
                      final_state, reinterpret_cast<cudaStream_t>(stream), dump, tprof);
}

extern "C" kda_status_t kda_device_status(const void* workspace, kda_stream_t stream) {
  if (!workspace) return KDA_ERR_NULL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t word = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
  if (cudaMemcpy(&word, workspace, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
  if (word == DS_OK) return KDA_OK;
  if (word == DS_PLAN) return KDA_ERR_PLAN;
  if (word == DS_TIMEOUT) return KDA_ERR_TIMEOUT;
  return KDA_ERR_CUDA;
}
