// kda_decode.cu -- the single-token decode step: one step of the KDA recurrence per (sequence,
// value head), the step that follows a prefill.
//
// The recurrence is the one the chunked prefill computes in 64-token blocks (FlashKDA README,
// 功能说明; FLA PR 656 keeps a naive token-by-token "recurrent" kernel beside its chunked ones):
//     S <- S Diag(e^g);   S <- S + beta (v - S k^) k^T;   o = scale S q^
// with the same in-op activations as kda_forward: q^, k^ L2-normalised (eps 1e-6), beta =
// sigmoid(logit), g = lb * sigmoid(e^A_log (g_raw + dt_bias)).
//
// Row i of S (value channel i) depends only on row i, so the state is streamed once: every warp
// owns D/8 rows, a lane D/32 columns (16 and 4 at D = 128; the head dims are 128 and 64); a row
// is read, decayed, corrected, read out against q^ and written back (in place when state_out ==
// state_in).  Per (sequence, head) at D = 128 the step moves 2 x 64 KB of fp32 state and about
// 1.3 KB of bf16 inputs and output: HBM-bound.  All math is fp32; no tensor cores (each step is
// a rank-1 update of a D x D matrix).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kDecThreads = 256;  // 8 warps; each owns D / 8 state rows, a lane D / 32 columns

struct DecodeParams {
  int Nqk, Nv, group;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* g;
  const __nv_bfloat16* beta;
  float scale;
  const float* S0;  // may be null (zero state)
  const float* A_log;
  const float* dt_bias;
  float lower_bound;
  __nv_bfloat16* out;
  float* S1;
};

// N consecutive bf16 (N = 2 or 4, 4N-byte aligned) -> fp32
template <int N>
__device__ __forceinline__ void load_bf16(const __nv_bfloat16* p, float (&x)[N]) {
  if constexpr (N == 4) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(p));
    x[0] = __uint_as_float(w.x << 16);
    x[1] = __uint_as_float(w.x & 0xFFFF0000u);
    x[2] = __uint_as_float(w.y << 16);
    x[3] = __uint_as_float(w.y & 0xFFFF0000u);
  } else {
    const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(p));
    x[0] = __uint_as_float(w << 16);
    x[1] = __uint_as_float(w & 0xFFFF0000u);
  }
}

// N consecutive fp32 (N = 2 or 4) with plain loads / stores (the state may be updated in place)
template <int N>
__device__ __forceinline__ void ld_f32(const float* p, float (&x)[N]) {
  if constexpr (N == 4) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  } else {
    const float2 v = *reinterpret_cast<const float2*>(p);
    x[0] = v.x; x[1] = v.y;
  }
}
template <int N>
__device__ __forceinline__ void st_f32(float* p, const float (&x)[N]) {
  if constexpr (N == 4) *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  else *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int D>
__global__ void __launch_bounds__(kDecThreads) kda_decode_kernel(const DecodeParams p) {
  constexpr int RPW = D / 8;   // state rows per warp
  constexpr int CPL = D / 32;  // columns per lane
  const int unit = blockIdx.x;  // b * Nv + h
  const int b = unit / p.Nv, h = unit - b * p.Nv;
  const int hq = h / p.group;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = CPL * lane;
  const size_t srow0 = ((size_t)unit * D + warp * RPW) * D + j0;

  // this warp's state rows are requested first, so the HBM reads overlap the activations
  float s[RPW][CPL];
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    if (p.S0) {
      ld_f32<CPL>(p.S0 + srow0 + (size_t)r * D, s[r]);  // plain loads: S0 may be S1 (in place)
    } else {
#pragma unroll
      for (int e = 0; e < CPL; ++e) s[r][e] = 0.f;
    }
  }

  // activations of this lane's columns (every warp computes them for itself)
  float qv[CPL], kv[CPL], gv[CPL];
  load_bf16<CPL>(p.q + ((size_t)b * p.Nqk + hq) * D + j0, qv);
  load_bf16<CPL>(p.k + ((size_t)b * p.Nqk + hq) * D + j0, kv);
  load_bf16<CPL>(p.g + (size_t)unit * D + j0, gv);
  float ssq = 0.f, ssk = 0.f;
#pragma unroll
  for (int e = 0; e < CPL; ++e) {
    ssq = fmaf(qv[e], qv[e], ssq);
    ssk = fmaf(kv[e], kv[e], ssk);
  }
  ssq = warp_sum(ssq);
  ssk = warp_sum(ssk);
  const float rq = p.scale / sqrtf(ssq + 1e-6f), rk = 1.0f / sqrtf(ssk + 1e-6f);
  const float a_h = expf(__ldg(p.A_log + h));
  float qh[CPL], kh[CPL], gam[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) {
    qh[e] = qv[e] * rq;
    kh[e] = kv[e] * rk;
    const float z = a_h * (gv[e] + __ldg(p.dt_bias + h * D + j0 + e));
    const float gact = p.lower_bound / (1.0f + expf(-z));
    gam[e] = expf(gact);
  }
  const float beta = 1.0f / (1.0f + expf(-__bfloat162float(p.beta[unit])));
  // v of this warp's rows: lane r < RPW holds row r's value
  const float vrow = lane < RPW ? __bfloat162float(p.v[(size_t)unit * D + warp * RPW + lane]) : 0.f;

  float o_mine = 0.f;  // lane r < RPW ends with o of row r
#pragma unroll
  for (int r0 = 0; r0 < RPW; r0 += 4) {
    float pred[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < CPL; ++e) {
        s[r0 + i][e] *= gam[e];
        acc = fmaf(s[r0 + i][e], kh[e], acc);
      }
      pred[i] = acc;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i) pred[i] += __shfl_xor_sync(0xffffffffu, pred[i], o);
    float op[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float u = beta * (__shfl_sync(0xffffffffu, vrow, r0 + i) - pred[i]);
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < CPL; ++e) {
        s[r0 + i][e] = fmaf(u, kh[e], s[r0 + i][e]);
        acc = fmaf(s[r0 + i][e], qh[e], acc);
      }
      op[i] = acc;
      st_f32<CPL>(p.S1 + srow0 + (size_t)(r0 + i) * D, s[r0 + i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i) op[i] += __shfl_xor_sync(0xffffffffu, op[i], o);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (lane == r0 + i) o_mine = op[i];
  }
  if (lane < RPW) p.out[(size_t)unit * D + warp * RPW + lane] = __float2bfloat16_rn(o_mine);
}

struct Range {
  uintptr_t lo, hi;
};
bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }
Range range_of(const void* p, size_t bytes) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return {lo, p ? lo + bytes : lo};
}

}  // namespace
}  // namespace kda

using namespace kda;

extern "C" kda_status_t kda_decode(int32_t B, int32_t Nqk, int32_t Nv, int32_t D, const void* q,
                                   const void* k, const void* v, const void* g, const void* beta,
                                   float scale, const float* state_in, const float* A_log,
                                   const float* dt_bias, float lower_bound, void* out,
                                   float* state_out, kda_stream_t stream) {
  if (D != kD && D != 64) return KDA_ERR_DIM;
  if (B < 1 || Nqk < 1 || Nv < 1) return KDA_ERR_SHAPE;
  if (Nv % Nqk != 0) return KDA_ERR_HEADS;
  if ((int64_t)B * Nv > INT32_MAX / 2) return KDA_ERR_SHAPE;
  if (!q || !k || !v || !g || !beta || !A_log || !dt_bias || !out || !state_out)
    return KDA_ERR_NULL;
  if (!std::isfinite(scale)) return KDA_ERR_LOWER_BOUND;
  if (!(lower_bound >= -5.0f && lower_bound <= 0.0f)) return KDA_ERR_LOWER_BOUND;
  {
    const void* a16[] = {q, k, v, g, out, state_out, state_in, A_log, dt_bias};
    for (const void* ptr : a16)
      if (reinterpret_cast<uintptr_t>(ptr) & 15u) return KDA_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(beta) & 1u) return KDA_ERR_ALIGN;
  }
  const size_t units = (size_t)B * Nv;
  const size_t st_bytes = units * D * D * 4;
  const Range r_out = range_of(out, units * D * 2), r_s1 = range_of(state_out, st_bytes);
  const Range r_s0 = range_of(state_in, st_bytes);
  // state_out may be state_in itself (update in place) but must not overlap it otherwise
  if (state_in && state_in != state_out && overlaps(r_s0, r_s1)) return KDA_ERR_ALIAS;
  const Range ins[] = {range_of(q, (size_t)B * Nqk * D * 2), range_of(k, (size_t)B * Nqk * D * 2),
                       range_of(v, units * D * 2), range_of(g, units * D * 2),
                       range_of(beta, units * 2), range_of(A_log, (size_t)Nv * 4),
                       range_of(dt_bias, (size_t)Nv * D * 4)};
  for (const Range& r : ins)
    if (overlaps(r, r_out) || overlaps(r, r_s1)) return KDA_ERR_ALIAS;
  if (overlaps(r_out, r_s1) || (state_in && overlaps(r_out, r_s0))) return KDA_ERR_ALIAS;

  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return KDA_ERR_CUDA;
  if (major != 10) return KDA_ERR_DEVICE;

  DecodeParams p{};
  p.Nqk = Nqk;
  p.Nv = Nv;
  p.group = Nv / Nqk;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.g = static_cast<const __nv_bfloat16*>(g);
  p.beta = static_cast<const __nv_bfloat16*>(beta);
  p.scale = scale;
  p.S0 = state_in;
  p.A_log = A_log;
  p.dt_bias = dt_bias;
  p.lower_bound = lower_bound;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.S1 = state_out;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (D == kD) kda_decode_kernel<kD><<<(unsigned)units, kDecThreads, 0, st>>>(p);
  else kda_decode_kernel<64><<<(unsigned)units, kDecThreads, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
