// kda_selftest.cu -- self-test of the sm_100a plumbing the fused kernel relies on: 128B-swizzled
// shared-memory operand tiles, tcgen05 shared-memory descriptors (K-major and MN-major), A taken
// from TMEM, the kind::f16 instruction descriptor, tcgen05.ld/st, and TMA 128B-swizzle loads.
//
// Internal entry point kda_selftest (not part of include/kda.h): one 128-thread CTA runs one
// M=128 MMA (or one TMA load) and writes the result to global memory for a host-side check.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "kda_sm100.cuh"
#include "kda_tmap.h"

namespace kda {
namespace {

using namespace sm100;

enum : int {
  ST_SS_KK = 0,    // A K-major, B K-major (shared memory)
  ST_SS_MNK = 1,   // A MN-major, B K-major
  ST_SS_KMN = 2,   // A K-major, B MN-major
  ST_TS_K = 3,     // A from TMEM, B K-major
  ST_TMA = 4,      // TMA load of a 64x128 box pair, raw shared-memory bytes out
  ST_TS_MN = 5,    // A from TMEM, B MN-major
  ST_TF32_SS = 6,  // kind::tf32, A K-major fp32, B K-major fp32 (shared memory)
  ST_TF32_TS = 7,  // kind::tf32, A fp32 from TMEM, B K-major fp32
  ST_TIMEOUT = 8,  // bounded wait on a barrier that nothing arrives on: must give up and report
  ST_M64 = 9,      // one M=64 MMA (A K-major [64][K], B K-major [N][K]); D = all 128 lanes x 2N
                   // columns of TMEM as they are, to map where an M=64 accumulator's rows land
};

constexpr uint32_t kWaitLimit = 1u << 24;

__global__ void __launch_bounds__(128, 1)
    selftest_kernel(int variant, const __nv_bfloat16* A, const __nv_bfloat16* B, float* D, int N,
                    int K, const __grid_constant__ CUtensorMap tmap, uint16_t* raw, int row0,
                    int* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint8_t* sA = sm;               // 32 KB
  uint8_t* sB = sm + 32768;       // 32 KB
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 65536);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + 65536 + 64);
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t bar_a = smem_u32(bar);

  if (tid == 0) {
    mbar_init(bar_a, 1);
    mbar_init(bar_a + 8, 1);  // ST_TIMEOUT's barrier: no thread, MMA or copy ever arrives on it
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  if (variant == ST_TIMEOUT) {
    // a short bounded wait that must run out; the kernel then leaves through its normal exit
    if (tid == 0 && !mbar_wait_bounded(bar_a + 8, 0, 1u << 14)) atomicExch(err, 3);
  } else if (variant == ST_TF32_SS || variant == ST_TF32_TS) {
    // fp32 operands (tf32 MMA): A [128][K] (fp32, passed as A), B [N][K] (fp32), both K-major
    const float* Af = reinterpret_cast<const float*>(A);
    const float* Bf = reinterpret_cast<const float*>(B);
    const bool a_tmem = (variant != ST_TF32_SS);
    if (!a_tmem) {
      for (int e = tid; e < 128 * K; e += 128) {
        const int m = e / K, k = e % K;
        *reinterpret_cast<float*>(sA + sw128_offset_f32(128, m, k)) = Af[e];
      }
    } else {
      const int m = tid;
      for (int c0 = 0; c0 < K; c0 += 16) {
        uint32_t r[16];
        for (int c = 0; c < 16; ++c) r[c] = __float_as_uint(Af[m * K + c0 + c]);
        tmem_st16(tbase + ((uint32_t)(warp * 32) << 16) + 256 + c0, r);
      }
      tmem_wait_st();
    }
    for (int e = tid; e < N * K; e += 128) {
      const int n = e / K, k = e % K;
      *reinterpret_cast<float*>(sB + sw128_offset_f32(N, n, k)) = Bf[e];
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_tf32(128, N, 0u, 0u);
      for (int kk = 0; kk < K / 8; ++kk) {
        const uint64_t bd =
            smem_desc(smem_u32(sB) + (kk / 4) * (N * 128) + (kk % 4) * 32, 16, 1024);
        if (a_tmem) {
          mma_ts_tf32(tbase, tbase + 256 + kk * 8, bd, idesc, kk > 0);
        } else {
          const uint64_t ad =
              smem_desc(smem_u32(sA) + (kk / 4) * (128 * 128) + (kk % 4) * 32, 16, 1024);
          mma_ss_tf32(tbase, ad, bd, idesc, kk > 0);
        }
      }
      mma_commit(bar_a);
    }
    if (!mbar_wait_bounded(bar_a, 0, kWaitLimit) && tid == 0) atomicExch(err, 2);
    tc_fence_after();
    for (int c0 = 0; c0 < N; c0 += 16) {
      uint32_t r[16];
      tmem_ld16(tbase + ((uint32_t)(warp * 32) << 16) + c0, r);
      tmem_wait_ld();
      for (int c = 0; c < 16; ++c) D[tid * N + c0 + c] = __uint_as_float(r[c]);
    }
  } else if (variant == ST_M64) {
    for (int e = tid; e < 64 * K; e += 128) {
      const int m = e / K, k = e % K;
      *reinterpret_cast<__nv_bfloat16*>(sA + sw128_offset(64, m, k)) = A[e];
    }
    for (int e = tid; e < N * K; e += 128) {
      const int n = e / K, k = e % K;
      *reinterpret_cast<__nv_bfloat16*>(sB + sw128_offset(N, n, k)) = B[e];
    }
    // zero the TMEM columns read back below, so untouched cells read as 0
    for (int c0 = 0; c0 < 2 * N; c0 += 16)
      tmem_st16_zero(tbase + ((uint32_t)(warp * 32) << 16) + c0);
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(64, N, 0u, 0u);
      for (int kk = 0; kk < K / 16; ++kk) {
        const uint64_t ad = smem_desc(smem_u32(sA) + (kk / 4) * (64 * 128) + (kk % 4) * 32, 16, 1024);
        const uint64_t bd = smem_desc(smem_u32(sB) + (kk / 4) * (N * 128) + (kk % 4) * 32, 16, 1024);
        mma_ss(tbase, ad, bd, idesc, kk > 0);
      }
      mma_commit(bar_a);
    }
    if (!mbar_wait_bounded(bar_a, 0, kWaitLimit) && tid == 0) atomicExch(err, 2);
    tc_fence_after();
    for (int c0 = 0; c0 < 2 * N; c0 += 16) {
      uint32_t r[16];
      tmem_ld16(tbase + ((uint32_t)(warp * 32) << 16) + c0, r);
      tmem_wait_ld();
      for (int c = 0; c < 16; ++c) D[tid * (2 * N) + c0 + c] = __uint_as_float(r[c]);
    }
  } else if (variant == ST_TMA) {
    if (tid == 0) {
      mbar_arrive_expect_tx(bar_a, 16384);
      tma_load_3d(smem_u32(sA), &tmap, bar_a, 0, row0, 0);
      tma_load_3d(smem_u32(sA + 8192), &tmap, bar_a, 64, row0, 0);
    }
    if (!mbar_wait_bounded(bar_a, 0, kWaitLimit) && tid == 0) atomicExch(err, 1);
    for (int i = tid; i < 8192; i += 128) raw[i] = reinterpret_cast<const uint16_t*>(sA)[i];
  } else {
    // operands into shared memory in the 128B-swizzled layouts
    const bool a_mn = (variant == ST_SS_MNK);
    const bool b_mn = (variant == ST_SS_KMN || variant == ST_TS_MN);
    const bool a_tmem = (variant == ST_TS_K || variant == ST_TS_MN);
    if (!a_tmem) {
      for (int e = tid; e < 128 * K; e += 128) {
        if (a_mn) {  // input A_t [K][128]
          const int k = e / 128, m = e % 128;
          *reinterpret_cast<__nv_bfloat16*>(sA + sw128_offset(K, k, m)) = A[e];
        } else {     // input A [128][K]
          const int m = e / K, k = e % K;
          *reinterpret_cast<__nv_bfloat16*>(sA + sw128_offset(128, m, k)) = A[e];
        }
      }
    } else {
      // thread m holds row m of A (warp w covers lanes 32w..32w+31) and stores it to TMEM
      const int m = tid;
      for (int c0 = 0; c0 < K / 2; c0 += 16) {
        uint32_t r[16];
        for (int c = 0; c < 16; ++c) {
          const int k = 2 * (c0 + c);
          r[c] = pack_bf16(__bfloat162float(A[m * K + k]), __bfloat162float(A[m * K + k + 1]));
        }
        tmem_st16(tbase + ((uint32_t)(warp * 32) << 16) + 256 + c0, r);
      }
      tmem_wait_st();
    }
    for (int e = tid; e < N * K; e += 128) {
      if (b_mn) {  // input B_t [K][N]
        const int k = e / N, n = e % N;
        *reinterpret_cast<__nv_bfloat16*>(sB + sw128_offset(K, k, n)) = B[e];
      } else {     // input B [N][K]
        const int n = e / K, k = e % K;
        *reinterpret_cast<__nv_bfloat16*>(sB + sw128_offset(N, n, k)) = B[e];
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(128, N, a_mn ? 1u : 0u, b_mn ? 1u : 0u);
      for (int kk = 0; kk < K / 16; ++kk) {
        uint64_t bd;
        if (b_mn) bd = smem_desc(smem_u32(sB) + kk * 2048, K * 128, 1024);
        else bd = smem_desc(smem_u32(sB) + (kk / 4) * (N * 128) + (kk % 4) * 32, 16, 1024);
        if (a_tmem) {
          mma_ts(tbase, tbase + 256 + kk * 8, bd, idesc, kk > 0);
        } else {
          uint64_t ad;
          if (a_mn) ad = smem_desc(smem_u32(sA) + kk * 2048, K * 128, 1024);
          else ad = smem_desc(smem_u32(sA) + (kk / 4) * (128 * 128) + (kk % 4) * 32, 16, 1024);
          mma_ss(tbase, ad, bd, idesc, kk > 0);
        }
      }
      mma_commit(bar_a);
    }
    if (!mbar_wait_bounded(bar_a, 0, kWaitLimit) && tid == 0) atomicExch(err, 2);
    tc_fence_after();
    for (int c0 = 0; c0 < N; c0 += 16) {
      uint32_t r[16];
      tmem_ld16(tbase + ((uint32_t)(warp * 32) << 16) + c0, r);
      tmem_wait_ld();
      for (int c = 0; c < 16; ++c) D[tid * N + c0 + c] = __uint_as_float(r[c]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

// y[i] = ex2(x[i]): the SFU exponential every decay of the fused kernel goes through.
__global__ void ex2_kernel(const float* x, float* y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = ex2(x[i]);
}

}  // namespace
}  // namespace kda

// Internal entry point (not part of include/kda.h): y = ex2.approx.ftz.f32(x) elementwise on the
// device, for a host-side accuracy check of the instruction.  Returns 0, 1 (bad argument) or 2.
extern "C" __attribute__((visibility("default"))) int kda_selftest_ex2(const float* x, float* y,
                                                                       int n, void* stream) {
  if (!x || !y || n < 1) return 1;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  kda::ex2_kernel<<<(n + 255) / 256, 256, 0, s>>>(x, y, n);
  if (cudaGetLastError() != cudaSuccess) return 2;
  return cudaStreamSynchronize(s) == cudaSuccess ? 0 : 2;
}

// Returns 0 on success, 1 on a bad argument, 2 on a CUDA error, 3 if a bounded wait gave up.
extern "C" __attribute__((visibility("default"))) int kda_selftest(
    int variant, const void* A, const void* B, float* D, int N, int K, void* raw,
    const void* tma_src, int tma_rows, int row0, int* err_dev, void* stream) {
  using namespace kda;
  if (variant < 0 || variant > ST_M64) return 1;
  if (variant == ST_M64 && (!A || !B || !D || N < 16 || N > 128 || N % 16 != 0 || (K != 64 && K != 128)))
    return 1;
  if (variant != ST_TMA && variant != ST_TIMEOUT && (!A || !B || !D || N < 16 || N > 128 || N % 16 != 0)) return 1;
  if (variant != ST_TMA && variant < ST_TF32_SS && K != 64 && K != 128) return 1;
  if ((variant == ST_TF32_SS || variant == ST_TF32_TS) && K != 32 && K != 64) return 1;
  if ((variant == ST_SS_KMN || variant == ST_TS_MN) && N != 64 && N != 128) return 1;
  CUtensorMap tmap;
  memset(&tmap, 0, sizeof(tmap));
  if (variant == ST_TMA) {
    if (!tma_src || !raw || tma_rows < 1 || row0 < 0) return 1;
    const uint64_t dims[3] = {128, (uint64_t)tma_rows, 1};
    const uint64_t strides[2] = {256, 256ull * tma_rows};
    const uint32_t box[3] = {64, 64, 1};
    if (!encode_bf16_3d(&tmap, tma_src, dims, strides, box)) return 2;
  }
  const size_t smem = 65536 + 1024 + 256;
  if (cudaFuncSetAttribute(selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return 2;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(err_dev, 0, 4, s) != cudaSuccess) return 2;
  selftest_kernel<<<1, 128, smem, s>>>(variant, static_cast<const __nv_bfloat16*>(A),
                                      static_cast<const __nv_bfloat16*>(B), D, N, K, tmap,
                                      static_cast<uint16_t*>(raw), row0, err_dev);
  if (cudaGetLastError() != cudaSuccess) return 2;
  if (cudaStreamSynchronize(s) != cudaSuccess) return 2;
  int err = 0;
  if (cudaMemcpy(&err, err_dev, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return 2;
  return err ? 3 : 0;
}
