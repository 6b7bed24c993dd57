// Shared helpers of the sm_100a TTT library: element types, the per-device error word,
// bounded waits and small launch utilities. Included by every .cu of the library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/ttt.h"

namespace ttt {

// Element type tags used by the host orchestration and the kernels.
enum DType : int { DT_F32 = 0, DT_BF16 = 1 };

inline size_t dtype_size(int dt) { return dt == DT_BF16 ? 2 : 4; }

// Bits of the device error word (one per device, file-scope __device__ variable in
// ttt_api.cu; kernels receive its address as an argument): a bounded wait ran out, a
// workspace guard word changed (debug checks), an output held NaN / Inf (debug checks).
enum : unsigned { DEVERR_TIMEOUT = 1u, DEVERR_BOUNDS = 2u, DEVERR_NONFINITE = 4u };

// Default limit of every bounded device-side wait, in nanoseconds.
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// silu(a) = a * sigmoid(a) and its derivative, in fp32 with CUDA's expf.
__device__ __forceinline__ float sigmoidf_(float a) { return 1.0f / (1.0f + expf(-a)); }
__device__ __forceinline__ float siluf_(float a) { return a * sigmoidf_(a); }
__device__ __forceinline__ float silu_primef_(float a) {
  const float s = sigmoidf_(a);
  return s * (1.0f + a * (1.0f - s));
}

// Grid-stride loop helper.
#define TTT_GRID_LOOP(i, n) \
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < (long long)(n); \
       i += (long long)gridDim.x * blockDim.x)

inline unsigned grid_for(long long n, int threads, int max_blocks = 148 * 16) {
  long long b = (n + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > max_blocks) b = max_blocks;
  return (unsigned)b;
}

}  // namespace ttt
