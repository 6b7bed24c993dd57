// Device side of the library's debug checks (ttt_set_debug_checks): guard words around the
// regions carved from a caller's workspace, and a scan of outputs for NaN / Inf. They stand
// in for a memory checker: a kernel that writes past the end (or before the start) of a
// workspace region changes a guard, and the check records DEVERR_BOUNDS in the device error
// word; a non-finite output records DEVERR_NONFINITE. Neither check faults or stops a
// kernel: they only set bits that ttt_last_device_status reports.
#include "ops.h"

namespace ttt {
namespace {

constexpr int kGuardWords = kGuardBytes / 4;

// Word i of every guard: a fixed pattern mixed with the word index, so a shifted or
// partially repeated copy of the pattern does not pass.
__device__ __forceinline__ unsigned guard_word(int i) {
  return 0x7E57C0DEu ^ (static_cast<unsigned>(i) * 0x9E3779B1u);
}

__global__ void guards_fill_kernel(GuardList g) {
  unsigned* p = g.p[blockIdx.x];
  for (int i = threadIdx.x; i < kGuardWords; i += blockDim.x) p[i] = guard_word(i);
}

__global__ void guards_check_kernel(GuardList g, unsigned* err) {
  const unsigned* p = g.p[blockIdx.x];
  bool bad = false;
  for (int i = threadIdx.x; i < kGuardWords; i += blockDim.x) bad |= p[i] != guard_word(i);
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(err, DEVERR_BOUNDS);
}

template <typename T>
__global__ void finite_scan_kernel(const T* x, long long n, unsigned* err) {
  bool bad = false;
  TTT_GRID_LOOP(i, n) {
    const float v = to_f32(x[i]);
    bad |= !isfinite(v);
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(err, DEVERR_NONFINITE);
}

}  // namespace

cudaError_t guards_fill(const GuardList& g, cudaStream_t s) {
  if (g.n <= 0) return cudaSuccess;
  guards_fill_kernel<<<g.n, kGuardWords, 0, s>>>(g);
  return cudaGetLastError();
}

cudaError_t guards_check(const GuardList& g, unsigned* err, cudaStream_t s) {
  if (g.n <= 0) return cudaSuccess;
  guards_check_kernel<<<g.n, kGuardWords, 0, s>>>(g, err);
  return cudaGetLastError();
}

cudaError_t finite_scan(int dt, const void* x, long long n, unsigned* err, cudaStream_t s) {
  if (n <= 0 || !x) return cudaSuccess;
  const unsigned grid = grid_for(n, 256, 148 * 8);
  if (dt == DT_BF16)
    finite_scan_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), n, err);
  else
    finite_scan_kernel<<<grid, 256, 0, s>>>(static_cast<const float*>(x), n, err);
  return cudaGetLastError();
}

}  // namespace ttt
