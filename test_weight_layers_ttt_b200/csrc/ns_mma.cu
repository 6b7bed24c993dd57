// Newton-Schulz orthogonalisation of the recurrent LaCT update ("Test-Time Training Done
// Right", §2.2 Muon update) on the tensor cores, one CTA per (batch, head, matrix):
//
//   X = U / (||U||_F + eps), oriented with rows <= cols
//   repeat `steps` times:  A = X X^T,  X <- a X + (b A + c A A) X
//   U <- X in U's own orientation
//
// Every matrix that feeds a product is kept as a pair of bf16 matrices, hi = bf16(x) and
// lo = bf16(x - hi) (x = hi + lo to about 2^-16 relative), and each product is the three
// tcgen05.mma kind::f16 terms hi*hi + hi*lo + lo*hi accumulated in fp32 in TMEM: close to
// fp32 accuracy on the bf16 tensor cores. The epilogues between products (TMEM -> smem)
// rebuild fp32 values, form the next matrix and split it again.
//
// Sizes: rows <= 128, cols <= 256, zero padded to 128 x 256 (the padding stays zero).
// Shared memory (bf16, 128-byte swizzle, blocks of 64 columns x 128 rows = 16 KB):
//   Xh, Xl  4 blocks each (64 KB each): X as the K-major operand of A = X X^T and as the
//           MN-major B operand of P X
//   Gh, Gl  2 blocks each (32 KB each): A, then (once A A has been read) P = b A + c A A;
//           K-major A operand and MN-major B operand
// TMEM columns: [0,128) A, [128,256) A A, [256,512) P X.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ops.h"
#include "umma.cuh"

namespace ttt {
namespace {

using namespace umma;

constexpr int NS_THREADS = 128;
constexpr int NS_ROWS = 128, NS_COLS = 256;
constexpr int BLK = 128 * 128;   // one 64-column block of 128 rows, bytes
constexpr int XH_OFF = 0, XL_OFF = 4 * BLK, GH_OFF = 8 * BLK, GL_OFF = 10 * BLK;
constexpr int BAR_OFF = 12 * BLK;
constexpr int NS_SMEM = BAR_OFF + 64 + 1024;   // + barrier/flags + alignment slack

// Byte offset of the 16-byte chunk holding columns 8q .. 8q+7 of row i.
__device__ __forceinline__ uint32_t chunk_off(int i, int q) {
  return (uint32_t)((q >> 3) * BLK + i * 128 + (((q & 7) ^ (i & 7)) << 4));
}

// K-major operand over K = k0 .. k0+15 (rows = M or N index, 8-row groups 1024 B apart);
// MN-major operand with MN = column, K = row k0 .. k0+15 (64-wide MN blocks BLK apart).
__device__ __forceinline__ uint64_t kmajor(uint32_t base, int k0) {
  return make_sw128_desc(base + (uint32_t)((k0 >> 6) * BLK + (k0 & 63) * 2), 16, 1024);
}
__device__ __forceinline__ uint64_t mnmajor(uint32_t base, int k0) {
  return make_sw128_desc(base + (uint32_t)(k0 * 128), BLK, 1024);
}

// x -> (hi, lo) packed as bf16x2 pairs for two values.
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Split 8 values into the hi / lo chunks at byte offset `off` of the two matrices.
__device__ __forceinline__ void store_split8(uint32_t hbase, uint32_t lbase, uint32_t off,
                                             const float (&v)[8]) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) split2(v[2 * t], v[2 * t + 1], h[t], l[t]);
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(hbase + off), "r"(h[0]),
               "r"(h[1]), "r"(h[2]), "r"(h[3])
               : "memory");
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(lbase + off), "r"(l[0]),
               "r"(l[1]), "r"(l[2]), "r"(l[3])
               : "memory");
}

// hi + lo of 8 values at byte offset `off`.
__device__ __forceinline__ void load_join8(uint32_t hbase, uint32_t lbase, uint32_t off,
                                           float (&v)[8]) {
  uint32_t h[4], l[4];
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
               : "r"(hbase + off)
               : "memory");
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(l[0]), "=r"(l[1]), "=r"(l[2]), "=r"(l[3])
               : "r"(lbase + off)
               : "memory");
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h[t]));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&l[t]));
    v[2 * t] = a.x + b.x;
    v[2 * t + 1] = a.y + b.y;
  }
}

__global__ void __launch_bounds__(NS_THREADS, 1)
    ns_mma_kernel(float* U, NsLayout Lay, int steps, float eps, float ca, float cb, float cc,
                  unsigned* err, unsigned long long wait_ns) {
  extern __shared__ uint8_t ns_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(ns_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  float* red = reinterpret_cast<float*>(tslot + 2);   // [4] warp partial sums

  const int p = blockIdx.x, z = blockIdx.y;
  if (!(Lay.mask & (1 << p))) return;
  const int R = Lay.R[p], Cc = Lay.C[p];               // U's own [R, Cc]
  const bool tr = R > Cc;
  const int r = tr ? Cc : R, cols = tr ? R : Cc;       // iterate on [r, cols], r <= cols
  const long long hm = (long long)R * Cc;
  float* u = U + z * Lay.zstride + p * Lay.pstride;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sb = smem_u32(smem);
  const uint32_t sXh = sb + XH_OFF, sXl = sb + XL_OFF, sGh = sb + GH_OFF, sGl = sb + GL_OFF;

  if (tid == 0) {
    mbar_init(smem_u32(bar), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }

  // ||U||_F
  float ss = 0.0f;
  for (long long e = tid; e < hm; e += NS_THREADS) ss = fmaf(u[e], u[e], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red[warp] = ss;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const float scale = 1.0f / (sqrtf(red[0] + red[1] + red[2] + red[3]) + eps);
  const uint32_t tmem = *tslot;

  // X = U * scale in the [r, cols] orientation, zero padded to 128 x 256
  for (int e = tid; e < NS_ROWS * (NS_COLS / 8); e += NS_THREADS) {
    const int i = e >> 5, q = e & 31;
    float v[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int j = 8 * q + t;
      float x = 0.0f;
      if (i < r && j < cols) x = tr ? u[(long long)j * Cc + i] : u[(long long)i * Cc + j];
      v[t] = x * scale;
    }
    store_split8(sXh, sXl, chunk_off(i, q), v);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
  const int row = tid;   // TMEM lane = matrix row
  uint32_t phase = 0;
  int commits = 0;
  bool ok = true;
  // One product (three hi/lo terms) issued by thread 0, waited for by all threads (bounded,
  // with a block-wide vote so every thread takes the same path).
  auto product = [&](int which) -> bool {
    if (tid == 0) {
      tc_fence_after();
      if (which == 0) {          // A = X X^T: M 128, N 128, K 256
        constexpr uint32_t ID = make_idesc_bf16(128, 128, false, false);
        for (int k0 = 0; k0 < NS_COLS; k0 += 16) {
          mma_f16(tmem, kmajor(sXh, k0), kmajor(sXh, k0), ID, k0 > 0);
          mma_f16(tmem, kmajor(sXh, k0), kmajor(sXl, k0), ID, 1);
          mma_f16(tmem, kmajor(sXl, k0), kmajor(sXh, k0), ID, 1);
        }
      } else if (which == 1) {   // A A: M 128, N 128, K 128 (B = A read MN-major)
        constexpr uint32_t ID = make_idesc_bf16(128, 128, false, true);
        for (int k0 = 0; k0 < NS_ROWS; k0 += 16) {
          mma_f16(tmem + 128, kmajor(sGh, k0), mnmajor(sGh, k0), ID, k0 > 0);
          mma_f16(tmem + 128, kmajor(sGh, k0), mnmajor(sGl, k0), ID, 1);
          mma_f16(tmem + 128, kmajor(sGl, k0), mnmajor(sGh, k0), ID, 1);
        }
      } else {                   // P X: M 128, N 256, K 128 (B = X read MN-major)
        constexpr uint32_t ID = make_idesc_bf16(128, 256, false, true);
        for (int k0 = 0; k0 < NS_ROWS; k0 += 16) {
          mma_f16(tmem + 256, kmajor(sGh, k0), mnmajor(sXh, k0), ID, k0 > 0);
          mma_f16(tmem + 256, kmajor(sGh, k0), mnmajor(sXl, k0), ID, 1);
          mma_f16(tmem + 256, kmajor(sGl, k0), mnmajor(sXh, k0), ID, 1);
        }
      }
      mma_commit(smem_u32(bar));
    }
    ++commits;
    const bool got = mbar_wait(smem_u32(bar), phase, abort_flag, err, wait_ns);
    phase ^= 1u;
    const bool all = __syncthreads_and(got) != 0;
    tc_fence_after();
    return all;
  };
  auto publish = [&]() {   // smem writes -> visible to the next product's MMAs
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
  };

  for (int it = 0; it < steps && ok; ++it) {
    // ---- A = X X^T -> (Gh, Gl)
    if (!(ok = product(0))) break;
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t g[32];
      tmem_ld32(lane_base + (uint32_t)c0, g);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = __uint_as_float(g[8 * q + t]);
        store_split8(sGh, sGl, chunk_off(row, (c0 >> 3) + q), v);
      }
    }
    publish();
    // ---- A A, then P = b A + c A A -> (Gh, Gl)
    if (!(ok = product(1))) break;
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t g[32], g2[32];
      tmem_ld32(lane_base + (uint32_t)c0, g);
      tmem_ld32(lane_base + 128u + (uint32_t)c0, g2);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v[8];
#pragma unroll
        for (int t = 0; t < 8; ++t)
          v[t] = fmaf(cc, __uint_as_float(g2[8 * q + t]), cb * __uint_as_float(g[8 * q + t]));
        store_split8(sGh, sGl, chunk_off(row, (c0 >> 3) + q), v);
      }
    }
    publish();
    // ---- Y = P X, then X <- a X + Y, each thread its own row
    if (!(ok = product(2))) break;
#pragma unroll 1
    for (int c0 = 0; c0 < NS_COLS; c0 += 32) {
      uint32_t y[32];
      tmem_ld32(lane_base + 256u + (uint32_t)c0, y);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t off = chunk_off(row, (c0 >> 3) + q);
        float x[8];
        load_join8(sXh, sXl, off, x);
#pragma unroll
        for (int t = 0; t < 8; ++t) x[t] = fmaf(ca, x[t], __uint_as_float(y[8 * q + t]));
        store_split8(sXh, sXl, off, x);
      }
    }
    publish();
  }

  if (ok) {
    // U <- X in U's orientation
    for (int e = tid; e < NS_ROWS * (NS_COLS / 8); e += NS_THREADS) {
      const int i = e >> 5, q = e & 31;
      if (i >= r || 8 * q >= cols) continue;
      float x[8];
      load_join8(sXh, sXl, chunk_off(i, q), x);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int j = 8 * q + t;
        if (j < cols) {
          if (tr) u[(long long)j * Cc + i] = x[t];
          else u[(long long)i * Cc + j] = x[t];
        }
      }
    }
  } else if (tid == 0 && commits > 0) {
    // a wait gave up: let the last committed product finish before TMEM is freed
    mbar_wait(smem_u32(bar), phase ^ 1u, abort_flag, nullptr, wait_ns, true);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool ns_mma_supported(int R, int C) {
  const int r = R < C ? R : C, c = R < C ? C : R;
  return r <= NS_ROWS && c <= NS_COLS;
}

cudaError_t ns_mma(float* U, int Z, const NsLayout& L, int steps, float eps, float a, float b,
                   float c, unsigned* err, unsigned long long wait_ns, cudaStream_t s) {
  if (Z <= 0) return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(ns_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, NS_SMEM);
  if (e != cudaSuccess) return e;
  ns_mma_kernel<<<dim3(L.parts, Z), NS_THREADS, NS_SMEM, s>>>(U, L, steps, eps, a, b, c, err,
                                                              wait_ns);
  return cudaGetLastError();
}

}  // namespace ttt
