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
// Shared memory (bf16, 128-byte swizzle, blocks of 64 columns x 128 rows = 16 KB), the hi
// and lo block of each 64-column range next to each other (hi at 2kb, lo at 2kb + 1):
//   X  8 blocks (128 KB): K-major operand of A = X X^T, MN-major B operand of P X
//   G  4 blocks (64 KB): A, then (once A A has been read) P = b A + c A A; K-major operand
// Because a hi block is followed by its lo block, one N=256 K-major B operand starting at a
// hi block reads [hi; lo] stacked: a single instruction gives hi*hi^T and hi*lo^T side by
// side, and a second N=128 one gives lo*hi^T.
// A is symmetric, so A A is formed as A A^T: both of its operands are read K-major.
// TMEM columns: [0,256) hi*hi^T | hi*lo^T, [256,384) lo*hi^T (products 0 and 1), then
// [0,256) P X.
// 256 threads: warp w drains TMEM lanes 32 (w % 4) .. +31 (matrix rows), columns of half
// w / 4 of each product; thread 0 issues the MMAs.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ops.h"
#include "umma.cuh"

namespace ttt {
namespace {

using namespace umma;

constexpr int NS_THREADS = 256;
constexpr int NS_ROWS = 128, NS_COLS = 256;
constexpr int BLK = 128 * 128;     // one 64-column block of 128 rows, bytes
constexpr int KB = 2 * BLK;        // hi + lo block pair of one 64-column range
constexpr int X_OFF = 0, G_OFF = 4 * KB;
constexpr int BAR_OFF = 6 * KB;
constexpr int NS_SMEM = BAR_OFF + 64 + 1024;   // + barrier/flags + alignment slack
constexpr int LD_BATCH = 8;        // 8-column chunks per thread per batch of global loads

// Byte offset of the 16-byte chunk holding columns 8q .. 8q+7 of row i in the hi block (the
// lo block's chunk is BLK further).
__device__ __forceinline__ uint32_t chunk_off(int i, int q) {
  return (uint32_t)((q >> 3) * KB + i * 128 + (((q & 7) ^ (i & 7)) << 4));
}

// K-major operand over K = k0 .. k0+15 (rows = M or N index, 8-row groups 1024 B apart);
// MN-major operand with MN = column, K = row k0 .. k0+15 (64-wide MN blocks KB apart).
__device__ __forceinline__ uint64_t kmajor(uint32_t base, int k0) {
  return make_sw128_desc(base + (uint32_t)((k0 >> 6) * KB + (k0 & 63) * 2), 16, 1024);
}
__device__ __forceinline__ uint64_t mnmajor(uint32_t base, int k0) {
  return make_sw128_desc(base + (uint32_t)(k0 * 128), KB, 1024);
}

// Values of a finished tcgen05.ld: the empty asm ties every use to the wait before it.
__device__ __forceinline__ void pin32(uint32_t (&a)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(a[i]));
}

// x -> (hi, lo) packed as bf16x2 pairs for two values.
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Split 8 values into the hi / lo chunks at byte offset `off` (hi) and off + BLK (lo).
__device__ __forceinline__ void store_split8(uint32_t base, uint32_t off, const float (&v)[8]) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) split2(v[2 * t], v[2 * t + 1], h[t], l[t]);
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + off), "r"(h[0]),
               "r"(h[1]), "r"(h[2]), "r"(h[3])
               : "memory");
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + off + BLK), "r"(l[0]),
               "r"(l[1]), "r"(l[2]), "r"(l[3])
               : "memory");
}

// hi + lo of the 8 values at byte offset `off`.
__device__ __forceinline__ void load_join8(uint32_t base, uint32_t off, float (&v)[8]) {
  uint32_t h[4], l[4];
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
               : "r"(base + off)
               : "memory");
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(l[0]), "=r"(l[1]), "=r"(l[2]), "=r"(l[3])
               : "r"(base + off + BLK)
               : "memory");
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h[t]));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&l[t]));
    v[2 * t] = a.x + b.x;
    v[2 * t + 1] = a.y + b.y;
  }
}

// The 8-column chunk (i, q) of X that chunk number e of this CTA's walk covers: along a
// row of U in memory (q fastest) when X is U itself, along a column of U (i fastest) when
// X is U^T, so that a warp's global accesses are contiguous either way.
__device__ __forceinline__ void chunk_of(int e, bool tr, int& i, int& q) {
  if (tr) { i = e & (NS_ROWS - 1); q = e >> 7; }
  else { i = e >> 5; q = e & 31; }
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
  float* red = reinterpret_cast<float*>(tslot + 2);   // [8] warp partial sums

  const int p = blockIdx.x, z = blockIdx.y;
  if (!(Lay.mask & (1 << p))) return;
  const int R = Lay.R[p], Cc = Lay.C[p];               // U's own [R, Cc]
  const bool tr = R > Cc;
  const int r = tr ? Cc : R, cols = tr ? R : Cc;       // iterate on [r, cols], r <= cols
  const long long hm = (long long)R * Cc;
  float* u = U + z * Lay.zstride + p * Lay.pstride;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sb = smem_u32(smem);
  const uint32_t sX = sb + X_OFF, sG = sb + G_OFF;
  // 16-byte vector access to U: aligned base and whole float4s per row
  const bool vec = ((reinterpret_cast<uintptr_t>(u) & 15) == 0) && ((Cc & 3) == 0);

  if (tid == 0) {
    mbar_init(smem_u32(bar), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }

  // ||U||_F, LD_BATCH independent loads in flight per thread
  float ss = 0.0f;
  if (vec) {
    const float4* u4 = reinterpret_cast<const float4*>(u);
    const long long n4 = hm >> 2;
    for (long long e0 = tid; e0 < n4; e0 += (long long)NS_THREADS * LD_BATCH) {
      float4 t[LD_BATCH];
#pragma unroll
      for (int k = 0; k < LD_BATCH; ++k) {
        const long long e = e0 + (long long)k * NS_THREADS;
        t[k] = e < n4 ? u4[e] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int k = 0; k < LD_BATCH; ++k)
        ss = fmaf(t[k].x, t[k].x, fmaf(t[k].y, t[k].y, fmaf(t[k].z, t[k].z,
                                                           fmaf(t[k].w, t[k].w, ss))));
    }
  } else {
    for (long long e0 = tid; e0 < hm; e0 += (long long)NS_THREADS * LD_BATCH) {
      float t[LD_BATCH];
#pragma unroll
      for (int k = 0; k < LD_BATCH; ++k) {
        const long long e = e0 + (long long)k * NS_THREADS;
        t[k] = e < hm ? u[e] : 0.0f;
      }
#pragma unroll
      for (int k = 0; k < LD_BATCH; ++k) ss = fmaf(t[k], t[k], ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red[warp] = ss;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  float tot = 0.0f;
#pragma unroll
  for (int w = 0; w < NS_THREADS / 32; ++w) tot += red[w];
  const float scale = 1.0f / (sqrtf(tot) + eps);
  const uint32_t tmem = *tslot;

  // X = U * scale in the [r, cols] orientation, zero padded to 128 x 256
  constexpr int NCHUNK = NS_ROWS * (NS_COLS / 8);
  for (int e0 = tid; e0 < NCHUNK; e0 += NS_THREADS * LD_BATCH) {
    float v[LD_BATCH][8];
#pragma unroll
    for (int k = 0; k < LD_BATCH; ++k) {
      int i, q;
      chunk_of(e0 + k * NS_THREADS, tr, i, q);
      const int j0 = 8 * q;
      if (!tr && vec && i < r && j0 + 8 <= cols) {
        const float4* s4 = reinterpret_cast<const float4*>(u + (long long)i * Cc + j0);
        const float4 a0 = s4[0], a1 = s4[1];
        v[k][0] = a0.x; v[k][1] = a0.y; v[k][2] = a0.z; v[k][3] = a0.w;
        v[k][4] = a1.x; v[k][5] = a1.y; v[k][6] = a1.z; v[k][7] = a1.w;
      } else {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int j = j0 + t;
          v[k][t] = (i < r && j < cols)
                        ? (tr ? u[(long long)j * Cc + i] : u[(long long)i * Cc + j])
                        : 0.0f;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < LD_BATCH; ++k) {
      int i, q;
      chunk_of(e0 + k * NS_THREADS, tr, i, q);
#pragma unroll
      for (int t = 0; t < 8; ++t) v[k][t] *= scale;
      store_split8(sX, chunk_off(i, q), v[k]);
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int quarter = warp & 3, half = warp >> 2;
  const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
  const int row = quarter * 32 + lane;   // TMEM lane = matrix row
  uint32_t phase = 0;
  int commits = 0;
  bool ok = true;
  // One product issued by thread 0, waited for by all threads (bounded, with a block-wide
  // vote so every thread takes the same path).
  //   0: X X^T   from X (K 256)  -> [hh | hl] at column 0, lh at column 256
  //   1: A A^T   from G (K 128)  -> the same columns
  //   2: P X     A = G, B = X MN-major (K 128, N 256) -> column 0, three terms
  auto product = [&](int which) -> bool {
    if (tid == 0) {
      tc_fence_after();
      if (which < 2) {
        const uint32_t base = which == 0 ? sX : sG;
        const int K = which == 0 ? NS_COLS : NS_ROWS;
        constexpr uint32_t ID256 = make_idesc_bf16(128, 256, false, false);
        constexpr uint32_t ID128 = make_idesc_bf16(128, 128, false, false);
        for (int k0 = 0; k0 < K; k0 += 16) {
          mma_f16(tmem, kmajor(base, k0), kmajor(base, k0), ID256, k0 > 0);
          mma_f16(tmem + 256, kmajor(base + BLK, k0), kmajor(base, k0), ID128, k0 > 0);
        }
      } else {
        constexpr uint32_t ID = make_idesc_bf16(128, 256, false, true);
        for (int k0 = 0; k0 < NS_ROWS; k0 += 16) {
          mma_f16(tmem, kmajor(sG, k0), mnmajor(sX, k0), ID, k0 > 0);
          mma_f16(tmem, kmajor(sG, k0), mnmajor(sX + BLK, k0), ID, 1);
          mma_f16(tmem, kmajor(sG + BLK, k0), mnmajor(sX, k0), ID, 1);
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
  // Columns c0 .. c0+31 of the three-term result of product 0 or 1 for this thread's row:
  // hh + (hl + lh), the bracket keeping a symmetric product bitwise symmetric.
  auto sum3 = [&](int c0, float (&o)[32]) {
    uint32_t hh[32], hl[32], lh[32];
    tmem_ld32(lane_base + (uint32_t)c0, hh);
    tmem_ld32(lane_base + 128u + (uint32_t)c0, hl);
    tmem_ld32(lane_base + 256u + (uint32_t)c0, lh);
    tmem_ld_wait();
    pin32(hh);
    pin32(hl);
    pin32(lh);
#pragma unroll
    for (int t = 0; t < 32; ++t)
      o[t] = __uint_as_float(hh[t]) + (__uint_as_float(hl[t]) + __uint_as_float(lh[t]));
  };

  for (int it = 0; it < steps && ok; ++it) {
    // ---- A = X X^T -> G
    if (!(ok = product(0))) break;
#pragma unroll 1
    for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
      float g[32];
      sum3(c0, g);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = g[8 * q + t];
        store_split8(sG, chunk_off(row, (c0 >> 3) + q), v);
      }
    }
    publish();
    // ---- A A^T, then P = b A + c A A^T -> G (A re-read from G)
    if (!(ok = product(1))) break;
#pragma unroll 1
    for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
      float g2[32];
      sum3(c0, g2);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t off = chunk_off(row, (c0 >> 3) + q);
        float v[8];
        load_join8(sG, off, v);
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = fmaf(cc, g2[8 * q + t], cb * v[t]);
        store_split8(sG, off, v);
      }
    }
    publish();
    // ---- Y = P X, then X <- a X + Y, each thread its own row
    if (!(ok = product(2))) break;
#pragma unroll 1
    for (int c0 = half * 128; c0 < half * 128 + 128; c0 += 32) {
      uint32_t y[32];
      tmem_ld32(lane_base + (uint32_t)c0, y);
      tmem_ld_wait();
      pin32(y);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t off = chunk_off(row, (c0 >> 3) + q);
        float x[8];
        load_join8(sX, off, x);
#pragma unroll
        for (int t = 0; t < 8; ++t) x[t] = fmaf(ca, x[t], __uint_as_float(y[8 * q + t]));
        store_split8(sX, off, x);
      }
    }
    publish();
  }

  if (ok) {
    // U <- X in U's orientation
    for (int e = tid; e < NCHUNK; e += NS_THREADS) {
      int i, q;
      chunk_of(e, tr, i, q);
      const int j0 = 8 * q;
      if (i >= r || j0 >= cols) continue;
      float x[8];
      load_join8(sX, chunk_off(i, q), x);
      if (!tr && vec && j0 + 8 <= cols) {
        float4* d4 = reinterpret_cast<float4*>(u + (long long)i * Cc + j0);
        d4[0] = make_float4(x[0], x[1], x[2], x[3]);
        d4[1] = make_float4(x[4], x[5], x[6], x[7]);
      } else {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int j = j0 + t;
          if (j < cols) {
            if (tr) u[(long long)j * Cc + i] = x[t];
            else u[(long long)i * Cc + j] = x[t];
          }
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
