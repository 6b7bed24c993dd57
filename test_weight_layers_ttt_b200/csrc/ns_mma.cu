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
//   X  8 blocks (128 KB): K-major operand of A = X X^T, MN-major B operand of P' X
//   G  4 blocks (64 KB): Abar, then (once Abar Abar^T has been read) P'; K-major operand
// Because a hi block is followed by its lo block, one N=256 K-major B operand starting at a
// hi block reads [hi; lo] stacked: a single instruction gives hi*hi^T and hi*lo^T side by
// side, and a second N=128 one gives lo*hi^T.
// The polynomial is applied in completed-square form, which leaves the epilogues nothing
// but a scale, a diagonal shift and the hi/lo split (no re-reading of A or X):
//   a X + (b A + c A^2) X = P' X,  P' = c Abar Abar^T + g I,  Abar = A + beta I,
//   beta = b / (2c),  g = a - b^2 / (4c)
// (A is symmetric, so Abar Abar = Abar Abar^T: both operands are read K-major). The
// lo*hi^T term of products 0 and 1 accumulates onto the hi*hi^T columns, so every product
// takes 256 TMEM columns: product n of the kernel writes columns (n % 2) * 256 .. +255 and
// the epilogue of product n overlaps the MMAs of product n + 1.
//
// Roles (544 threads): warps 0-15 drain TMEM (warp w: lanes 32 (w % 4) .. +31 = matrix
// rows, 16 of the 64 columns of each round), warp 16 allocates TMEM and issues the MMAs.
// Each epilogue proceeds in rounds of 64 columns; when all 16 warps have written a round, the
// next product's MMAs over that 64-wide K block start (one mbarrier per round), so the
// products run back to back with only the last round of each epilogue exposed:
//   product 0  A = X X^T        K = 256 (4 blocks), waits for the rounds of X
//   product 1  Abar Abar^T      K = 128 (2 blocks), waits for the rounds of Abar
//   product 2  X <- P' X        K = 128 (2 blocks), waits for the rounds of P'
// Every epilogue value is a sum of at most two accumulator columns, scaled and split; the
// pair arithmetic uses packed fp32x2 instructions.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ops.h"
#include "umma.cuh"

namespace ttt {
namespace {

using namespace umma;

constexpr int NS_EPI_WARPS = 16;
constexpr int NS_EPI = 32 * NS_EPI_WARPS;   // epilogue threads
constexpr int NS_THREADS = NS_EPI + 32;     // + the MMA warp
constexpr int NS_ROWS = 128, NS_COLS = 256;
constexpr int BLK = 128 * 128;     // one 64-column block of 128 rows, bytes
constexpr int KB = 2 * BLK;        // hi + lo block pair of one 64-column range
constexpr int X_OFF = 0, G_OFF = 4 * KB;
constexpr int BAR_OFF = 6 * KB;
// mbarriers: 0 product done (MMA commit), 1-2 rounds of A, 3-4 rounds of P, 5-8 rounds of
// the X update, 9 final drain of the MMA pipe
constexpr int NBAR = 10;
constexpr int NS_SMEM = BAR_OFF + 256 + 1024;  // + barriers/flags + alignment slack
constexpr int NORM_BATCH = 8;      // float4 loads in flight per thread for the norm
constexpr int LD_BATCH = 4;        // 8-column chunks per thread per batch of global loads

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

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
// Values of a finished tcgen05.ld: the empty asm ties every use to the wait before it.
__device__ __forceinline__ void pin16(uint32_t (&a)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) asm volatile("" : "+r"(a[i]));
}
// (x0, x1) -> bf16x2 words hi = bf16(x) and lo = bf16(x - float(hi)), both round to
// nearest; x - float(hi) is exact and formed as one packed fma with -1.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  asm("{\n\t.reg .b64 X, H, N;\n\t.reg .b32 a, b, m;\n\t"
      "cvt.rn.bf16x2.f32 %0, %3, %2;\n\t"
      "shl.b32 a, %0, 16;\n\t"
      "and.b32 b, %0, 0xffff0000;\n\t"
      "mov.b32 m, 0fBF800000;\n\t"
      "mov.b64 X, {%2, %3};\n\t"
      "mov.b64 H, {a, b};\n\t"
      "mov.b64 N, {m, m};\n\t"
      "fma.rn.f32x2 X, H, N, X;\n\t"
      "mov.b64 {a, b}, X;\n\t"
      "cvt.rn.bf16x2.f32 %1, b, a;\n\t}"
      : "=r"(hi), "=r"(lo)
      : "f"(x0), "f"(x1));
}
// (u0 + u1, w0 + w1) * s as one packed add and one packed multiply.
__device__ __forceinline__ void add_scale_pair(uint32_t u0, uint32_t u1, uint32_t w0,
                                               uint32_t w1, float s, float& o0, float& o1) {
  asm("{\n\t.reg .b64 U, W, S;\n\t"
      "mov.b64 U, {%2, %3};\n\tmov.b64 W, {%4, %5};\n\tmov.b64 S, {%6, %6};\n\t"
      "add.rn.f32x2 U, U, W;\n\tmul.rn.f32x2 U, U, S;\n\t"
      "mov.b64 {%0, %1}, U;\n\t}"
      : "=f"(o0), "=f"(o1)
      : "r"(u0), "r"(u1), "r"(w0), "r"(w1), "f"(s));
}
// 8 values -> the hi chunk at base + off and the lo chunk at base + off + BLK.
__device__ __forceinline__ void store_split8x(uint32_t base, uint32_t off, const float* v) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) split_pair(v[2 * t], v[2 * t + 1], h[t], l[t]);
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + off), "r"(h[0]),
               "r"(h[1]), "r"(h[2]), "r"(h[3])
               : "memory");
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + off + BLK), "r"(l[0]),
               "r"(l[1]), "r"(l[2]), "r"(l[3])
               : "memory");
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
// X = U^T with 16-byte access: unit u covers rows 4a .. 4a+3 and chunk q of X, i.e. the
// float4s U[8q + t][4a .. 4a+3], t < 8. Eight consecutive lanes take consecutive a (one
// 128-byte segment of a row of U), four lane groups take four q (shared-memory chunks in
// eight distinct 16-byte bank slots).
__device__ __forceinline__ void quad_of(int u, int& a, int& q) {
  a = (u & 7) + 8 * ((u >> 5) & 3);
  q = ((u >> 3) & 3) + 4 * (u >> 7);
}

__global__ void __launch_bounds__(NS_THREADS, 1)
    ns_mma_kernel(float* U, NsLayout Lay, int steps, float eps, float cc, float beta, float g,
                  unsigned* err, unsigned long long wait_ns) {
  extern __shared__ uint8_t ns_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(ns_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  float* red = reinterpret_cast<float*>(tslot + 2);   // [16] warp partial sums

  const int p = blockIdx.x, z = blockIdx.y;
  if (!(Lay.mask & (1 << p))) return;
  const int R = Lay.R[p], Cc = Lay.C[p];               // U's own [R, Cc]
  const bool tr = R > Cc;
  const int r = tr ? Cc : R, cols = tr ? R : Cc;       // iterate on [r, cols], r <= cols
  const long long hm = (long long)R * Cc;
  float* u = U + z * Lay.zstride + p * Lay.pstride;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool epi = warp < NS_EPI_WARPS;
  const uint32_t sb = smem_u32(smem);
  const uint32_t sX = sb + X_OFF, sG = sb + G_OFF;
  auto bar = [&](int i) { return smem_u32(bars + i); };
  // 16-byte vector access to U: aligned base and whole float4s per row
  const bool vec = ((reinterpret_cast<uintptr_t>(u) & 15) == 0) && ((Cc & 3) == 0);

  if (warp == NS_EPI_WARPS) {
    if (lane == 0) {
      mbar_init(bar(0), 1);
      for (int i = 1; i <= 8; ++i) mbar_init(bar(i), NS_EPI_WARPS);
      mbar_init(bar(9), 1);
      *abort_flag = 0;
      mbar_fence_init();
    }
    __syncwarp();
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }

  // ||U||_F, NORM_BATCH independent loads in flight per thread
  float ss = 0.0f;
  if (epi) {
    if (vec) {
      const float4* u4 = reinterpret_cast<const float4*>(u);
      const long long n4 = hm >> 2;
      for (long long e0 = tid; e0 < n4; e0 += (long long)NS_EPI * NORM_BATCH) {
        float4 t[NORM_BATCH];
#pragma unroll
        for (int k = 0; k < NORM_BATCH; ++k) {
          const long long e = e0 + (long long)k * NS_EPI;
          t[k] = e < n4 ? u4[e] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < NORM_BATCH; ++k)
          ss = fmaf(t[k].x, t[k].x, fmaf(t[k].y, t[k].y, fmaf(t[k].z, t[k].z,
                                                             fmaf(t[k].w, t[k].w, ss))));
      }
    } else {
      for (long long e0 = tid; e0 < hm; e0 += (long long)NS_EPI * NORM_BATCH) {
        float t[NORM_BATCH];
#pragma unroll
        for (int k = 0; k < NORM_BATCH; ++k) {
          const long long e = e0 + (long long)k * NS_EPI;
          t[k] = e < hm ? u[e] : 0.0f;
        }
#pragma unroll
        for (int k = 0; k < NORM_BATCH; ++k) ss = fmaf(t[k], t[k], ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) red[warp] = ss;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  float tot = 0.0f;
#pragma unroll
  for (int w = 0; w < NS_EPI_WARPS; ++w) tot += red[w];
  const float scale = 1.0f / (sqrtf(tot) + eps);
  const uint32_t tmem = *tslot;

  // X = U * scale in the [r, cols] orientation, zero padded to 128 x 256
  constexpr int NCHUNK = NS_ROWS * (NS_COLS / 8);
  if (epi && tr && vec) {
    constexpr int NQUAD = NCHUNK / 4, QB = 1;
    for (int u0 = tid; u0 < NQUAD; u0 += NS_EPI * QB) {
      float4 f[QB][8];
#pragma unroll
      for (int k = 0; k < QB; ++k) {
        int a, q;
        quad_of(u0 + k * NS_EPI, a, q);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int j = 8 * q + t;
          f[k][t] = (4 * a < r && j < cols)
                        ? *reinterpret_cast<const float4*>(u + (long long)j * Cc + 4 * a)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int k = 0; k < QB; ++k) {
        int a, q;
        quad_of(u0 + k * NS_EPI, a, q);
        float v[4][8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          v[0][t] = f[k][t].x * scale;
          v[1][t] = f[k][t].y * scale;
          v[2][t] = f[k][t].z * scale;
          v[3][t] = f[k][t].w * scale;
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) store_split8(sX, chunk_off(4 * a + ii, q), v[ii]);
      }
    }
  } else if (epi) {
    for (int e0 = tid; e0 < NCHUNK; e0 += NS_EPI * LD_BATCH) {
      float v[LD_BATCH][8];
#pragma unroll
      for (int k = 0; k < LD_BATCH; ++k) {
        int i, q;
        chunk_of(e0 + k * NS_EPI, tr, i, q);
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
        chunk_of(e0 + k * NS_EPI, tr, i, q);
#pragma unroll
        for (int t = 0; t < 8; ++t) v[k][t] *= scale;
        store_split8(sX, chunk_off(i, q), v[k]);
      }
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == NS_EPI_WARPS) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID256 = make_idesc_bf16(128, 256, false, false);
      constexpr uint32_t ID128 = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t IDPX = make_idesc_bf16(128, 256, false, true);
      bool go = true, issued = false;
      for (int it = 0; it < steps && go; ++it) {
        for (int k = 0; k < 3 && go; ++k) {
          const int n = 3 * it + k;
          const uint32_t D = tmem + (uint32_t)((n & 1) * 256);
          const int nkb = k == 0 ? 4 : 2;
          for (int kb = 0; kb < nkb && go; ++kb) {
            if (n > 0) {   // this K block's operand columns: one round of the last epilogue
              const int rb = k == 0 ? 5 + kb : (k == 1 ? 1 + kb : 3 + kb);
              const uint32_t par = (uint32_t)((k == 0 ? it - 1 : it) & 1);
              if (!(go = mbar_wait(bar(rb), par, abort_flag, err, wait_ns))) break;
              tc_fence_after();
            }
            issued = true;
            for (int k0 = 64 * kb; k0 < 64 * kb + 64; k0 += 16) {
              if (k < 2) {     // [hi*hi^T | hi*lo^T], then lo*hi^T onto the first half
                const uint32_t base = k == 0 ? sX : sG;
                mma_f16(D, kmajor(base, k0), kmajor(base, k0), ID256, k0 > 0);
                mma_f16(D, kmajor(base + BLK, k0), kmajor(base, k0), ID128, 1);
              } else {         // P X: hi*hi + hi*lo + lo*hi
                mma_f16(D, kmajor(sG, k0), mnmajor(sX, k0), IDPX, k0 > 0);
                mma_f16(D, kmajor(sG, k0), mnmajor(sX + BLK, k0), IDPX, 1);
                mma_f16(D, kmajor(sG + BLK, k0), mnmajor(sX, k0), IDPX, 1);
              }
            }
          }
          if (go) mma_commit(bar(0));
        }
      }
      if (issued) {   // every issued MMA has finished before TMEM and shared memory go
        mma_commit(bar(9));
        mbar_wait(bar(9), 0, abort_flag, nullptr, wait_ns, true);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue warps
    const int quarter = warp & 3, sub = warp >> 2;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int row = quarter * 32 + lane;   // TMEM lane = matrix row
    bool go = true;
    for (int it = 0; it < steps && go; ++it) {
      for (int k = 0; k < 3 && go; ++k) {
        const int n = 3 * it + k;
        // warp-uniform outcome: the lanes take the same path through the rounds below
        go = __all_sync(0xffffffffu,
                        mbar_wait(bar(0), (uint32_t)(n & 1), abort_flag, err, wait_ns));
        if (!go) break;
        tc_fence_after();
        const uint32_t D = lane_base + (uint32_t)((n & 1) * 256);
        const int nr = k == 2 ? 4 : 2;
        for (int rd = 0; rd < nr; ++rd) {
          // this warp's 16 columns of the round: chunks q0, q0 + 1 of its row
          const int c0 = 64 * rd + 16 * sub, q0 = c0 >> 3;
          const uint32_t base = k == 2 ? sX : sG;
          uint32_t x0[16];
          float v[16];
          if (k < 2) {
            // (hi*hi^T + lo*hi^T) + hi*lo^T, times 1 (Abar) or c (P')
            uint32_t x1[16];
            tmem_ld16(D + (uint32_t)c0, x0);
            tmem_ld16(D + 128u + (uint32_t)c0, x1);
            tmem_ld_wait();
            pin16(x0);
            pin16(x1);
            const float sc = k == 0 ? 1.0f : cc;
#pragma unroll
            for (int t = 0; t < 16; t += 2)
              add_scale_pair(x0[t], x0[t + 1], x1[t], x1[t + 1], sc, v[t], v[t + 1]);
            // the diagonal shift: beta for Abar, g for P' (this warp's columns meet the
            // diagonal only where they overlap its 32 rows)
            if (c0 + 16 > quarter * 32 && c0 < quarter * 32 + 32) {
              const float dg = k == 0 ? beta : g;
#pragma unroll
              for (int t = 0; t < 16; ++t)
                if (c0 + t == row) v[t] += dg;
            }
          } else {
            // X <- P' X
            tmem_ld16(D + (uint32_t)c0, x0);
            tmem_ld_wait();
            pin16(x0);
#pragma unroll
            for (int t = 0; t < 16; ++t) v[t] = __uint_as_float(x0[t]);
          }
          store_split8x(base, chunk_off(row, q0), v);
          store_split8x(base, chunk_off(row, q0 + 1), v + 8);
          // this round's shared-memory writes -> the MMAs of the next product
          fence_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(k == 0 ? 1 + rd : (k == 1 ? 3 + rd : 5 + rd)));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  const bool ok = *abort_flag == 0;

  if (ok && epi) {
    // U <- X in U's orientation
    if (tr && vec) {
      for (int u0 = tid; u0 < NCHUNK / 4; u0 += NS_EPI) {
        int a, q;
        quad_of(u0, a, q);
        if (4 * a >= r || 8 * q >= cols) continue;
        float x[4][8];
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) load_join8(sX, chunk_off(4 * a + ii, q), x[ii]);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int j = 8 * q + t;
          if (j < cols)
            *reinterpret_cast<float4*>(u + (long long)j * Cc + 4 * a) =
                make_float4(x[0][t], x[1][t], x[2][t], x[3][t]);
        }
      }
    } else {
      for (int e = tid; e < NCHUNK; e += NS_EPI) {
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
    }
  }
  if (warp == NS_EPI_WARPS) {
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
  if (c == 0.0f) return cudaErrorInvalidValue;   // the completed square needs c != 0
  cudaError_t e =
      cudaFuncSetAttribute(ns_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, NS_SMEM);
  if (e != cudaSuccess) return e;
  const float beta = (float)((double)b / (2.0 * (double)c));
  const float g = (float)((double)a - (double)b * (double)b / (4.0 * (double)c));
  ns_mma_kernel<<<dim3(L.parts, Z), NS_THREADS, NS_SMEM, s>>>(U, L, steps, eps, c, beta, g,
                                                              err, wait_ns);
  return cudaGetLastError();
}

}  // namespace ttt
