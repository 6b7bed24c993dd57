// Tensor-core batched GEMM engine for sm_100a: bf16 operands staged in shared memory by
// TMA (128-byte swizzle, one destination CTA), tcgen05.mma kind::f16 with fp32 accumulators in
// tensor memory, and CUDA-core epilogues that read TMEM with tcgen05.ld.
//
// Persistent CTAs walk the 128 x BN output tiles of all batch entries round-robin. Two
// TMEM accumulators alternate, so the epilogue of one tile overlaps the MMAs of the next.
// Warp roles (320 threads):
//   warp 0 (one lane)  TMA producer over a STAGES-deep shared-memory ring
//   warp 1             TMEM allocation; one lane issues the MMAs and the commits
//   warps 2..9         epilogue; warp w reads TMEM lanes 32*(w%4) .. +31, and warps 2-5 /
//                      6-9 take the first / second half of the tile's columns
// Epilogue modes:
//   STORE*  C = alpha * acc + beta * Cin (fp32 or bf16 C): lane-per-row stores, TMA stores
//           from per-warp staging boxes (no addend), row-contiguous stores through a staged
//           chunk (fp32 with an addend; optionally a bf16 copy)
//   SWIGLU  the tile's columns are [A block | B block] of the fused SwiGLU input weights;
//           writes phi = silu(a) * b times a per-row factor (bf16), and optionally the
//           unscaled phi to a second output; the gradient variant writes the recurrent
//           form's pieces (phi * eta, D * silu(a), D * b * silu'(a)) instead, in one pass.
// tf32 operands (TF): fp32 A and B through the same 128-byte-swizzled k-blocks (K-major: 32
// fp32 of K per 128-byte row instead of 64 bf16; MN-major: 32-element MN blocks of 32 k rows,
// 4 KB apart, in the 128-byte swizzle on 32-byte chunks) and tcgen05.mma kind::tf32.
// Every mbarrier wait is bounded; a timeout records DEVERR_TIMEOUT in the device error
// word, raises a CTA-wide abort flag, and the CTA drains its in-flight copies and MMAs
// (again with bounded waits) and frees its TMEM before returning.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <mutex>

#include "gemm.h"
#include "swiglu_epi.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

using namespace umma;

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;

// STORE: each lane stores its row directly (no addend, or bf16 C). STORE_STG: fp32 C with an
// addend, staged per warp so Cin loads and C stores are row-contiguous. STORE_COPY: STORE_STG
// plus a bf16 copy of the result. STORE_TMA: C without an addend, each warp's 32 rows
// staged 64 bf16 (or 32 fp32) columns at a time in its 4 KB box and written with TMA tensor
// stores.
// Separate instantiations, so no mode pays for another's code.
enum EpiMode : int {
  EPI_STORE = 0, EPI_SWIGLU = 1, EPI_STORE_STG = 2, EPI_STORE_COPY = 3, EPI_STORE_TMA = 5
};

struct UArgs {
  int M, N, K, Z0, Z1;
  int a_b0, a_b1, b_b0, b_b1;  // 1 = operand uses that batch coordinate
  void* C; long long ldc, cs0, cs1;
  __nv_bfloat16* C16;   // fp32 C: bf16 copy with C's strides, or null
  const float* Cin; long long ldi, is0, is1;
  float alpha, beta;
  const float* zss; float zeps; int zpa, zpb;   // per-z0 scale of alpha / beta, or null
  // SWIGLU: phi columns < n_valid are written; row factor rs[z0*rs0 + z1*rs1 + row]
  void* C2; long long ld2, c2s0, c2s1;
  const float* rs; long long rs0, rs1;
  int n_valid;
  // SWIGLU gradient variant: third output and the Dv input (bf16)
  int grad;
  int skip_out1;
  void* C3;
  const __nv_bfloat16* dv; long long ldd, ds0, ds1;
  unsigned* err;
  unsigned long long wait_ns;
};

// Shared-memory layout. Streaming mode: a ring of STAGES (A tile + B tile) stages.
// B-resident mode (BRES): the CTA's whole B tile for K <= 256 (up to four 64-wide k-blocks)
// stays in shared memory and the ring carries only A tiles.
// Every mode but the lane-per-row STORE adds 32 KB of staging, one 4 KB box per epilogue
// warp: SWIGLU and STORE_TMA stage 32 rows x 64 bf16 (or 32 fp32) columns and store them
// with TMA; STORE_STG / COPY stage 32 x 32 fp32 values and write them back row-contiguous.
template <int BN, int STAGES, bool BRES, int MODE>
struct Smem {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;             // one k-block of B
  static constexpr int B_RES = BRES ? 4 * B_BYTES : 0;    // resident B, at most 4 k-blocks
  static constexpr int STAGE = BRES ? A_BYTES : A_BYTES + B_BYTES;
  // one 4 KB box per epilogue warp
  static constexpr int OUT_BYTES =
      MODE == EPI_STORE ? 0 : BM * 128 * 2;
  static constexpr int OUT_OFF = B_RES;
  static constexpr int RING_OFF = OUT_OFF + OUT_BYTES;
  static constexpr int BAR_OFF = RING_OFF + STAGES * STAGE;
  static constexpr int TOTAL = BAR_OFF + 256 + 1024;      // + barriers + alignment slack
};

// 32 consecutive values of a row to 16-byte-aligned memory.
__device__ __forceinline__ void store32(float* dst, const float (&w)[32]) {
#pragma unroll
  for (int j = 0; j < 32; j += 4)
    *reinterpret_cast<float4*>(dst + j) = make_float4(w[j], w[j + 1], w[j + 2], w[j + 3]);
}
__device__ __forceinline__ void store32(__nv_bfloat16* dst, const float (&w)[32]) {
#pragma unroll
  for (int j = 0; j < 32; j += 8) {
    uint4 pk;
    pk.x = pack_bf16x2(w[j], w[j + 1]);
    pk.y = pack_bf16x2(w[j + 2], w[j + 3]);
    pk.z = pack_bf16x2(w[j + 4], w[j + 5]);
    pk.w = pack_bf16x2(w[j + 6], w[j + 7]);
    *reinterpret_cast<uint4*>(dst + j) = pk;
  }
}

// Four consecutive values to 16-byte-aligned fp32 memory.
__device__ __forceinline__ void store4(float* dst, const float (&x)[4]) {
  *reinterpret_cast<float4*>(dst) = make_float4(x[0], x[1], x[2], x[3]);
}

struct TileCoord {
  int tm, tn, z0, z1;
};

__device__ __forceinline__ TileCoord decode_tile(int t, int tiles_n, int tiles_mn, int Z0) {
  TileCoord c;
  const int z = t / tiles_mn, rem = t - z * tiles_mn;
  c.tm = rem / tiles_n;
  c.tn = rem - c.tm * tiles_n;
  c.z0 = z % Z0;
  c.z1 = z / Z0;
  return c;
}

// The sequence of tiles one CTA processes; every warp role walks the same sequence.
// Streaming mode: tiles blockIdx.x, blockIdx.x + gridDim.x, ... of the (z, tm, tn) order
// (n fastest, so the CTAs working at the same time share A tiles in L2).
// B-resident mode: CTA c keeps n-tile c % tiles_n and walks a contiguous range of the
// flattened (z, tm) row tiles, shared with the other n-tile CTAs of its group, so a
// group reads each A tile from HBM once and each CTA reloads B only when z changes.
struct TileWalker {
  int tiles_n, tiles_m, Z0, total, count;
  int bres, nt, r0;
  __device__ TileWalker(int M, int N, int Z0_, int Z1, int BN, bool b_res) {
    tiles_n = (N + BN - 1) / BN;
    tiles_m = (M + BM - 1) / BM;
    Z0 = Z0_;
    total = tiles_n * tiles_m * Z0_ * Z1;
    bres = b_res;
    if (!b_res) {
      count = blockIdx.x < (unsigned)total ? (total - 1 - blockIdx.x) / gridDim.x + 1 : 0;
      nt = r0 = 0;
    } else {
      const int groups = gridDim.x / tiles_n, g = blockIdx.x / tiles_n;
      const int rows = tiles_m * Z0_ * Z1;
      nt = blockIdx.x % tiles_n;
      if (g >= groups) {
        count = 0;
        r0 = 0;
      } else {
        const long long lo = (long long)rows * g / groups, hi = (long long)rows * (g + 1) / groups;
        r0 = (int)lo;
        count = (int)(hi - lo);
      }
    }
  }
  __device__ TileCoord at(int i) const {
    if (!bres) return decode_tile(blockIdx.x + i * gridDim.x, tiles_n, tiles_n * tiles_m, Z0);
    const int r = r0 + i, z = r / tiles_m;
    TileCoord c;
    c.tm = r - z * tiles_m;
    c.tn = nt;
    c.z0 = z % Z0;
    c.z1 = z / Z0;
    return c;
  }
};

// Tensor maps of the (up to three) TMA-stored outputs of the SWIGLU epilogue.
struct OutMaps {
  CUtensorMap m[3];
};

template <int BN, bool A_MN, bool B_MN, int STAGES, int MODE, typename TC, bool BRES, bool TF>
__global__ void __launch_bounds__(THREADS, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ OutMaps om, const UArgs args) {
  static_assert(!TF || (!BRES && MODE != EPI_SWIGLU),
                "tf32 operands: streamed operands, plain epilogues");
  constexpr int BKE = TF ? 32 : BK;      // K elements per 128-byte k-block row
  using L = Smem<BN, STAGES, BRES, MODE>;
  constexpr uint32_t ACC_COLS = 2 * BN;  // two accumulators
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* b_full = acc_empty + 2;     // resident B loaded
  uint64_t* b_empty = b_full + 1;       // resident B no longer read by MMAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(b_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = (args.K + BKE - 1) / BKE;
  const TileWalker walk(args.M, args.N, args.Z0, args.Z1, BN, BRES);
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t ring_base = smem_base + L::RING_OFF;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), EPI_WARPS * 32);
    }
    mbar_init(smem_u32(b_full), 1);
    mbar_init(smem_u32(b_empty), 1);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), ACC_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  uint32_t issued = 0;   // producer: k-blocks whose loads were issued (all tiles)
  int b_loads = 0;       // producer: resident-B loads issued
  int mma_tiles = 0;     // MMA lane: tiles whose MMAs were issued
  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      int bkey = -1;
      for (int i = 0; i < walk.count && !*abort_flag; ++i) {
        const TileCoord tc = walk.at(i);
        const int ac2 = args.a_b0 ? tc.z0 : 0, ac3 = args.a_b1 ? tc.z1 : 0;
        const int bc2 = args.b_b0 ? tc.z0 : 0, bc3 = args.b_b1 ? tc.z1 : 0;
        if (BRES && (bc2 * 65536 + bc3) != bkey) {
          // (Re)load the CTA's B tile once the MMAs have stopped reading the previous one.
          if (b_loads > 0 && !mbar_wait(smem_u32(b_empty), (b_loads - 1) & 1, abort_flag,
                                        args.err, args.wait_ns))
            break;
          const uint32_t bb = smem_u32(b_full);
          mbar_arrive_expect_tx(bb, KB * L::B_BYTES);
          for (int kb = 0; kb < KB; ++kb) {
            const uint32_t sB = smem_base + kb * L::B_BYTES;
            const int kB = kb * BKE;
            if (B_MN) {
#pragma unroll
              for (int q = 0; q < BN / BKE; ++q)
                tma_load_4d(sB + q * BKE * 128, &tmB, bb, tc.tn * BN + BKE * q, kB, bc2, bc3);
            } else {
              tma_load_4d(sB, &tmB, bb, kB, tc.tn * BN, bc2, bc3);
            }
          }
          ++b_loads;
          bkey = bc2 * 65536 + bc3;
        }
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          if (it >= STAGES &&
              !mbar_wait(smem_u32(&empty[s]), ((it / STAGES) & 1) ^ 1, abort_flag, args.err,
                         args.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[s]);
          mbar_arrive_expect_tx(fb, L::STAGE);
          const uint32_t sA = ring_base + s * L::STAGE;
          const int kA = kb * BKE;
          if (A_MN) {
            // MN-major: BM / BKE blocks of BKE MN elements (128 bytes) x BKE k rows
#pragma unroll
            for (int q = 0; q < BM / BKE; ++q)
              tma_load_4d(sA + q * BKE * 128, &tmA, fb, tc.tm * BM + BKE * q, kA, ac2, ac3);
          } else {
            tma_load_4d(sA, &tmA, fb, kA, tc.tm * BM, ac2, ac3);
          }
          if (!BRES) {
            const uint32_t sB = sA + L::A_BYTES;
            const int kB = kb * BKE;
            if (B_MN) {
#pragma unroll
              for (int q = 0; q < BN / BKE; ++q)
                tma_load_4d(sB + q * BKE * 128, &tmB, fb, tc.tn * BN + BKE * q, kB, bc2, bc3);
            } else {
              tma_load_4d(sB, &tmB, fb, kB, tc.tn * BN, bc2, bc3);
            }
          }
          issued = it + 1;
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC =
          TF ? make_idesc_tf32(BM, BN, A_MN, B_MN) : make_idesc_bf16(BM, BN, A_MN, B_MN);
      uint32_t it = 0;
      int bkey = -1, b_uses = 0;
      bool ok = true;
      for (int lt = 0; lt < walk.count && ok; ++lt) {
        const TileCoord tc = walk.at(lt);
        const int buf = lt & 1;
        if (lt >= 2 && !mbar_wait(smem_u32(&acc_empty[buf]), ((lt >> 1) & 1) ^ 1, abort_flag,
                                  args.err, args.wait_ns)) {
          ok = false;
          break;
        }
        if (BRES) {
          const int key = (args.b_b0 ? tc.z0 : 0) * 65536 + (args.b_b1 ? tc.z1 : 0);
          if (key != bkey) {
            if (b_uses > 0) mma_commit(smem_u32(b_empty));  // old B free once MMAs finish
            if (!mbar_wait(smem_u32(b_full), b_uses & 1, abort_flag, args.err, args.wait_ns)) {
              ok = false;
              break;
            }
            ++b_uses;
            bkey = key;
          }
        }
        tc_fence_after();
        const uint32_t dt = tmem + (uint32_t)(buf * BN);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(smem_u32(&full[s]), (it / STAGES) & 1, abort_flag, args.err,
                         args.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = ring_base + s * L::STAGE;
          const uint32_t sB = BRES ? smem_base + kb * L::B_BYTES : sA + L::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // one instruction covers 32 bytes of K: K-major, 32 bytes along the row; MN-major,
            // 16 (bf16) or 8 (tf32) k rows of 128 bytes, MN blocks BKE * 128 bytes apart
            // (tf32: the 32-byte-base swizzle, 4-row groups 512 bytes apart)
            auto mn_desc = [&](uint32_t base) {
              return TF ? make_sw128b32_desc(base + kk * 1024, BKE * 128, 512)
                        : make_sw128_desc(base + kk * 2048, BKE * 128, 1024);
            };
            const uint64_t ad = A_MN ? mn_desc(sA) : make_sw128_desc(sA + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? mn_desc(sB) : make_sw128_desc(sB + kk * 32, 16, 1024);
            if constexpr (TF)
              mma_tf32(dt, ad, bd, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
            else
              mma_f16(dt, ad, bd, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(smem_u32(&empty[s]));
        }
        // Arrives once the tile's MMAs are done (also on the abort path, so the teardown
        // can wait for in-flight MMAs before freeing TMEM).
        mma_commit(smem_u32(&acc_full[buf]));
        mma_tiles = lt + 1;
      }
    }
  } else {
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int part = ew >> 2;  // 0: first half of the tile's columns, 1: second half
    int grad_stores = 0;       // gradient epilogue: stores issued (sub-box = count % 2)
    for (int lt = 0; lt < walk.count; ++lt) {
      const int buf = lt & 1;
      const TileCoord tc = walk.at(lt);
      const int row = tc.tm * BM + quarter * 32 + lane;
      // the SwiGLU row scale is fetched before the wait, so its latency hides behind it
      const float rsv = (MODE == EPI_SWIGLU && !args.grad && args.rs && row < args.M)
                            ? args.rs[tc.z0 * args.rs0 + tc.z1 * args.rs1 + row]
                            : 1.0f;
      bool ok = mbar_wait(smem_u32(&acc_full[buf]), (lt >> 1) & 1, abort_flag, args.err,
                          args.wait_ns);
      if (!ok) break;
      tc_fence_after();
      const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
      if constexpr (MODE != EPI_SWIGLU) {
        float alpha = args.alpha, beta = args.beta;
        if (args.zss) {
          const float sc = 1.0f / (sqrtf(args.zss[tc.z0]) + args.zeps);
          if (args.zpa) alpha *= args.zpa == 2 ? sc * sc : sc;
          if (args.zpb) beta *= sc;
        }
        // alpha * acc (+ beta * Cin): each lane holds one row. EPI_STORE: each lane stores its
        // row's values directly (stores do not wait, so their scatter costs little).
        // EPI_STORE_STG / COPY (fp32 C with an addend): per 32-column chunk the warp stages
        // its 32 x 32 values in shared memory (128-byte rows, 16-byte chunks XOR-swizzled by
        // row) and writes them back row-contiguous, eight lanes per row, so the loads of Cin,
        // which the lanes wait for, are coalesced too.
        constexpr int HALF = BN / 2;
        const int rbase = tc.tm * BM + quarter * 32;
        TC* cbase = static_cast<TC*>(args.C) + tc.z0 * args.cs0 + tc.z1 * args.cs1;
        const float* ibase =
            args.Cin ? args.Cin + tc.z0 * args.is0 + tc.z1 * args.is1 : nullptr;
        const bool vec =
            ((reinterpret_cast<uintptr_t>(cbase) | reinterpret_cast<uintptr_t>(ibase)) & 15) ==
                0 &&
            (args.ldc * (long long)sizeof(TC)) % 16 == 0 && (!ibase || args.ldi % 4 == 0);
        const int rr0 = lane >> 3, cq = (lane & 7) * 4;
        if constexpr (MODE == EPI_STORE_TMA) {
          // alpha * acc (bf16: 64 columns, fp32: 32 columns per 128-byte box row) per TMA
          // store from this warp's 4 KB box; the accumulator is released after the last
          // TMEM read
          constexpr int PC = sizeof(TC) == 2 ? 64 : 32;   // columns per store
          static_assert(HALF % PC == 0, "whole store boxes");
          const uint32_t box = smem_base + L::OUT_OFF + ew * 4096;
          const int oy = tc.tm * BM + quarter * 32;
          const int c2 = args.cs0 ? tc.z0 : 0, c3 = args.cs1 ? tc.z1 : 0;
#pragma unroll
          for (int c0 = 0; c0 < HALF; c0 += PC) {
            const int ox = tc.tn * BN + part * HALF + c0;
            uint32_t ra[32], rb[32];
            tmem_ld32(lane_addr + (uint32_t)(part * HALF + c0), ra);
            if constexpr (PC == 64) {
              tmem_ld32(lane_addr + (uint32_t)(part * HALF + c0 + 32), rb);
              tmem_ld_wait_regs(ra, rb);
            } else {
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) asm volatile("" : "+r"(ra[j]));
            }
            if (c0 + PC >= HALF) {
              tc_fence_before();
              mbar_arrive(smem_u32(&acc_empty[buf]));
            }
            if (ox >= args.N) continue;
            if (lane == 0) tma_store_wait_read();
            __syncwarp();
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
              const uint32_t addr = box + lane * 128 + ((cc ^ (lane & 7)) << 4);
              uint32_t w[4];
              if constexpr (PC == 64) {
                const uint32_t* v = cc < 4 ? &ra[8 * cc] : &rb[8 * (cc - 4)];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  w[q] = pack_bf16x2(alpha * __uint_as_float(v[2 * q]),
                                     alpha * __uint_as_float(v[2 * q + 1]));
              } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  w[q] = __float_as_uint(alpha * __uint_as_float(ra[4 * cc + q]));
              }
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]),
                           "r"(w[1]), "r"(w[2]), "r"(w[3])
                           : "memory");
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_4d(&om.m[0], box, ox, oy, c2, c3);
              tma_store_commit();
            }
          }
        } else if constexpr (MODE == EPI_STORE) {
          uint32_t r[HALF];
#pragma unroll
          for (int c0 = 0; c0 < HALF; c0 += 32)
            tmem_ld32(lane_addr + (uint32_t)(part * HALF + c0),
                      *reinterpret_cast<uint32_t(*)[32]>(&r[c0]));
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < HALF; ++j) asm volatile("" : "+r"(r[j]));
          tc_fence_before();
          mbar_arrive(smem_u32(&acc_empty[buf]));
          if (row < args.M) {
            TC* crow = cbase + (long long)row * args.ldc;
            const float* irow = ibase ? ibase + (long long)row * args.ldi : nullptr;
            const bool vrow = ((reinterpret_cast<uintptr_t>(crow) & 15) == 0) &&
                              ((args.ldc * (long long)sizeof(TC)) % 16 == 0);
#pragma unroll
            for (int c0 = 0; c0 < HALF; c0 += 32) {
              const int col0 = tc.tn * BN + part * HALF + c0;
              const int nv = min(32, args.N - col0);
              if (nv <= 0) break;
              float w[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) w[j] = alpha * __uint_as_float(r[c0 + j]);
              if (irow) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (j < nv) w[j] += beta * irow[col0 + j];
              }
              if (vrow && nv == 32) {
                store32(crow + col0, w);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (j < nv) crow[col0 + j] = from_f32<TC>(w[j]);
              }
            }
          }
        } else {
          // the accumulator is read 32 columns at a time and released after the last read
          float4* sbuf = reinterpret_cast<float4*>(smem + L::OUT_OFF + ew * 4096);
#pragma unroll
          for (int c0 = 0; c0 < HALF; c0 += 32) {
            const int col0 = tc.tn * BN + part * HALF + c0;
            uint32_t r[32];
            tmem_ld32(lane_addr + (uint32_t)(part * HALF + c0), r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) asm volatile("" : "+r"(r[j]));
            // the last chunk with columns inside N releases the accumulator, exactly once
            const bool last = c0 + 32 >= HALF || col0 + 32 >= args.N;
            if (last) {
              tc_fence_before();
              mbar_arrive(smem_u32(&acc_empty[buf]));
            }
            if (col0 >= args.N) break;
            const int col = col0 + cq;
            const bool cfull = vec && col + 4 <= args.N;
            // this chunk's Cin values first, all eight 16-byte loads in flight together
            float4 cin[8];
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int row_o = rbase + it * 4 + rr0;
              cin[it] = (ibase && cfull && row_o < args.M)
                            ? *reinterpret_cast<const float4*>(
                                  ibase + (long long)row_o * args.ldi + col)
                            : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            }
            __syncwarp();   // the previous chunk's staged values have been read
#pragma unroll
            for (int q = 0; q < 8; ++q)
              sbuf[lane * 8 + (q ^ (lane & 7))] =
                  make_float4(alpha * __uint_as_float(r[4 * q]),
                              alpha * __uint_as_float(r[4 * q + 1]),
                              alpha * __uint_as_float(r[4 * q + 2]),
                              alpha * __uint_as_float(r[4 * q + 3]));
            __syncwarp();
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int rr = it * 4 + rr0, row_o = rbase + rr;
              const float4 sv = sbuf[rr * 8 + ((cq >> 2) ^ (rr & 7))];
              if (row_o >= args.M || col >= args.N) continue;
              TC* crow = cbase + (long long)row_o * args.ldc;
              float x[4] = {sv.x, sv.y, sv.z, sv.w};
              if (cfull) {
                if (ibase) {
                  x[0] = fmaf(beta, cin[it].x, x[0]);
                  x[1] = fmaf(beta, cin[it].y, x[1]);
                  x[2] = fmaf(beta, cin[it].z, x[2]);
                  x[3] = fmaf(beta, cin[it].w, x[3]);
                }
                store4(crow + col, x);
                if constexpr (MODE == EPI_STORE_COPY) {
                  __nv_bfloat16* c16 = args.C16 + tc.z0 * args.cs0 + tc.z1 * args.cs1 +
                                       (long long)row_o * args.ldc + col;
                  *reinterpret_cast<uint2*>(c16) =
                      make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
                }
              } else {
                const float* irow = ibase ? ibase + (long long)row_o * args.ldi : nullptr;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  if (col + j >= args.N) break;
                  float y = x[j];
                  if (irow) y = fmaf(beta, irow[col + j], y);
                  crow[col + j] = from_f32<TC>(y);
                  x[j] = y;
                  if constexpr (MODE == EPI_STORE_COPY)
                    args.C16[tc.z0 * args.cs0 + tc.z1 * args.cs1 + (long long)row_o * args.ldc +
                             col + j] = __float2bfloat16_rn(y);
                }
              }
            }
            if (last) break;
          }
        }
      } else if (args.grad) {
        // Gradient pieces of the recurrent form in one pass: per 32-column half, A/2 and B
        // are read from TMEM once, tanh(a/2) is evaluated once per element, and the (up to)
        // three outputs are packed to bf16 together; each output half leaves through one of
        // this warp's two 2 KB sub-boxes (64-byte swizzle) with a TMA store, a sub-box being
        // refilled once the store before the last has read it. TMEM is released after the
        // second half's loads.
        constexpr int PH = BN / 2;
        constexpr int QW = PH / 2;
        const bool live = row < args.M;
        const float eta = live ? args.rs[tc.z0 * args.rs0 + tc.z1 * args.rs1 + row] : 0.0f;
        const __nv_bfloat16* dvrow =
            args.dv + tc.z0 * args.ds0 + tc.z1 * args.ds1 + (long long)(live ? row : 0) * args.ldd;
        const int ox = tc.tn * PH + part * QW;
        const int oy = tc.tm * BM + quarter * 32;
        const int c2 = args.cs0 ? tc.z0 : 0, c3 = args.cs1 ? tc.z1 : 0;
        const uint32_t box = smem_base + L::OUT_OFF + ew * 4096;
        const bool want[3] = {!args.skip_out1, args.C2 != nullptr, args.C3 != nullptr};
        const bool need_dv = want[1] || want[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          // this row's 32 dv values of the half, all four 16-byte loads in flight together
          uint4 dvq[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int col = ox + hh * 32 + j * 8;
            dvq[j] = (live && need_dv && col + 8 <= args.n_valid)
                         ? *reinterpret_cast<const uint4*>(dvrow + col)
                         : make_uint4(0u, 0u, 0u, 0u);
          }
          uint32_t ra[32], rb[32];
          tmem_ld32(lane_addr + (uint32_t)(part * QW + hh * 32), ra);
          tmem_ld32(lane_addr + (uint32_t)(PH + part * QW + hh * 32), rb);
          tmem_ld_wait_regs(ra, rb);
          if (hh == 1) {
            tc_fence_before();
            mbar_arrive(smem_u32(&acc_empty[buf]));
          }
          uint32_t pk[3][16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const uint32_t dw = (&dvq[j >> 3].x)[(j & 7) >> 1];
            const float2 dvf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dw));
            float v[3][2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              // accumulator half A holds a/2 (the operand carries W0 / 2)
              const float hlf = __uint_as_float(ra[j + u]), bb = __uint_as_float(rb[j + u]);
              const float t = tanh_fast(hlf);
              const float sg = fmaf(0.5f, t, 0.5f);   // sigmoid(a)
              const float sa = fmaf(hlf, t, hlf);     // silu(a) = (a/2)(1 + tanh(a/2))
              const float d = -eta * (u ? dvf.y : dvf.x);
              v[0][u] = sa * bb * eta;
              v[1][u] = d * sa;
              v[2][u] = d * bb * sg * fmaf(2.0f * hlf, 1.0f - sg, 1.0f);   // silu'(a)
            }
#pragma unroll
            for (int o = 0; o < 3; ++o) pk[o][j / 2] = pack_bf16x2(v[o][0], v[o][1]);
          }
#pragma unroll
          for (int o = 0; o < 3; ++o) {
            if (!want[o] || ox + hh * 32 >= args.n_valid) continue;
            const uint32_t sub = box + (uint32_t)((grad_stores & 1) * 2048);
            if (lane == 0) tma_store_wait_read_1();
            __syncwarp();
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const uint32_t addr = sub + lane * 64 + ((cc ^ ((lane >> 1) & 3)) << 4);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                           "r"(pk[o][4 * cc]), "r"(pk[o][4 * cc + 1]), "r"(pk[o][4 * cc + 2]),
                           "r"(pk[o][4 * cc + 3])
                           : "memory");
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_4d(&om.m[o], sub, ox + hh * 32, oy, c2, c3);
              tma_store_commit();
            }
            ++grad_stores;
          }
        }
      } else {
        // SWIGLU: phi column p of this tile uses accumulator columns p (A/2) and BN/2 + p (B).
        // Each epilogue warp owns 32 rows x 64 phi columns: two 32-column pieces, the
        // second piece's TMEM loads in flight while the first is computed. It stages them
        // in its own 4 KB box (128-byte swizzle) and its lane 0 stores the box with TMA,
        // so the warps never wait on each other; a warp reuses its box once its previous
        // store has read it. With a second output (the unscaled phi) the accumulator is
        // read twice and released after the second read.
        static_assert(BN == 256, "the SwiGLU epilogue works on 256-column tiles");
        constexpr int PH = BN / 2;       // phi columns per tile
        constexpr int QW = PH / 2;       // phi columns per epilogue warp
        const int ox = tc.tn * PH + part * QW;   // first phi column of this warp's box
        const int oy = tc.tm * BM + quarter * 32;
        const int c2 = args.cs0 ? tc.z0 : 0, c3 = args.cs1 ? tc.z1 : 0;
        const uint32_t box = smem_base + L::OUT_OFF + ew * 4096;
        const uint32_t ta = lane_addr + (uint32_t)(part * QW), tb = ta + (uint32_t)PH;
        const int nout = args.C2 ? 2 : 1;
        for (int o = 0; o < nout; ++o) {
          const float sc = o == 0 ? rsv : 1.0f;
          if (lane == 0) tma_store_wait_read();
          __syncwarp();
          uint32_t ra0[32], rb0[32], ra1[32], rb1[32];
          tmem_ld32(ta, ra0);
          tmem_ld32(tb, rb0);
          tmem_ld_wait_regs(ra0, rb0);
          tmem_ld32(ta + 32, ra1);
          tmem_ld32(tb + 32, rb1);
          swiglu_piece(ra0, rb0, sc, box, lane, 0);
          tmem_ld_wait_regs(ra1, rb1);
          if (o == nout - 1) {
            tc_fence_before();
            mbar_arrive(smem_u32(&acc_empty[buf]));
          }
          swiglu_piece(ra1, rb1, sc, box, lane, 4);
          fence_async_smem();
          __syncwarp();
          if (lane == 0 && ox < args.n_valid) {
            tma_store_4d(&om.m[o], box, ox, oy, c2, c3);
            tma_store_commit();
          }
        }
      }
    }
    if ((MODE == EPI_SWIGLU || MODE == EPI_STORE_TMA) && lane == 0)
      tma_store_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // Drain: the producer waits for its loads still in flight; warp 1 for its MMAs.
    if (warp == 0 && lane == 0) {
      const uint32_t lo = issued > (uint32_t)STAGES ? issued - STAGES : 0;
      for (uint32_t it = lo; it < issued; ++it)
        mbar_wait(smem_u32(&full[it % STAGES]), (it / STAGES) & 1, abort_flag, nullptr,
                  args.wait_ns, true);
      if (BRES && b_loads > 0)
        mbar_wait(smem_u32(b_full), (b_loads - 1) & 1, abort_flag, nullptr, args.wait_ns, true);
    }
    if (warp == 1 && lane == 0 && mma_tiles > 0) {
      const int lt = mma_tiles - 1;
      mbar_wait(smem_u32(&acc_full[lt & 1]), (lt >> 1) & 1, abort_flag, nullptr, args.wait_ns,
                true);
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, ACC_COLS);
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

int sm_count() {
  static int cache[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// 4-D map {inner, outer, z0, z1} over one operand; box {64, box_outer, 1, 1} (bf16), or
// {32, box_outer, 1, 1} over fp32 for tf32 operands (128-byte rows either way).
bool make_map(CUtensorMap* map, const GemmOperand& op, int rows, int K, int Z0, int Z1,
              int box_rows, bool tf32 = false) {
  auto fn = encode_fn();
  if (!fn) return false;
  const bool mn = op.mn_major;
  cuuint64_t dims[4];
  cuuint64_t strides[3];
  cuuint32_t box[4];
  cuuint32_t estr[4] = {1, 1, 1, 1};
  dims[0] = (cuuint64_t)(mn ? rows : K);
  dims[1] = (cuuint64_t)(mn ? K : rows);
  dims[2] = (cuuint64_t)(op.s0 ? Z0 : 1);
  dims[3] = (cuuint64_t)(op.s1 ? Z1 : 1);
  const cuuint64_t es = tf32 ? 4 : 2;
  const cuuint64_t row_bytes = (cuuint64_t)op.ld * es;
  const cuuint64_t plane = ((row_bytes * dims[1]) + 15) & ~(cuuint64_t)15;
  strides[0] = row_bytes;
  strides[1] = op.s0 ? (cuuint64_t)op.s0 * es : plane;
  strides[2] = op.s1 ? (cuuint64_t)op.s1 * es : plane * dims[2];
  box[0] = tf32 ? 32 : 64;
  box[1] = (cuuint32_t)(mn ? (tf32 ? 32 : 64) : box_rows);   // MN-major: one k-block of rows
  box[2] = 1;
  box[3] = 1;
  // MN-major tf32 operands: the 128-byte swizzle on 32-byte chunks, their only UMMA layout
  const CUtensorMapSwizzle sw =
      (tf32 && mn) ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = fn(map, tf32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                  4, const_cast<void*>(op.ptr), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Map of a bf16 [rows, cols] output with two batch strides; box {64, 32} with 128-byte
// swizzle, or (half) {32, 32} with 64-byte swizzle; or (f32) of an fp32 output, box
// {32, 32} with 128-byte swizzle.
bool make_out_map(CUtensorMap* map, void* ptr, int cols, int rows, long long ld, long long s0,
                  long long s1, int Z0, int Z1, bool half = false, bool f32 = false) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)(s0 ? Z0 : 1),
                        (cuuint64_t)(s1 ? Z1 : 1)};
  const cuuint64_t es = f32 ? 4 : 2;
  const cuuint64_t row_bytes = (cuuint64_t)ld * es;
  const cuuint64_t plane = ((row_bytes * dims[1]) + 15) & ~(cuuint64_t)15;
  cuuint64_t strides[3] = {row_bytes, s0 ? (cuuint64_t)s0 * es : plane,
                           s1 ? (cuuint64_t)s1 * es : plane * dims[2]};
  // one epilogue warp's 32 rows x 64 (or 32) columns
  cuuint32_t box[4] = {(half || f32) ? 32u : 64u, 32, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
            ptr, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            half ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, bool A_MN, bool B_MN, int STAGES, int MODE, typename TC, bool BRES,
          bool TF = false>
ttt_status launch_umma(const GemmProblem& p, const UArgs& a, cudaStream_t s) {
  CUtensorMap ma, mb;
  OutMaps om;
  if (!make_map(&ma, p.A, p.M, p.K, p.Z0, p.Z1, BM, TF) ||
      !make_map(&mb, p.B, p.N, p.K, p.Z0, p.Z1, BN, TF)) {
    set_error_message("gemm_umma: cuTensorMapEncodeTiled failed (M=%d N=%d K=%d)", p.M, p.N, p.K);
    return TTT_ERR_CUDA;
  }
  memset(&om, 0, sizeof(om));
  if (MODE == EPI_STORE_TMA && !make_out_map(&om.m[0], a.C, p.N, p.M, a.ldc, a.cs0, a.cs1, p.Z0,
                                             p.Z1, false, sizeof(TC) == 4)) {
    set_error_message("gemm_umma: output tensor map encoding failed");
    return TTT_ERR_CUDA;
  }
  if (MODE == EPI_SWIGLU) {
    // out2 / out3 share gemm.C's strides except for their own row stride and base
    // the gradient epilogue stores 32-column halves
    const bool h = a.grad != 0;
    if (!make_out_map(&om.m[0], a.C, a.n_valid, p.M, a.ldc, a.cs0, a.cs1, p.Z0, p.Z1, h) ||
        (a.C2 &&
         !make_out_map(&om.m[1], a.C2, a.n_valid, p.M, a.ld2, a.c2s0, a.c2s1, p.Z0, p.Z1, h)) ||
        (a.C3 &&
         !make_out_map(&om.m[2], a.C3, a.n_valid, p.M, a.ldc, a.cs0, a.cs1, p.Z0, p.Z1, h))) {
      set_error_message("gemm_umma: output tensor map encoding failed");
      return TTT_ERR_CUDA;
    }
  }
  auto kern = umma_gemm_kernel<BN, A_MN, B_MN, STAGES, MODE, TC, BRES, TF>;
  constexpr int SMEM = Smem<BN, STAGES, BRES, MODE>::TOTAL;
  static_assert(SMEM <= 232448, "shared memory budget");
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) !=
      cudaSuccess) {
    set_error_message("gemm_umma: cannot set %d bytes of dynamic shared memory", SMEM);
    return TTT_ERR_CUDA;
  }
  const long long tiles_n = (p.N + BN - 1) / BN;
  const long long tiles = tiles_n * ((p.M + BM - 1) / BM) * p.Z0 * p.Z1;
  const int per_sm = (SMEM <= 110 * 1024) ? 2 : 1;
  long long grid = (long long)sm_count() * per_sm;
  if (BRES) grid = (grid / tiles_n) * tiles_n;  // whole groups of n-tile CTAs
  if (tiles < grid) grid = tiles;
  if (grid < 1) grid = 1;
  kern<<<(unsigned)grid, THREADS, SMEM, s>>>(ma, mb, om, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error_message("gemm_umma launch: %s", cudaGetErrorString(e));
    return TTT_ERR_CUDA;
  }
  return TTT_OK;
}

// B-resident pays when K fits the resident buffer, the B operand is K-major, and each
// resident B tile serves many row tiles: a CTA reloads B (128 KB, after its MMAs on the old
// one drain) whenever the batch entry changes, so a B per batch entry with few row tiles
// per entry (the recurrent form's per-(batch, head) weights over one chunk) streams B
// through the ring with A instead.
bool use_bres(const GemmProblem& p, int BN) {
  const long long rows_per_b = (long long)((p.M + BM - 1) / BM) * (p.B.s0 ? 1 : p.Z0) *
                               (p.B.s1 ? 1 : p.Z1);
  return BN == 256 && p.K <= 4 * BK && !p.B.mn_major && (p.N + BN - 1) / BN <= sm_count() &&
         rows_per_b >= 64;
}

template <int BN, int STAGES, int MODE, typename TC>
ttt_status dispatch_major(const GemmProblem& p, const UArgs& a, cudaStream_t s) {
  constexpr int RES_STAGES = MODE == EPI_STORE ? 6 : 4;
  if (BN == 256 && use_bres(p, BN)) {
    if (p.A.mn_major) return launch_umma<BN, true, false, RES_STAGES, MODE, TC, true>(p, a, s);
    return launch_umma<BN, false, false, RES_STAGES, MODE, TC, true>(p, a, s);
  }
  const int key = (p.A.mn_major ? 2 : 0) | (p.B.mn_major ? 1 : 0);
  switch (key) {
    case 0: return launch_umma<BN, false, false, STAGES, MODE, TC, false>(p, a, s);
    case 1: return launch_umma<BN, false, true, STAGES, MODE, TC, false>(p, a, s);
    case 2: return launch_umma<BN, true, false, STAGES, MODE, TC, false>(p, a, s);
    default: return launch_umma<BN, true, true, STAGES, MODE, TC, false>(p, a, s);
  }
}

template <typename TC, int MODE>
ttt_status dispatch_bn_mode(const GemmProblem& p, const UArgs& a, cudaStream_t s) {
  if (p.N > 128) return dispatch_major<256, 4, MODE, TC>(p, a, s);
  if (p.N > 64) return dispatch_major<128, 3, MODE, TC>(p, a, s);
  return dispatch_major<64, 4, MODE, TC>(p, a, s);
}

template <typename TC>
ttt_status dispatch_bn(const GemmProblem& p, const UArgs& a, cudaStream_t s) {
  {
    // C without an addend (and without a copy) leaves through TMA stores, except where the
    // resident B tile leaves no room for the staging boxes (256-column tiles: narrower
    // ones keep two CTAs per SM without the boxes)
    constexpr long long q = 16 / sizeof(TC);   // elements per 16 bytes
    const bool tma_ok = !a.Cin && !a.C16 && p.N > 128 &&
                        (reinterpret_cast<uintptr_t>(a.C) & 15) == 0 && a.ldc % q == 0 &&
                        a.cs0 % q == 0 && a.cs1 % q == 0 && !use_bres(p, 256);
    if (tma_ok) return dispatch_major<256, 4, EPI_STORE_TMA, TC>(p, a, s);
  }
  if constexpr (sizeof(TC) == 4) {
    // staged fp32 stores where the lanes wait for an addend, or where the output leaves L2
    // and HBM write efficiency decides (more than 64 MB)
    if (a.C16) return dispatch_bn_mode<TC, EPI_STORE_COPY>(p, a, s);
    if (a.Cin || (long long)p.M * p.N * p.Z0 * p.Z1 * 4 > (64LL << 20))
      return dispatch_bn_mode<TC, EPI_STORE_STG>(p, a, s);
  }
  return dispatch_bn_mode<TC, EPI_STORE>(p, a, s);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// tf32 operands: streamed operands of either major, fp32 C; TMA stores without an addend,
// the staged epilogue with an addend or a large output, else direct row stores.
template <int BN, int STAGES, int MODE>
ttt_status launch_tf32(const GemmProblem& p, const UArgs& a, cudaStream_t s) {
  switch ((p.A.mn_major ? 2 : 0) | (p.B.mn_major ? 1 : 0)) {
    case 0: return launch_umma<BN, false, false, STAGES, MODE, float, false, true>(p, a, s);
    case 1: return launch_umma<BN, false, true, STAGES, MODE, float, false, true>(p, a, s);
    case 2: return launch_umma<BN, true, false, STAGES, MODE, float, false, true>(p, a, s);
    default: return launch_umma<BN, true, true, STAGES, MODE, float, false, true>(p, a, s);
  }
}
template <int MODE>
ttt_status dispatch_tf32_mode(const GemmProblem& p, const UArgs& a, cudaStream_t s) {
  // 128-column tiles with four ring stages: these epilogues, not the MMAs, set the pace,
  // and the narrower tile halves each tile's epilogue and doubles the tile count (a fuller
  // last wave). Faster than 256 columns (three or four stages) and than five or six stages.
  if (p.N > 64) return launch_tf32<128, 4, MODE>(p, a, s);
  return launch_tf32<64, 4, MODE>(p, a, s);
}
ttt_status dispatch_tf32(const GemmProblem& p, const UArgs& a, cudaStream_t s) {
  if (!a.Cin && p.N > 128 && (reinterpret_cast<uintptr_t>(a.C) & 15) == 0 && a.ldc % 4 == 0 &&
      a.cs0 % 4 == 0 && a.cs1 % 4 == 0)
    return launch_tf32<256, 4, EPI_STORE_TMA>(p, a, s);
  if (a.Cin || (long long)p.M * p.N * p.Z0 * p.Z1 * 4 > (64LL << 20))
    return dispatch_tf32_mode<EPI_STORE_STG>(p, a, s);
  return dispatch_tf32_mode<EPI_STORE>(p, a, s);
}

UArgs base_args(const GemmProblem& p, unsigned* dev_err, unsigned long long wait_ns) {
  UArgs a{};
  a.M = p.M; a.N = p.N; a.K = p.K; a.Z0 = p.Z0; a.Z1 = p.Z1;
  a.a_b0 = p.A.s0 != 0; a.a_b1 = p.A.s1 != 0; a.b_b0 = p.B.s0 != 0; a.b_b1 = p.B.s1 != 0;
  a.C = p.C.ptr; a.ldc = p.C.ld; a.cs0 = p.C.s0; a.cs1 = p.C.s1;
  a.C16 = static_cast<__nv_bfloat16*>(p.C.copy16);
  a.Cin = p.beta != 0.0f ? p.Cin.ptr : nullptr;
  a.ldi = p.Cin.ld; a.is0 = p.Cin.s0; a.is1 = p.Cin.s1;
  a.alpha = p.alpha; a.beta = p.beta;
  a.zss = p.zss; a.zeps = p.zeps; a.zpa = p.zpa; a.zpb = p.zpb;
  a.err = dev_err;
  a.wait_ns = wait_ns;
  return a;
}

}  // namespace

const char* umma_unsupported_reason(const GemmProblem& p) {
  for (const GemmOperand* o : {&p.A, &p.B}) {
    if (o->dtype != DT_BF16) return "operands must be bf16";
    if (!o->ptr || !aligned16(o->ptr)) return "operand base must be 16-byte aligned";
    if (o->ld <= 0 || o->ld % 8 != 0) return "operand row stride must be a multiple of 8";
    if (o->s0 < 0 || o->s1 < 0 || o->s0 % 8 != 0 || o->s1 % 8 != 0)
      return "operand batch strides must be non-negative multiples of 8";
  }
  if (p.K <= 0 || p.M <= 0 || p.N <= 0) return "M, N and K must be positive";
  if ((long long)p.Z0 * p.Z1 * ((p.M + BM - 1) / BM) * ((p.N + 63) / 64) > (1LL << 31))
    return "too many output tiles";
  if (p.beta != 0.0f && !p.Cin.ptr) return "beta != 0 needs an addend";
  if (p.zss) return "per-entry scales are taken only with tf32 operands";
  if (p.C.copy16 && (p.C.dtype != DT_F32 || !aligned16(p.C.copy16) || !aligned16(p.C.ptr) ||
                     p.C.ld % 4 != 0 || p.C.s0 % 4 != 0 || p.C.s1 % 4 != 0))
    return "a bf16 copy needs an fp32 result with 16-byte aligned bases, strides multiples of 4";
  if (encode_fn() == nullptr) return "cuTensorMapEncodeTiled is unavailable";
  return nullptr;
}

const char* umma_tf32_unsupported_reason(const GemmProblem& p) {
  for (const GemmOperand* o : {&p.A, &p.B}) {
    if (o->dtype != DT_F32) return "tf32 operands must be fp32";
    if (!o->ptr || !aligned16(o->ptr)) return "operand base must be 16-byte aligned";
    if (o->ld <= 0 || o->ld % 4 != 0) return "operand row stride must be a multiple of 4";
    if (o->s0 < 0 || o->s1 < 0 || o->s0 % 4 != 0 || o->s1 % 4 != 0)
      return "operand batch strides must be non-negative multiples of 4";
  }
  if (p.K <= 0 || p.M <= 0 || p.N <= 0) return "M, N and K must be positive";
  if ((long long)p.Z0 * p.Z1 * ((p.M + BM - 1) / BM) * ((p.N + 63) / 64) > (1LL << 31))
    return "too many output tiles";
  if (p.C.dtype != DT_F32) return "tf32 products write fp32";
  if (p.beta != 0.0f && !p.Cin.ptr) return "beta != 0 needs an addend";
  if (p.C.copy16) return "no bf16 copy with tf32 operands";
  if (encode_fn() == nullptr) return "cuTensorMapEncodeTiled is unavailable";
  return nullptr;
}

bool umma_supported(const GemmProblem& p) { return umma_unsupported_reason(p) == nullptr; }

ttt_status gemm_umma(const GemmProblem& p, cudaStream_t stream, unsigned* dev_err,
                     unsigned long long wait_ns) {
  if (p.M <= 0 || p.N <= 0 || p.Z0 <= 0 || p.Z1 <= 0) return TTT_OK;
  if (!umma_supported(p)) {
    set_error_message("gemm_umma: unsupported operand layout");
    return TTT_ERR_UNSUPPORTED;
  }
  const UArgs a = base_args(p, dev_err, wait_ns);
  if (p.C.dtype == DT_BF16) return dispatch_bn<__nv_bfloat16>(p, a, stream);
  return dispatch_bn<float>(p, a, stream);
}

ttt_status gemm_umma_tf32(const GemmProblem& p, cudaStream_t stream, unsigned* dev_err,
                          unsigned long long wait_ns) {
  if (p.M <= 0 || p.N <= 0 || p.Z0 <= 0 || p.Z1 <= 0) return TTT_OK;
  if (const char* why = umma_tf32_unsupported_reason(p)) {
    set_error_message("gemm_umma_tf32: %s", why);
    return TTT_ERR_UNSUPPORTED;
  }
  return dispatch_tf32(p, base_args(p, dev_err, wait_ns), stream);
}

const char* umma_swiglu_unsupported_reason(const SwigluGemm& g) {
  const GemmProblem& p = g.gemm;
  auto strides_ok = [](long long ld, long long s0, long long s1) {
    return ld % 8 == 0 && s0 % 8 == 0 && s1 % 8 == 0 && s0 >= 0 && s1 >= 0;
  };
  if (const char* r = umma_unsupported_reason(p)) return r;
  if (p.C.dtype != DT_BF16) return "SwiGLU output must be bf16";
  if (p.N % 256 != 0) return "SwiGLU GEMM width must be a multiple of 256";
  if (p.beta != 0.0f) return "SwiGLU GEMM takes no addend";
  if (!aligned16(p.C.ptr) || !strides_ok(p.C.ld, p.C.s0, p.C.s1))
    return "SwiGLU output must be 16-byte aligned with strides a multiple of 8";
  if (g.out2 && (!aligned16(g.out2) || !strides_ok(g.ld2, g.s20, g.s21)))
    return "second SwiGLU output must be 16-byte aligned with strides a multiple of 8";
  if (g.grad) {
    if (!g.rowscale || !g.dv || !aligned16(g.dv) || !strides_ok(g.ldd, g.ds0, g.ds1))
      return "gradient epilogue needs the row scale and an aligned dv";
    if (g.out3 && (!aligned16(g.out3) || g.ld3 != p.C.ld || g.s30 != p.C.s0 || g.s31 != p.C.s1))
      return "gradient epilogue: third output must share the first output's strides";
    if (g.out2 && (g.ld2 != p.C.ld || g.s20 != p.C.s0 || g.s21 != p.C.s1))
      return "gradient epilogue: second output must share the first output's strides";
  }
  return nullptr;
}

bool umma_swiglu_supported(const SwigluGemm& g) {
  return umma_swiglu_unsupported_reason(g) == nullptr;
}

ttt_status gemm_umma_swiglu(const SwigluGemm& g, cudaStream_t stream, unsigned* dev_err,
                            unsigned long long wait_ns) {
  const GemmProblem& p = g.gemm;
  if (p.M <= 0 || p.N <= 0 || p.Z0 <= 0 || p.Z1 <= 0) return TTT_OK;
  if (!umma_swiglu_supported(g)) {
    set_error_message("gemm_umma_swiglu: unsupported problem");
    return TTT_ERR_UNSUPPORTED;
  }
  UArgs a = base_args(p, dev_err, wait_ns);
  a.C2 = g.out2; a.ld2 = g.ld2; a.c2s0 = g.s20; a.c2s1 = g.s21;
  a.rs = g.rowscale; a.rs0 = g.rs0; a.rs1 = g.rs1;
  a.n_valid = g.n_valid;
  a.grad = g.grad;
  a.skip_out1 = g.grad ? g.skip_out1 : 0;
  a.C3 = g.grad ? g.out3 : nullptr;
  a.dv = static_cast<const __nv_bfloat16*>(g.dv);
  a.ldd = g.ldd; a.ds0 = g.ds0; a.ds1 = g.ds1;
  if (!g.grad) a.dv = nullptr;
  return dispatch_major<256, 4, EPI_SWIGLU, __nv_bfloat16>(p, a, stream);
}

}  // namespace ttt
