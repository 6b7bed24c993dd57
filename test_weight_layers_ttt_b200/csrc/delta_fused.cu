// Key side of the parallel form in one kernel: for one (batch, head), one chunk c and one
// 128-column block j of phi,
//     phi_j(K_c) = silu(K_c W0[:, j]) * (K_c W2[:, j]),
//     Delta S_c[j, :] = sign * phi_j(K_c)^T diag(eta_c) V_c
// ("Test-Time Training with KV Binding Is Secretly Linear Attention", 方法步骤详情: the state
// delta of a chunk is one contraction over the chunk's tokens, Theorem 5.2). phi(K) eta never
// leaves the SM: per 128-token tile of the chunk, one 128 x 256 MMA of the K tile against the
// resident blocked [W0/2 ; W2] weights of block j gives [A/2 | B] in TMEM; the epilogue warps
// turn it into bf16 sign * eta * phi straight into shared memory; a 128 x h MMA then adds
// (phi eta)_tile^T V_tile into the Delta S accumulator in TMEM (A operand phi eta read
// MN-major, B operand the V tile read MN-major). Delta S is written once per unit, fp32.
//
// Warp roles (320 threads): warp 0 one lane issues TMA loads (the block's weights, resident
// while the head stays the same; then per tile the K k-blocks, and the V stages of the
// previous tile, in the order the MMAs consume them, through a ring of 16 KB stages); warp 1
// allocates TMEM and one lane issues the MMAs; warps 2-9 are the epilogue (warp w reads TMEM
// lanes 32 (w % 4) .. +31; warps 2-5 / 6-9 take the first / second half of the columns).
// TMEM: [0, 256) the A/2 | B pre-activations of one tile, [256, 256 + h) Delta S.
// Shared memory (bf16, 128-byte swizzle): weights 256 x h, ring, phi eta 128 x 128.
// Units: CTA b works on phi block b % MB and a contiguous range of the (b, head, chunk)
// pairs, so the weights are reloaded only when the head changes and the MB CTAs of a group
// read the same K and V tiles at about the same time (L2 hits).
//
// Every mbarrier wait is bounded; a timeout records DEVERR_TIMEOUT and raises the CTA's
// abort flag; the CTA then waits (bounded) for its loads and MMAs in flight and frees TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "gemm.h"
#include "swiglu_epi.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

using namespace umma;

constexpr int DF_THREADS = 320;
constexpr int DF_STAGE = 16384;   // one ring stage: a K k-block (128 x 64) or a V stage
constexpr int DF_PBLK = 16384;    // one 64-column block of the 128-token phi eta tile
// At h = 256 (a 4-stage ring, too few bytes in flight to cover HBM latency) the first CTA
// of each group pulls the K and V tiles this many tiles ahead of its own into L2 with
// prefetch instructions. At h = 128 the 8-stage ring covers it and prefetching costs time.
constexpr int DF_PREFETCH = 2;

template <int HD>
struct DfSmem {
  static constexpr int RING = HD == 256 ? 4 : 8;
  static constexpr int VT = DF_STAGE / (2 * HD);   // tokens per V stage (32 or 64)
  static constexpr int W_OFF = 0;
  static constexpr int W_BYTES = 256 * HD * 2;     // HD / 64 k-blocks of 256 x 64
  static constexpr int RING_OFF = W_OFF + W_BYTES;
  static constexpr int P_OFF = RING_OFF + RING * DF_STAGE;
  static constexpr int BAR_OFF = P_OFF + 2 * DF_PBLK;
  static constexpr int TOTAL = BAR_OFF + 256 + 1024;
};

struct DfArgs {
  int BH, H, N, m, mblocks, chunk, C, groups;
  float sign;
  const __nv_bfloat16* kp;   // K and V [BH, N, HD], for the L2 prefetch
  const __nv_bfloat16* vp;
  const float* eta;   // [BH, N]
  float* dS;          // [BH, C, m, HD] fp32
  unsigned* err;
  unsigned long long wait_ns;
};

// The (b, head, chunk) pairs of this CTA's group: [lo, hi) of BH * C.
struct DfWalk {
  int j, lo, count;
  __device__ DfWalk(const DfArgs& a) {
    j = (int)blockIdx.x % a.mblocks;
    const int g = (int)blockIdx.x / a.mblocks;
    const long long rows = (long long)a.BH * a.C;
    if (g >= a.groups) {
      lo = 0;
      count = 0;
    } else {
      lo = (int)(rows * g / a.groups);
      count = (int)(rows * (g + 1) / a.groups) - lo;
    }
  }
};

template <int HD>
__global__ void __launch_bounds__(DF_THREADS, 1)
    delta_fused_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmD, const DfArgs a) {
  using L = DfSmem<HD>;
  constexpr int RING = L::RING;
  constexpr int VT = L::VT;
  constexpr int KKB = HD / 64;          // K k-blocks per tile
  constexpr int VST = 128 / VT;         // V stages per tile
  extern __shared__ uint8_t df_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(df_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* full = bars;                // [RING]
  uint64_t* empty = full + RING;        // [RING]
  uint64_t* w_full = empty + RING;
  uint64_t* w_empty = w_full + 1;
  uint64_t* ab_full = w_empty + 1;
  uint64_t* ab_empty = ab_full + 1;
  uint64_t* p_full = ab_empty + 1;
  uint64_t* p_empty = p_full + 1;
  uint64_t* d_full = p_empty + 1;
  uint64_t* d_empty = d_full + 1;
  uint64_t* drain = d_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sb = smem_u32(smem);
  const uint32_t sW = sb + L::W_OFF, sR = sb + L::RING_OFF, sP = sb + L::P_OFF;
  const DfWalk walk(a);

  if (threadIdx.x == 0) {
    for (int s = 0; s < RING; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(w_full), 1);
    mbar_init(smem_u32(w_empty), 1);
    mbar_init(smem_u32(ab_full), 1);
    mbar_init(smem_u32(ab_empty), 256);
    mbar_init(smem_u32(p_full), 256);
    mbar_init(smem_u32(p_empty), 1);
    mbar_init(smem_u32(d_full), 1);
    mbar_init(smem_u32(d_empty), 256);
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmD);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  uint32_t issued = 0;    // producer: ring loads issued
  int w_loads = 0;        // producer: weight loads issued
  bool mma_any = false;   // MMA lane: issued anything
  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      int wkey = -1;
      auto slot = [&](uint32_t& s_out) -> bool {
        const uint32_t s = it % RING;
        if (it >= (uint32_t)RING && !mbar_wait(smem_u32(&empty[s]), ((it / RING) & 1) ^ 1,
                                               abort_flag, a.err, a.wait_ns))
          return false;
        s_out = s;
        return true;
      };
      for (int i = 0; i < walk.count && ok; ++i) {
        const int pair = walk.lo + i, bh = pair / a.C, c = pair - bh * a.C;
        const int head = bh % a.H, t0 = c * a.chunk;
        const int Lc = min(a.chunk, a.N - t0), T = (Lc + 127) / 128;
        if (head != wkey) {
          // reload the block's weights once the MMAs have stopped reading the old ones
          if (w_loads > 0 && !mbar_wait(smem_u32(w_empty), (w_loads - 1) & 1, abort_flag, a.err,
                                        a.wait_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(smem_u32(w_full), L::W_BYTES);
#pragma unroll
          for (int kb = 0; kb < KKB; ++kb)
            tma_load_4d(sW + kb * 32768, &tmW, smem_u32(w_full), kb * 64, walk.j * 256, head, 0);
          ++w_loads;
          wkey = head;
        }
        auto push_v = [&](int t) -> bool {
          for (int vs = 0; vs < VST; ++vs) {
            uint32_t s;
            if (!slot(s)) return false;
            const uint32_t fb = smem_u32(&full[s]), dst = sR + s * DF_STAGE;
            mbar_arrive_expect_tx(fb, DF_STAGE);
#pragma unroll
            for (int q = 0; q < KKB; ++q)
              tma_load_4d(dst + q * (128 * VT), &tmV, fb, q * 64, t0 + t * 128 + vs * VT, bh, 0);
            issued = ++it;
          }
          return true;
        };
        for (int t = 0; t < T && ok; ++t) {
          for (int kb = 0; kb < KKB; ++kb) {
            uint32_t s;
            if (!slot(s)) {
              ok = false;
              break;
            }
            const uint32_t fb = smem_u32(&full[s]);
            mbar_arrive_expect_tx(fb, DF_STAGE);
            tma_load_4d(sR + s * DF_STAGE, &tmK, fb, kb * 64, t0 + t * 128, bh, 0);
            issued = ++it;
          }
          if (ok && t > 0) ok = push_v(t - 1);
        }
        if (ok) ok = push_v(T - 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t ID_AB = make_idesc_bf16(128, 256, false, false);
      constexpr uint32_t ID_D = make_idesc_bf16(128, HD, true, true);
      uint32_t it = 0;
      int ab_n = 0, p_n = 0, d_n = 0, w_uses = 0, wkey = -1;
      bool ok = true;
      auto wait_stage = [&]() -> int {
        const int s = (int)(it % RING);
        if (!mbar_wait(smem_u32(&full[s]), (it / RING) & 1, abort_flag, a.err, a.wait_ns))
          return -1;
        tc_fence_after();
        return s;
      };
      // Delta S += (phi eta)_t^T V_t: A = the phi eta tile (MN-major: 64 phi columns per
      // 128-byte token row), B = the V stages (MN-major: 64 h columns per token row)
      auto d_step = [&](int t) -> bool {
        if (!mbar_wait(smem_u32(p_full), p_n & 1, abort_flag, a.err, a.wait_ns)) return false;
        ++p_n;
        if (t == 0 && d_n > 0 &&
            !mbar_wait(smem_u32(d_empty), (d_n - 1) & 1, abort_flag, a.err, a.wait_ns))
          return false;
        tc_fence_after();
        for (int vs = 0; vs < VST; ++vs, ++it) {
          const int s = wait_stage();
          if (s < 0) return false;
          const uint32_t sv = sR + s * DF_STAGE;
#pragma unroll
          for (int kk = 0; kk < VT / 16; ++kk)
            mma_f16(tmem + 256, make_sw128_desc(sP + (vs * (VT / 16) + kk) * 2048, DF_PBLK, 1024),
                    make_sw128_desc(sv + kk * 2048, 128 * VT, 1024), ID_D,
                    (t > 0 || vs > 0 || kk > 0) ? 1u : 0u);
          mma_commit(smem_u32(&empty[s]));
          mma_any = true;
        }
        mma_commit(smem_u32(p_empty));
        return true;
      };
      for (int i = 0; i < walk.count && ok; ++i) {
        const int pair = walk.lo + i, bh = pair / a.C, c = pair - bh * a.C;
        const int head = bh % a.H, t0 = c * a.chunk;
        const int Lc = min(a.chunk, a.N - t0), T = (Lc + 127) / 128;
        if (head != wkey) {
          if (w_uses > 0) mma_commit(smem_u32(w_empty));   // old weights free once MMAs finish
          if (!mbar_wait(smem_u32(w_full), w_uses & 1, abort_flag, a.err, a.wait_ns)) {
            ok = false;
            break;
          }
          ++w_uses;
          wkey = head;
        }
        for (int t = 0; t < T && ok; ++t) {
          if (ab_n > 0 &&
              !mbar_wait(smem_u32(ab_empty), (ab_n - 1) & 1, abort_flag, a.err, a.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int kb = 0; kb < KKB; ++kb, ++it) {
            const int s = wait_stage();
            if (s < 0) {
              ok = false;
              break;
            }
            const uint32_t ka = sR + s * DF_STAGE, wb = sW + kb * 32768;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16(tmem, make_sw128_desc(ka + kk * 32, 16, 1024),
                      make_sw128_desc(wb + kk * 32, 16, 1024), ID_AB, (kb > 0 || kk > 0) ? 1u : 0u);
            mma_commit(smem_u32(&empty[s]));
            mma_any = true;
          }
          if (!ok) break;
          mma_commit(smem_u32(ab_full));
          ++ab_n;
          if (t > 0) ok = d_step(t - 1);
        }
        if (ok) ok = d_step(T - 1);
        if (ok) {
          mma_commit(smem_u32(d_full));
          ++d_n;
        }
      }
      // every MMA this lane issued has completed once `drain` flips
      if (mma_any) {
        mma_commit(smem_u32(drain));
        mbar_wait(smem_u32(drain), 0, abort_flag, nullptr, a.wait_ns, true);
      }
    }
  } else {
    const int ew = warp - 2, quarter = warp & 3, part = ew >> 2;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    int ab_n = 0, p_n = 0, d_n = 0;
    for (int i = 0; i < walk.count; ++i) {
      const int pair = walk.lo + i, bh = pair / a.C, c = pair - bh * a.C;
      const int t0 = c * a.chunk;
      const int Lc = min(a.chunk, a.N - t0), T = (Lc + 127) / 128;
      const float* eta_c = a.eta + (long long)bh * a.N + t0;
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        // this thread's token row of the tile; rows past the chunk contribute nothing
        const int row = t * 128 + quarter * 32 + lane;
        const float sc = row < Lc ? a.sign * eta_c[row] : 0.0f;
        if (HD == 256 && walk.j == 0) {
          // the tile DF_PREFETCH ahead: in this unit, else in the range's next unit
          int pt = t + DF_PREFETCH, pbh = bh, pt0 = t0, pL = Lc;
          bool have = pt < T;
          if (!have && i + 1 < walk.count) {
            const int np = pair + 1, nbh = np / a.C, nc = np - nbh * a.C;
            pt -= T;
            pbh = nbh;
            pt0 = nc * a.chunk;
            pL = min(a.chunk, a.N - pt0);
            have = pt * 128 < pL;
          }
          if (have) {
            // whole 128-byte lines of the tile's rows that exist: HD / 128 per thread and tensor
            const int rows_in = min(128, pL - pt * 128);
            const long long base = ((long long)pbh * a.N + pt0 + pt * 128) * HD;
            const int tid = threadIdx.x - 64;   // the 256 epilogue threads
#pragma unroll
            for (int q = 0; q < HD / 128; ++q) {
              const int line = tid + 256 * q;   // 64 bf16 = 128 bytes per line
              if (line / (HD / 64) < rows_in) {
                asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(a.kp + base + line * 64));
                asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(a.vp + base + line * 64));
              }
            }
          }
        }
        if (!mbar_wait(smem_u32(ab_full), ab_n & 1, abort_flag, a.err, a.wait_ns)) {
          ok = false;
          break;
        }
        ++ab_n;
        tc_fence_after();
        // phi columns part*64 .. +63 of block j: A/2 at part*64, B at 128 + part*64
        uint32_t ra0[32], rb0[32], ra1[32], rb1[32];
        const uint32_t ta = lane_addr + (uint32_t)(part * 64), tb = ta + 128u;
        tmem_ld32(ta, ra0);
        tmem_ld32(tb, rb0);
        tmem_ld32(ta + 32, ra1);
        tmem_ld32(tb + 32, rb1);
        tmem_ld_wait_regs(ra0, rb0);
        tmem_ld_wait_regs(ra1, rb1);
        tc_fence_before();
        mbar_arrive(smem_u32(ab_empty));
        if (p_n > 0 &&
            !mbar_wait(smem_u32(p_empty), (p_n - 1) & 1, abort_flag, a.err, a.wait_ns)) {
          ok = false;
          break;
        }
        ++p_n;
        const uint32_t box = sP + part * DF_PBLK + quarter * 4096;
        // the previous unit's Delta S stores from this box have read it
        if (t == 0) {
          if (lane == 0) tma_store_wait_read();
          __syncwarp();
        }
        swiglu_piece(ra0, rb0, sc, box, lane, 0);
        swiglu_piece(ra1, rb1, sc, box, lane, 4);
        fence_async_smem();
        mbar_arrive(smem_u32(p_full));
      }
      if (!ok) break;
      if (!mbar_wait(smem_u32(d_full), d_n & 1, abort_flag, a.err, a.wait_ns)) break;
      ++d_n;
      tc_fence_after();
      // Delta S rows (phi columns) j*128 + quarter*32 + lane, columns part*HD/2 .. +HD/2
      constexpr int HALF = HD / 2;
      uint32_t r[HALF];
#pragma unroll
      for (int c0 = 0; c0 < HALF; c0 += 32)
        tmem_ld32(lane_addr + 256u + (uint32_t)(part * HALF + c0),
                  *reinterpret_cast<uint32_t(*)[32]>(&r[c0]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(d_empty));
      // rows quarter*32 .. +31 through this warp's phi box (the unit's MMAs have all
      // completed), 32 fp32 columns per TMA store; rows past m are clipped by the store
      const uint32_t box = sP + part * DF_PBLK + quarter * 4096;
#pragma unroll
      for (int c0 = 0; c0 < HALF; c0 += 32) {
        if (c0 > 0) {
          if (lane == 0) tma_store_wait_read();
          __syncwarp();
        }
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          const uint32_t addr = box + lane * 128 + ((cc ^ (lane & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                       "r"(r[c0 + 4 * cc]), "r"(r[c0 + 4 * cc + 1]), "r"(r[c0 + 4 * cc + 2]),
                       "r"(r[c0 + 4 * cc + 3])
                       : "memory");
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_4d(&tmD, box, part * HALF + c0, walk.j * 128 + quarter * 32,
                       bh * a.C + c, 0);
          tma_store_commit();
        }
      }
    }
    if (lane == 0) tma_store_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && warp == 0 && lane == 0) {
    // loads still in flight land before the CTA's shared memory goes away
    const uint32_t lo = issued > (uint32_t)RING ? issued - RING : 0;
    for (uint32_t it = lo; it < issued; ++it)
      mbar_wait(smem_u32(&full[it % RING]), (it / RING) & 1, abort_flag, nullptr, a.wait_ns,
                true);
    if (w_loads > 0)
      mbar_wait(smem_u32(w_full), (w_loads - 1) & 1, abort_flag, nullptr, a.wait_ns, true);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 df_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool done = false;
  if (!done) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    done = true;
  }
  return fn;
}

// bf16 map over [z][rows][inner] (inner contiguous), box {64, box_rows}, 128-byte swizzle.
bool df_map(CUtensorMap* map, const void* ptr, long long inner, long long rows, long long z,
            int box_rows) {
  auto fn = df_encode();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)z, 1};
  cuuint64_t strides[3] = {(cuuint64_t)inner * 2, (cuuint64_t)(inner * rows * 2),
                           (cuuint64_t)(inner * rows * z * 2)};
  cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 map of Delta S [z][m][HD], box {32, 32}, 128-byte swizzle (one warp's 32 rows x 32
// columns per store).
bool df_map_out(CUtensorMap* map, float* ptr, long long inner, long long rows, long long z) {
  auto fn = df_encode();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)z, 1};
  cuuint64_t strides[3] = {(cuuint64_t)inner * 4, (cuuint64_t)(inner * rows * 4),
                           (cuuint64_t)(inner * rows * z * 4)};
  cuuint32_t box[4] = {32, 32, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ptr, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int df_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

template <int HD>
ttt_status launch_df(const void* k, const void* v, const float* eta, const void* Wk, float* dS,
                     int B, int H, int N, int m, int chunk, float sign, unsigned* err,
                     unsigned long long wait_ns, cudaStream_t s) {
  const long long BH = (long long)B * H, C = (N + chunk - 1) / chunk;
  const long long mpad = (m + 127LL) / 128 * 128;
  CUtensorMap mk, mw, mv, md;
  if (!df_map(&mk, k, HD, N, BH, 128) || !df_map(&mw, Wk, HD, 2 * mpad, H, 256) ||
      !df_map(&mv, v, HD, N, BH, DfSmem<HD>::VT) || !df_map_out(&md, dS, HD, m, BH * C)) {
    set_error_message("fused state delta: cuTensorMapEncodeTiled failed");
    return TTT_ERR_CUDA;
  }
  DfArgs a;
  a.BH = (int)BH; a.H = H; a.N = N; a.m = m; a.mblocks = (int)(mpad / 128);
  a.chunk = chunk; a.C = (int)C;
  a.sign = sign;
  a.eta = eta;
  a.dS = dS;
  a.kp = static_cast<const __nv_bfloat16*>(k);
  a.vp = static_cast<const __nv_bfloat16*>(v);
  a.err = err;
  a.wait_ns = wait_ns;
  // groups of mblocks CTAs (one per phi block) share the (b, head, chunk) pairs
  const long long pairs = BH * C;
  long long groups = df_sm_count() / a.mblocks;
  if (groups > pairs) groups = pairs;
  if (groups < 1) groups = 1;
  a.groups = (int)groups;
  const long long grid = groups * a.mblocks;
  auto kern = delta_fused_kernel<HD>;
  constexpr int SMEM = DfSmem<HD>::TOTAL;
  static_assert(SMEM <= 232448, "shared memory budget");
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) !=
      cudaSuccess) {
    set_error_message("fused state delta: cannot set %d bytes of dynamic shared memory", SMEM);
    return TTT_ERR_CUDA;
  }
  kern<<<(unsigned)grid, DF_THREADS, SMEM, s>>>(mk, mw, mv, md, a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error_message("fused state delta launch: %s", cudaGetErrorString(e));
    return TTT_ERR_CUDA;
  }
  return TTT_OK;
}

bool al16d(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

bool fused_delta_supported(int dtype, int h, int m, const void* k, const void* v,
                           const float* eta, const void* Wk, const float* dS) {
  return dtype == DT_BF16 && (h == 128 || h == 256) && m >= 1 && al16d(k) && al16d(v) &&
         eta && al16d(Wk) && al16d(dS) && df_encode() != nullptr;
}

ttt_status fused_delta(const void* k, const void* v, const float* eta, const void* Wk, float* dS,
                       int B, int H, int N, int h, int m, int chunk, int sign, unsigned* err,
                       unsigned long long wait_ns, cudaStream_t s) {
  if ((long long)B * H == 0 || N == 0) return TTT_OK;
  if (h == 256)
    return launch_df<256>(k, v, eta, Wk, dS, B, H, N, m, chunk, (float)sign, err, wait_ns, s);
  return launch_df<128>(k, v, eta, Wk, dS, B, H, N, m, chunk, (float)sign, err, wait_ns, s);
}

}  // namespace ttt
