// Query side of the parallel form in one kernel: for a tile of 128 query rows of one
// (batch, head) inside one chunk,
//     phi_j = silu(Q W0[:, j]) * (Q W2[:, j])      for each 128-column block j of phi,
//     O    += phi_j S_c[j, :]                       (S_c: the state read by the chunk)
// ("Test-Time Training with KV Binding Is Secretly Linear Attention", 方法步骤详情: the
// outputs of the parallel form are phi(Q_c) S_c). phi never leaves the SM: each block is
// computed into TMEM by one 128 x 256 MMA against the blocked [W0/2 ; W2] operand, turned
// into bf16 phi by the epilogue warps straight into shared memory, and consumed there by
// the next MMA as the A operand of phi_j S_c[j]. The output accumulates in TMEM and is
// written once per tile: each epilogue warp converts its 32 rows to bf16 in its own 4 KB box
// of the phi tile (free once the tile's last MMA completed) and writes them with TMA tensor
// stores, 64 columns at a time, so the rows leave as whole lines.
//
// Warp roles (320 threads): warp 0 one lane issues TMA loads (Q tile; then, in the order
// the MMAs consume them, 64-deep k-blocks of the weights and of S_c through a 3-stage ring);
// warp 1 allocates TMEM and one lane issues the MMAs; warps 2-9 are the epilogue (warp w
// reads TMEM lanes 32 (w % 4) .. +31; warps 2-5 / 6-9 take the first / second half of the
// columns). TMEM: [0, 256) the A/2 | B pre-activations of one phi block, [256, 256 + h) O.
// Shared memory (bf16, 128-byte swizzle): Q 128 x h, ring 4 x 32 KB, phi 128 x 128.
//
// Every mbarrier wait is bounded; a timeout records DEVERR_TIMEOUT and raises the CTA's
// abort flag; the CTA then waits (bounded) for its loads and MMAs in flight and frees TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "gemm.h"
#include "ops.h"
#include "swiglu_epi.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

using namespace umma;

constexpr int FA_THREADS = 320;
// Every tile streams all of the weights and its chunk's state through the ring (768 KB at
// h = 256, m = 512), so the ring is as deep as shared memory allows: the copies in flight
// per SM, divided by the L2 latency, bound the kernel. One phi buffer leaves room for four
// stages.
constexpr int FA_RING = 4;
constexpr int FA_NP = 1;              // phi buffers
constexpr int FA_STAGE = 32768;       // one ring stage
constexpr int FA_PBLK = 16384;        // one 64-column k-block of a 128-row phi tile

template <int HD>
struct FaSmem {
  static constexpr int Q_OFF = 0;
  static constexpr int Q_BYTES = 128 * HD * 2;
  static constexpr int RING_OFF = Q_OFF + Q_BYTES;
  static constexpr int P_OFF = RING_OFF + FA_RING * FA_STAGE;
  static constexpr int BAR_OFF = P_OFF + FA_NP * 2 * FA_PBLK;
  static constexpr int TOTAL = BAR_OFF + 256 + 1024;
};

struct FaArgs {
  int BH, H, N, m, mblocks, chunk, C, tiles_per_bh, tiles;
  __nv_bfloat16* out;
  unsigned* err;
  unsigned long long wait_ns;
};

// 64 fp32 values of this lane's row as bf16 into row `lane` of a 128-byte-swizzled
// 32 x 64 staging box (the layout of a TMA box {64, 32} with 128-byte swizzle).
__device__ __forceinline__ void stage_row_bf16(const uint32_t* r, uint32_t box, int lane) {
#pragma unroll
  for (int cc = 0; cc < 8; ++cc) {
    const uint32_t addr = box + lane * 128 + ((cc ^ (lane & 7)) << 4);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                 "r"(pack_bf16x2(__uint_as_float(r[8 * cc]), __uint_as_float(r[8 * cc + 1]))),
                 "r"(pack_bf16x2(__uint_as_float(r[8 * cc + 2]), __uint_as_float(r[8 * cc + 3]))),
                 "r"(pack_bf16x2(__uint_as_float(r[8 * cc + 4]), __uint_as_float(r[8 * cc + 5]))),
                 "r"(pack_bf16x2(__uint_as_float(r[8 * cc + 6]), __uint_as_float(r[8 * cc + 7])))
                 : "memory");
  }
}

template <int HD>
__global__ void __launch_bounds__(FA_THREADS, 1)
    apply_fused_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmS,
                       const __grid_constant__ CUtensorMap tmO, const FaArgs a) {
  using L = FaSmem<HD>;
  constexpr int QKB = HD / 64;          // k-blocks of the Q tile
  constexpr int S_STAGE = 64 * HD * 2;  // bytes of one S_c k-block (64 state rows x h)
  extern __shared__ uint8_t fa_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(fa_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* full = bars;                // [FA_RING]
  uint64_t* empty = full + FA_RING;     // [FA_RING]
  uint64_t* q_full = empty + FA_RING;
  uint64_t* q_empty = q_full + 1;
  uint64_t* ab_full = q_empty + 1;
  uint64_t* ab_empty = ab_full + 1;
  uint64_t* p_full = ab_empty + 1;      // [2]
  uint64_t* p_empty = p_full + 2;       // [2]
  uint64_t* o_full = p_empty + 2;
  uint64_t* o_empty = o_full + 1;
  uint64_t* drain = o_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sb = smem_u32(smem);
  const uint32_t sQ = sb + L::Q_OFF, sR = sb + L::RING_OFF, sP = sb + L::P_OFF;
  const int count = (int)blockIdx.x < a.tiles ? (a.tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int MB = a.mblocks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < FA_RING; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(q_full), 1);
    mbar_init(smem_u32(q_empty), 1);
    mbar_init(smem_u32(ab_full), 1);
    mbar_init(smem_u32(ab_empty), 256);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&p_full[b]), 256);
      mbar_init(smem_u32(&p_empty[b]), 1);
    }
    mbar_init(smem_u32(o_full), 1);
    mbar_init(smem_u32(o_empty), 256);
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmS);
    tma_prefetch_desc(&tmO);
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
  int q_loads = 0;        // producer: Q tiles loaded
  bool mma_any = false;   // MMA lane: issued anything
  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      // next ring slot, once the MMAs have released it
      auto slot = [&](uint32_t& s_out) -> bool {
        const uint32_t s = it % FA_RING;
        if (it >= FA_RING && !mbar_wait(smem_u32(&empty[s]), ((it / FA_RING) & 1) ^ 1,
                                        abort_flag, a.err, a.wait_ns))
          return false;
        s_out = s;
        return true;
      };
      for (int i = 0; i < count && ok; ++i) {
        const int t = (int)blockIdx.x + i * (int)gridDim.x;
        const int bh = t / a.tiles_per_bh, row0 = (t - bh * a.tiles_per_bh) * 128;
        const int head = bh % a.H, zc = bh * a.C + row0 / a.chunk;
        if (q_loads > 0 && !mbar_wait(smem_u32(q_empty), (q_loads - 1) & 1, abort_flag, a.err,
                                      a.wait_ns)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(smem_u32(q_full), L::Q_BYTES);
#pragma unroll
        for (int kb = 0; kb < QKB; ++kb)
          tma_load_4d(sQ + kb * 16384, &tmQ, smem_u32(q_full), kb * 64, row0, bh, 0);
        ++q_loads;
        auto push_s = [&](int jb) -> bool {
          for (int kb = 0; kb < 2; ++kb) {
            uint32_t s;
            if (!slot(s)) return false;
            const uint32_t fb = smem_u32(&full[s]), dst = sR + s * FA_STAGE;
            mbar_arrive_expect_tx(fb, S_STAGE);
#pragma unroll
            for (int q = 0; q < QKB; ++q)
              tma_load_4d(dst + q * 8192, &tmS, fb, q * 64, jb * 128 + kb * 64, zc, 0);
            issued = ++it;
          }
          return true;
        };
        for (int j = 0; j < MB && ok; ++j) {
          for (int kb = 0; kb < QKB; ++kb) {
            uint32_t s;
            if (!slot(s)) {
              ok = false;
              break;
            }
            const uint32_t fb = smem_u32(&full[s]);
            mbar_arrive_expect_tx(fb, FA_STAGE);
            tma_load_4d(sR + s * FA_STAGE, &tmW, fb, kb * 64, j * 256, head, 0);
            issued = ++it;
          }
          if (ok && j > 0) ok = push_s(j - 1);
        }
        if (ok) ok = push_s(MB - 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t ID_AB = make_idesc_bf16(128, 256, false, false);
      constexpr uint32_t ID_O = make_idesc_bf16(128, HD, false, true);
      uint32_t it = 0;
      int ab_n = 0, o_n = 0, p_n[2] = {0, 0};
      bool ok = true;
      auto wait_stage = [&]() -> int {
        const int s = (int)(it % FA_RING);
        if (!mbar_wait(smem_u32(&full[s]), (it / FA_RING) & 1, abort_flag, a.err, a.wait_ns))
          return -1;
        tc_fence_after();
        return s;
      };
      // O += phi_jb S_c[jb]: A = phi tile (K-major), B = S_c rows (MN-major)
      auto o_step = [&](int jb) -> bool {
        const int b = FA_NP == 1 ? 0 : (jb & 1);
        if (!mbar_wait(smem_u32(&p_full[b]), p_n[b] & 1, abort_flag, a.err, a.wait_ns))
          return false;
        ++p_n[b];
        if (jb == 0 && o_n > 0 &&
            !mbar_wait(smem_u32(o_empty), (o_n - 1) & 1, abort_flag, a.err, a.wait_ns))
          return false;
        tc_fence_after();
        for (int kb = 0; kb < 2; ++kb, ++it) {
          const int s = wait_stage();
          if (s < 0) return false;
          const uint32_t pa = sP + b * 2 * FA_PBLK + kb * FA_PBLK, sbs = sR + s * FA_STAGE;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem + 256, make_sw128_desc(pa + kk * 32, 16, 1024),
                    make_sw128_desc(sbs + kk * 2048, 8192, 1024), ID_O,
                    (jb > 0 || kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(smem_u32(&empty[s]));
          mma_any = true;
        }
        mma_commit(smem_u32(&p_empty[b]));
        return true;
      };
      for (int i = 0; i < count && ok; ++i) {
        if (!mbar_wait(smem_u32(q_full), i & 1, abort_flag, a.err, a.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int j = 0; j < MB && ok; ++j) {
          if (ab_n > 0 &&
              !mbar_wait(smem_u32(ab_empty), (ab_n - 1) & 1, abort_flag, a.err, a.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int kb = 0; kb < QKB; ++kb, ++it) {
            const int s = wait_stage();
            if (s < 0) {
              ok = false;
              break;
            }
            const uint32_t qa = sQ + kb * 16384, wb = sR + s * FA_STAGE;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16(tmem, make_sw128_desc(qa + kk * 32, 16, 1024),
                      make_sw128_desc(wb + kk * 32, 16, 1024), ID_AB, (kb > 0 || kk > 0) ? 1u : 0u);
            mma_commit(smem_u32(&empty[s]));
            mma_any = true;
          }
          if (!ok) break;
          mma_commit(smem_u32(ab_full));
          ++ab_n;
          if (j == MB - 1) mma_commit(smem_u32(q_empty));
          if (j > 0) ok = o_step(j - 1);
        }
        if (ok) ok = o_step(MB - 1);
        if (ok) {
          mma_commit(smem_u32(o_full));
          ++o_n;
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
    int ab_n = 0, o_n = 0, p_n[2] = {0, 0};
    for (int i = 0; i < count; ++i) {
      const int t = (int)blockIdx.x + i * (int)gridDim.x;
      const int bh = t / a.tiles_per_bh, row0 = (t - bh * a.tiles_per_bh) * 128;
      bool ok = true;
      for (int j = 0; j < MB && ok; ++j) {
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
        const int b = FA_NP == 1 ? 0 : (j & 1);
        if (p_n[b] > 0 &&
            !mbar_wait(smem_u32(&p_empty[b]), (p_n[b] - 1) & 1, abort_flag, a.err, a.wait_ns)) {
          ok = false;
          break;
        }
        ++p_n[b];
        const uint32_t box = sP + b * 2 * FA_PBLK + part * FA_PBLK + quarter * 4096;
        // the previous tile's output stores from this box have read it
        if (j == 0) {
          if (lane == 0) tma_store_wait_read();
          __syncwarp();
        }
        swiglu_piece(ra0, rb0, 1.0f, box, lane, 0);
        swiglu_piece(ra1, rb1, 1.0f, box, lane, 4);
        fence_async_smem();
        mbar_arrive(smem_u32(&p_full[b]));
      }
      if (!ok) break;
      if (!mbar_wait(smem_u32(o_full), o_n & 1, abort_flag, a.err, a.wait_ns)) break;
      ++o_n;
      tc_fence_after();
      // O rows quarter*32 + lane, columns part*HD/2 .. +HD/2
      constexpr int HALF = HD / 2;
      uint32_t r[HALF];
#pragma unroll
      for (int c0 = 0; c0 < HALF; c0 += 32)
        tmem_ld32(lane_addr + 256u + (uint32_t)(part * HALF + c0),
                  *reinterpret_cast<uint32_t(*)[32]>(&r[c0]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(o_empty));
      // rows quarter*32 .. +31 through this warp's phi box (the tile's MMAs have all
      // completed): 64 columns per TMA store; rows past N are clipped by the store
      const uint32_t box = sP + part * FA_PBLK + quarter * 4096;
#pragma unroll
      for (int c0 = 0; c0 < HALF; c0 += 64) {
        if (c0 > 0) {
          if (lane == 0) tma_store_wait_read();
          __syncwarp();
        }
        stage_row_bf16(&r[c0], box, lane);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_4d(&tmO, box, part * HALF + c0, row0 + quarter * 32, bh, 0);
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
    const uint32_t lo = issued > (uint32_t)FA_RING ? issued - FA_RING : 0;
    for (uint32_t it = lo; it < issued; ++it)
      mbar_wait(smem_u32(&full[it % FA_RING]), (it / FA_RING) & 1, abort_flag, nullptr,
                a.wait_ns, true);
    if (q_loads > 0)
      mbar_wait(smem_u32(q_full), (q_loads - 1) & 1, abort_flag, nullptr, a.wait_ns, true);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 fa_encode() {
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
bool fa_map(CUtensorMap* map, const void* ptr, long long inner, long long rows, long long z,
            int box_rows) {
  auto fn = fa_encode();
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

int fa_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

template <int HD>
ttt_status launch_fa(const void* q, const void* Wk, const void* Sc, void* out, int B, int H,
                     int N, int m, int chunk, unsigned* err, unsigned long long wait_ns,
                     cudaStream_t s) {
  const long long BH = (long long)B * H, C = (N + chunk - 1) / chunk;
  const long long mpad = (m + 127LL) / 128 * 128;
  CUtensorMap mq, mw, ms, mo;
  if (!fa_map(&mq, q, HD, N, BH, 128) || !fa_map(&mw, Wk, HD, 2 * mpad, H, 256) ||
      !fa_map(&ms, Sc, HD, m, BH * C, 64) || !fa_map(&mo, out, HD, N, BH, 32)) {
    set_error_message("fused apply: cuTensorMapEncodeTiled failed");
    return TTT_ERR_CUDA;
  }
  FaArgs a;
  a.BH = (int)BH; a.H = H; a.N = N; a.m = m; a.mblocks = (int)(mpad / 128);
  a.chunk = chunk; a.C = (int)C;
  a.tiles_per_bh = (N + 127) / 128;
  a.tiles = (int)(BH * a.tiles_per_bh);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.err = err;
  a.wait_ns = wait_ns;
  auto kern = apply_fused_kernel<HD>;
  constexpr int SMEM = FaSmem<HD>::TOTAL;
  static_assert(SMEM <= 232448, "shared memory budget");
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) !=
      cudaSuccess) {
    set_error_message("fused apply: cannot set %d bytes of dynamic shared memory", SMEM);
    return TTT_ERR_CUDA;
  }
  int grid = fa_sm_count();
  if (a.tiles < grid) grid = a.tiles;
  if (grid < 1) return TTT_OK;
  kern<<<grid, FA_THREADS, SMEM, s>>>(mq, mw, ms, mo, a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error_message("fused apply launch: %s", cudaGetErrorString(e));
    return TTT_ERR_CUDA;
  }
  return TTT_OK;
}

bool al16p(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

bool fused_apply_supported(int dtype, int h, int m, int chunk, const void* q, const void* Wk,
                           const void* Sc, const void* out) {
  return dtype == DT_BF16 && (h == 128 || h == 256) && chunk % 128 == 0 && m >= 1 &&
         al16p(q) && al16p(Wk) && al16p(Sc) && al16p(out) && fa_encode() != nullptr;
}

ttt_status fused_apply(const void* q, const void* Wk, const void* Sc, void* out, int B, int H,
                       int N, int h, int m, int chunk, unsigned* err,
                       unsigned long long wait_ns, cudaStream_t s) {
  if ((long long)B * H == 0 || N == 0) return TTT_OK;
  if (h == 256) return launch_fa<256>(q, Wk, Sc, out, B, H, N, m, chunk, err, wait_ns, s);
  return launch_fa<128>(q, Wk, Sc, out, B, H, N, m, chunk, err, wait_ns, s);
}

}  // namespace ttt
