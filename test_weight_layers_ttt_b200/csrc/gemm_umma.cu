// Tensor-core batched GEMM engine for sm_100a: bf16 operands staged in shared memory by
// TMA (128-byte swizzle, no multicast), tcgen05.mma kind::f16 with the fp32 accumulator
// in tensor memory, and a CUDA-core epilogue that reads TMEM with tcgen05.ld.
//
// One CTA computes one 128 x BN output tile. Warp roles (192 threads):
//   warp 0 (one lane)  TMA producer over a STAGES-deep shared-memory ring
//   warp 1             TMEM allocation; one lane issues the MMAs and the commits
//   warps 2..5         epilogue, warp w reads TMEM lanes 32*(w%4) .. 32*(w%4)+31
// Every mbarrier wait is bounded; a timeout records DEVERR_TIMEOUT in the device error
// word, raises a CTA-wide abort flag, and the CTA drains its in-flight copies and MMAs
// (again with bounded waits) and frees its TMEM before returning.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "gemm.h"
#include "umma.cuh"

namespace ttt {
namespace {

using namespace umma;

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int EPI_WARPS = 4;
constexpr int THREADS = 64 + 32 * EPI_WARPS;

struct UArgs {
  int M, N, K, Z0;
  int a_b0, a_b1, b_b0, b_b1;  // 1 = operand uses that batch coordinate
  void* C; long long ldc, cs0, cs1;
  const float* Cin; long long ldi, is0, is1;
  float alpha, beta;
  unsigned* err;
  unsigned long long wait_ns;
};

template <int BN, int STAGES>
struct Smem {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int BAR_OFF = STAGES * STAGE;
  static constexpr int TOTAL = BAR_OFF + 256 + 1024;  // + barriers + alignment slack
};

template <typename TC>
__device__ __forceinline__ void store_row32(TC* dst, const float* v, int n_valid, bool vec_ok);

template <>
__device__ __forceinline__ void store_row32<float>(float* dst, const float* v, int n_valid,
                                                   bool vec_ok) {
  if (vec_ok && n_valid == 32) {
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
  } else {
    for (int j = 0; j < n_valid; ++j) dst[j] = v[j];
  }
}

template <>
__device__ __forceinline__ void store_row32<__nv_bfloat16>(__nv_bfloat16* dst, const float* v,
                                                           int n_valid, bool vec_ok) {
  if (vec_ok && n_valid == 32) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      uint4 pk;
      __nv_bfloat162 t0 = __floats2bfloat162_rn(v[j], v[j + 1]);
      __nv_bfloat162 t1 = __floats2bfloat162_rn(v[j + 2], v[j + 3]);
      __nv_bfloat162 t2 = __floats2bfloat162_rn(v[j + 4], v[j + 5]);
      __nv_bfloat162 t3 = __floats2bfloat162_rn(v[j + 6], v[j + 7]);
      pk.x = *reinterpret_cast<uint32_t*>(&t0);
      pk.y = *reinterpret_cast<uint32_t*>(&t1);
      pk.z = *reinterpret_cast<uint32_t*>(&t2);
      pk.w = *reinterpret_cast<uint32_t*>(&t3);
      *reinterpret_cast<uint4*>(dst + j) = pk;
    }
  } else {
    for (int j = 0; j < n_valid; ++j) dst[j] = __float2bfloat16_rn(v[j]);
  }
}

template <int BN, bool A_MN, bool B_MN, int STAGES, typename TC>
__global__ void __launch_bounds__(THREADS, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB, const UArgs args) {
  using L = Smem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile_n = blockIdx.x, tile_m = blockIdx.y;
  const int z0 = blockIdx.z % args.Z0, z1 = blockIdx.z / args.Z0;
  const int KB = (args.K + BK - 1) / BK;
  const uint32_t smem_base = smem_u32(smem);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(tfull), 1);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int issued = 0;        // producer: k-blocks whose loads were issued
  bool mma_any = false;  // MMA lane: at least one MMA issued
  if (warp == 0) {
    if (lane == 0) {
      const int ac2 = args.a_b0 ? z0 : 0, ac3 = args.a_b1 ? z1 : 0;
      const int bc2 = args.b_b0 ? z0 : 0, bc3 = args.b_b1 ? z1 : 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES;
        if (kb >= STAGES &&
            !mbar_wait(smem_u32(&empty[s]), ((kb / STAGES) & 1) ^ 1, abort_flag, args.err,
                       args.wait_ns))
          break;
        const uint32_t fb = smem_u32(&full[s]);
        mbar_arrive_expect_tx(fb, L::STAGE);
        const uint32_t sA = smem_base + s * L::STAGE;
        const uint32_t sB = sA + L::A_BYTES;
        if (A_MN) {
          tma_load_4d(sA, &tmA, fb, tile_m * BM, kb * BK, ac2, ac3);
          tma_load_4d(sA + 8192, &tmA, fb, tile_m * BM + 64, kb * BK, ac2, ac3);
        } else {
          tma_load_4d(sA, &tmA, fb, kb * BK, tile_m * BM, ac2, ac3);
        }
        if (B_MN) {
#pragma unroll
          for (int t = 0; t < BN / 64; ++t)
            tma_load_4d(sB + t * 8192, &tmB, fb, tile_n * BN + 64 * t, kb * BK, bc2, bc3);
        } else {
          tma_load_4d(sB, &tmB, fb, kb * BK, tile_n * BN, bc2, bc3);
        }
        issued = kb + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = make_idesc_bf16(BM, BN, A_MN, B_MN);
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES;
        if (!mbar_wait(smem_u32(&full[s]), (kb / STAGES) & 1, abort_flag, args.err, args.wait_ns))
          break;
        tc_fence_after();
        const uint32_t sA = smem_base + s * L::STAGE;
        const uint32_t sB = sA + L::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = A_MN ? make_sw128_desc(sA + kk * 2048, 8192, 1024)
                                   : make_sw128_desc(sA + kk * 32, 16, 1024);
          const uint64_t bd = B_MN ? make_sw128_desc(sB + kk * 2048, 8192, 1024)
                                   : make_sw128_desc(sB + kk * 32, 16, 1024);
          mma_f16(tmem, ad, bd, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
        }
        mma_any = true;
        mma_commit(smem_u32(&empty[s]));
      }
      // Arrives once every MMA above is done (also on the abort path, so that the
      // teardown can wait for in-flight MMAs before freeing TMEM).
      mma_commit(smem_u32(tfull));
    }
  } else {
    // Epilogue: TMEM -> registers -> alpha * acc + beta * Cin -> global.
    const bool ok = mbar_wait(smem_u32(tfull), 0, abort_flag, args.err, args.wait_ns);
    tc_fence_after();
    const int quarter = warp & 3;
    const int row = tile_m * BM + quarter * 32 + lane;
    TC* crow = static_cast<TC*>(args.C) + z0 * args.cs0 + z1 * args.cs1 + (long long)row * args.ldc;
    const float* irow = args.Cin ? args.Cin + z0 * args.is0 + z1 * args.is1 +
                                       (long long)row * args.ldi
                                 : nullptr;
    const bool vec_ok =
        ((reinterpret_cast<uintptr_t>(crow) & 15) == 0) && ((args.ldc * sizeof(TC)) % 16 == 0);
    if (ok) {
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c0, r);
        tmem_ld_wait();
        const int col0 = tile_n * BN + c0;
        int nv = args.N - col0;
        nv = nv > 32 ? 32 : nv;
        if (row < args.M && nv > 0) {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = args.alpha * __uint_as_float(r[j]);
          if (irow) {
            for (int j = 0; j < nv; ++j) v[j] += args.beta * irow[col0 + j];
          }
          store_row32<TC>(crow + col0, v, nv, vec_ok);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // Drain: the producer waits for its loads still in flight; warp 1 for its MMAs.
    if (warp == 0 && lane == 0) {
      for (int kb = issued - STAGES < 0 ? 0 : issued - STAGES; kb < issued; ++kb)
        mbar_wait(smem_u32(&full[kb % STAGES]), (kb / STAGES) & 1, abort_flag, nullptr,
                  args.wait_ns, true);
    }
    if (warp == 1 && lane == 0 && mma_any)
      mbar_wait(smem_u32(tfull), 0, abort_flag, nullptr, args.wait_ns, true);
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
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

// 4-D map {inner, outer, z0, z1} over one operand; box {64, box_outer, 1, 1}.
bool make_map(CUtensorMap* map, const GemmOperand& op, int rows, int K, int Z0, int Z1,
              int box_rows) {
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
  const cuuint64_t row_bytes = (cuuint64_t)op.ld * 2;
  const cuuint64_t plane = ((row_bytes * dims[1]) + 15) & ~(cuuint64_t)15;
  strides[0] = row_bytes;
  strides[1] = op.s0 ? (cuuint64_t)op.s0 * 2 : plane;
  strides[2] = op.s1 ? (cuuint64_t)op.s1 * 2 : plane * dims[2];
  box[0] = 64;
  box[1] = (cuuint32_t)(mn ? 64 : box_rows);
  box[2] = 1;
  box[3] = 1;
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(op.ptr), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, bool A_MN, bool B_MN, int STAGES, typename TC>
ttt_status launch_umma(const GemmProblem& p, const UArgs& a, cudaStream_t s) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, p.A, p.M, p.K, p.Z0, p.Z1, BM) ||
      !make_map(&mb, p.B, p.N, p.K, p.Z0, p.Z1, BN)) {
    set_error_message("gemm_umma: cuTensorMapEncodeTiled failed (M=%d N=%d K=%d)", p.M, p.N, p.K);
    return TTT_ERR_CUDA;
  }
  auto kern = umma_gemm_kernel<BN, A_MN, B_MN, STAGES, TC>;
  constexpr int SMEM = Smem<BN, STAGES>::TOTAL;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) !=
      cudaSuccess) {
    set_error_message("gemm_umma: cannot set %d bytes of dynamic shared memory", SMEM);
    return TTT_ERR_CUDA;
  }
  dim3 grid((p.N + BN - 1) / BN, (p.M + BM - 1) / BM, p.Z0 * p.Z1);
  kern<<<grid, THREADS, SMEM, s>>>(ma, mb, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error_message("gemm_umma launch: %s", cudaGetErrorString(e));
    return TTT_ERR_CUDA;
  }
  return TTT_OK;
}

template <int BN, int STAGES, typename TC>
ttt_status dispatch_major(const GemmProblem& p, const UArgs& a, cudaStream_t s) {
  const int key = (p.A.mn_major ? 2 : 0) | (p.B.mn_major ? 1 : 0);
  switch (key) {
    case 0: return launch_umma<BN, false, false, STAGES, TC>(p, a, s);
    case 1: return launch_umma<BN, false, true, STAGES, TC>(p, a, s);
    case 2: return launch_umma<BN, true, false, STAGES, TC>(p, a, s);
    default: return launch_umma<BN, true, true, STAGES, TC>(p, a, s);
  }
}

template <typename TC>
ttt_status dispatch_bn(const GemmProblem& p, const UArgs& a, cudaStream_t s) {
  if (p.N > 128) return dispatch_major<256, 4, TC>(p, a, s);
  if (p.N > 64) return dispatch_major<128, 3, TC>(p, a, s);
  return dispatch_major<64, 4, TC>(p, a, s);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bool operand_ok(const GemmOperand& o) {
  return o.dtype == DT_BF16 && o.ptr && aligned16(o.ptr) && o.ld > 0 && (o.ld % 8) == 0 &&
         (o.s0 % 8) == 0 && (o.s1 % 8) == 0 && o.s0 >= 0 && o.s1 >= 0;
}

}  // namespace

bool umma_supported(const GemmProblem& p) {
  if (!operand_ok(p.A) || !operand_ok(p.B)) return false;
  if (p.K <= 0 || p.M <= 0 || p.N <= 0) return false;
  if ((long long)p.Z0 * p.Z1 > 65535 || (p.M + BM - 1) / BM > 65535) return false;
  if (p.beta != 0.0f && !p.Cin.ptr) return false;
  return encode_fn() != nullptr;
}

ttt_status gemm_umma(const GemmProblem& p, cudaStream_t stream, unsigned* dev_err,
                     unsigned long long wait_ns) {
  if (p.M <= 0 || p.N <= 0 || p.Z0 <= 0 || p.Z1 <= 0) return TTT_OK;
  if (!umma_supported(p)) {
    set_error_message("gemm_umma: unsupported operand layout");
    return TTT_ERR_UNSUPPORTED;
  }
  UArgs a;
  a.M = p.M; a.N = p.N; a.K = p.K; a.Z0 = p.Z0;
  a.a_b0 = p.A.s0 != 0; a.a_b1 = p.A.s1 != 0; a.b_b0 = p.B.s0 != 0; a.b_b1 = p.B.s1 != 0;
  a.C = p.C.ptr; a.ldc = p.C.ld; a.cs0 = p.C.s0; a.cs1 = p.C.s1;
  a.Cin = p.beta != 0.0f ? p.Cin.ptr : nullptr;
  a.ldi = p.Cin.ld; a.is0 = p.Cin.s0; a.is1 = p.Cin.s1;
  a.alpha = p.alpha; a.beta = p.beta;
  a.err = dev_err;
  a.wait_ns = wait_ns;
  if (p.C.dtype == DT_BF16) return dispatch_bn<__nv_bfloat16>(p, a, stream);
  return dispatch_bn<float>(p, a, stream);
}

}  // namespace ttt
