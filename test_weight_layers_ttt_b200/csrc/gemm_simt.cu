// CUDA-core batched GEMM engine: fp32 or bf16 operands with arbitrary strides, fp32
// accumulation. Used for every contraction in fp32 mode (where the fp64 parity bound of
// 1e-4 rules out reduced-precision tensor-core inputs) and for the small fp32
// Newton-Schulz products of the recurrent form.
#include <cstdio>

#include "gemm.h"

namespace ttt {
namespace {

constexpr int TM = 64, TN = 64, TK = 16, THREADS = 256;

struct SimtArgs {
  int M, N, K, Z0;
  const void* A; long long lda, as0, as1; int a_mn;
  const void* B; long long ldb, bs0, bs1; int b_mn;
  void* C; long long ldc, cs0, cs1;
  const float* Cin; long long ldi, is0, is1;
  float alpha, beta;
};

template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(THREADS) simt_gemm_kernel(const SimtArgs a) {
  __shared__ float As[TK][TM + 1];
  __shared__ float Bs[TK][TN + 1];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int i0 = blockIdx.y * TM, j0 = blockIdx.x * TN;
  const int z0 = blockIdx.z % a.Z0, z1 = blockIdx.z / a.Z0;
  const TA* A = static_cast<const TA*>(a.A) + z0 * a.as0 + z1 * a.as1;
  const TB* B = static_cast<const TB*>(a.B) + z0 * a.bs0 + z1 * a.bs1;

  float acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.0f;

  for (int k0 = 0; k0 < a.K; k0 += TK) {
    for (int e = tid; e < TM * TK; e += THREADS) {
      int ii, kk;
      if (a.a_mn) { ii = e % TM; kk = e / TM; } else { kk = e % TK; ii = e / TK; }
      const int gi = i0 + ii, gk = k0 + kk;
      float val = 0.0f;
      if (gi < a.M && gk < a.K)
        val = to_f32(A[a.a_mn ? (long long)gk * a.lda + gi : (long long)gi * a.lda + gk]);
      As[kk][ii] = val;
    }
    for (int e = tid; e < TN * TK; e += THREADS) {
      int jj, kk;
      if (a.b_mn) { jj = e % TN; kk = e / TN; } else { kk = e % TK; jj = e / TK; }
      const int gj = j0 + jj, gk = k0 + kk;
      float val = 0.0f;
      if (gj < a.N && gk < a.K)
        val = to_f32(B[a.b_mn ? (long long)gk * a.ldb + gj : (long long)gj * a.ldb + gk]);
      Bs[kk][jj] = val;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float af[4], bf[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) af[r] = As[kk][ty + 16 * r];
#pragma unroll
      for (int c = 0; c < 4; ++c) bf[c] = Bs[kk][tx + 16 * c];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(af[r], bf[c], acc[r][c]);
    }
    __syncthreads();
  }

  TC* C = static_cast<TC*>(a.C) + z0 * a.cs0 + z1 * a.cs1;
  const float* Ci = a.Cin ? a.Cin + z0 * a.is0 + z1 * a.is1 : nullptr;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int gi = i0 + ty + 16 * r;
    if (gi >= a.M) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int gj = j0 + tx + 16 * c;
      if (gj >= a.N) continue;
      float val = a.alpha * acc[r][c];
      if (Ci) val += a.beta * Ci[(long long)gi * a.ldi + gj];
      C[(long long)gi * a.ldc + gj] = from_f32<TC>(val);
    }
  }
}

template <typename TA, typename TB, typename TC>
void launch_simt(const SimtArgs& a, dim3 grid, cudaStream_t s) {
  simt_gemm_kernel<TA, TB, TC><<<grid, THREADS, 0, s>>>(a);
}

// SwiGLU-epilogue feature GEMM on CUDA cores. B holds 128-row blocks [W0^T ; W2^T]; output
// column j (< n_valid) pairs B rows blk*256 + w (A part) and blk*256 + 128 + w (B part),
// blk = j / 128, w = j % 128. Writes phi * rowscale to C and phi to C2 (when set).
struct SimtSwiglu {
  SimtArgs g;
  void* C2; long long ld2, c2s0, c2s1;
  const float* rs; long long rs0, rs1;
  // gradient variant (see SwigluGemm): C = phi * eta, C2 = d silu(A), C3 = d B silu'(A)
  int grad, skip_out1;
  void* C3;
  const void* dv; long long ldd, ds0, ds1;
};

template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(THREADS) simt_swiglu_kernel(const SimtSwiglu sw) {
  const SimtArgs& a = sw.g;
  __shared__ float As[TK][TM + 1];
  __shared__ float Ba[TK][TN + 1];
  __shared__ float Bb[TK][TN + 1];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int i0 = blockIdx.y * TM, j0 = blockIdx.x * TN;
  const int z0 = blockIdx.z % a.Z0, z1 = blockIdx.z / a.Z0;
  const TA* A = static_cast<const TA*>(a.A) + z0 * a.as0 + z1 * a.as1;
  const TB* B = static_cast<const TB*>(a.B) + z0 * a.bs0 + z1 * a.bs1;
  float acc_a[4][4], acc_b[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc_a[r][c] = acc_b[r][c] = 0.0f;
  for (int k0 = 0; k0 < a.K; k0 += TK) {
    for (int e = tid; e < TM * TK; e += THREADS) {
      int ii, kk;
      if (a.a_mn) { ii = e % TM; kk = e / TM; } else { kk = e % TK; ii = e / TK; }
      const int gi = i0 + ii, gk = k0 + kk;
      float val = 0.0f;
      if (gi < a.M && gk < a.K)
        val = to_f32(A[a.a_mn ? (long long)gk * a.lda + gi : (long long)gi * a.lda + gk]);
      As[kk][ii] = val;
    }
    for (int e = tid; e < TN * TK; e += THREADS) {
      const int kk = e % TK, jj = e / TK;
      const int gj = j0 + jj, gk = k0 + kk;
      float va = 0.0f, vb = 0.0f;
      if (gj < a.N && gk < a.K) {
        const long long ra = (long long)(gj / 128) * 256 + (gj % 128);
        va = to_f32(B[ra * a.ldb + gk]);
        vb = to_f32(B[(ra + 128) * a.ldb + gk]);
      }
      Ba[kk][jj] = va;
      Bb[kk][jj] = vb;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float af[4], ba[4], bb[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) af[r] = As[kk][ty + 16 * r];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        ba[c] = Ba[kk][tx + 16 * c];
        bb[c] = Bb[kk][tx + 16 * c];
      }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc_a[r][c] = fmaf(af[r], ba[c], acc_a[r][c]);
          acc_b[r][c] = fmaf(af[r], bb[c], acc_b[r][c]);
        }
    }
    __syncthreads();
  }
  TC* C = static_cast<TC*>(a.C) + z0 * a.cs0 + z1 * a.cs1;
  TC* C2 = sw.C2 ? static_cast<TC*>(sw.C2) + z0 * sw.c2s0 + z1 * sw.c2s1 : nullptr;
  TC* C3 = sw.C3 ? static_cast<TC*>(sw.C3) + z0 * a.cs0 + z1 * a.cs1 : nullptr;
  const TC* DV = sw.dv ? static_cast<const TC*>(sw.dv) + z0 * sw.ds0 + z1 * sw.ds1 : nullptr;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int gi = i0 + ty + 16 * r;
    if (gi >= a.M) continue;
    const float rsv = sw.rs ? sw.rs[z0 * sw.rs0 + z1 * sw.rs1 + gi] : 1.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int gj = j0 + tx + 16 * c;
      if (gj >= a.N) continue;
      const float av = 2.0f * acc_a[r][c], bv = acc_b[r][c];   // the operand holds W0 / 2
      const float sa = siluf_(av);
      const float p = sa * bv;
      if (!sw.skip_out1) C[(long long)gi * a.ldc + gj] = from_f32<TC>(p * rsv);
      if (sw.grad) {
        const float d = -rsv * to_f32(DV[(long long)gi * sw.ldd + gj]);
        if (C2) C2[(long long)gi * a.ldc + gj] = from_f32<TC>(d * sa);
        if (C3) C3[(long long)gi * a.ldc + gj] = from_f32<TC>(d * bv * silu_primef_(av));
      } else if (C2) {
        C2[(long long)gi * sw.ld2 + gj] = from_f32<TC>(p);
      }
    }
  }
}

}  // namespace

ttt_status gemm_simt_swiglu(const SwigluGemm& g, cudaStream_t stream) {
  const GemmProblem& p = g.gemm;
  if (p.M <= 0 || g.n_valid <= 0 || p.Z0 <= 0 || p.Z1 <= 0) return TTT_OK;
  const long long gy = (p.M + TM - 1) / TM, gz = (long long)p.Z0 * p.Z1;
  if (gy > 65535 || gz > 65535 || p.B.mn_major) {
    set_error_message("gemm_simt_swiglu: unsupported problem (M=%d, Z=%lld)", p.M, gz);
    return TTT_ERR_UNSUPPORTED;
  }
  SimtSwiglu sw;
  SimtArgs& a = sw.g;
  a.M = p.M; a.N = g.n_valid; a.K = p.K; a.Z0 = p.Z0;
  a.A = p.A.ptr; a.lda = p.A.ld; a.as0 = p.A.s0; a.as1 = p.A.s1; a.a_mn = p.A.mn_major;
  a.B = p.B.ptr; a.ldb = p.B.ld; a.bs0 = p.B.s0; a.bs1 = p.B.s1; a.b_mn = 0;
  a.C = p.C.ptr; a.ldc = p.C.ld; a.cs0 = p.C.s0; a.cs1 = p.C.s1;
  a.Cin = nullptr; a.ldi = a.is0 = a.is1 = 0;
  a.alpha = 1.0f; a.beta = 0.0f;
  sw.C2 = g.out2; sw.ld2 = g.ld2; sw.c2s0 = g.s20; sw.c2s1 = g.s21;
  sw.rs = g.rowscale; sw.rs0 = g.rs0; sw.rs1 = g.rs1;
  sw.grad = g.grad;
  sw.skip_out1 = g.grad ? g.skip_out1 : 0;
  sw.C3 = g.grad ? g.out3 : nullptr;
  sw.dv = g.grad ? g.dv : nullptr;
  sw.ldd = g.ldd; sw.ds0 = g.ds0; sw.ds1 = g.ds1;
  if (g.grad && (!g.rowscale || !g.dv)) {
    set_error_message("gemm_simt_swiglu: the gradient variant needs eta and Dv");
    return TTT_ERR_INVALID_ARG;
  }
  dim3 grid((g.n_valid + TN - 1) / TN, (unsigned)gy, (unsigned)gz);
  using bf = __nv_bfloat16;
  const int key = (p.A.dtype << 2) | (p.B.dtype << 1) | p.C.dtype;
  switch (key) {
    case 0: simt_swiglu_kernel<float, float, float><<<grid, THREADS, 0, stream>>>(sw); break;
    case 7: simt_swiglu_kernel<bf, bf, bf><<<grid, THREADS, 0, stream>>>(sw); break;
    default:
      set_error_message("gemm_simt_swiglu: operands and output must share one element type");
      return TTT_ERR_UNSUPPORTED;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error_message("gemm_simt_swiglu launch: %s", cudaGetErrorString(e));
    return TTT_ERR_CUDA;
  }
  return TTT_OK;
}

ttt_status gemm_simt(const GemmProblem& p, cudaStream_t stream) {
  if (p.M <= 0 || p.N <= 0 || p.Z0 <= 0 || p.Z1 <= 0) return TTT_OK;
  if (p.zss) {
    set_error_message("gemm_simt: per-entry scales are taken only by the tf32 engine");
    return TTT_ERR_UNSUPPORTED;
  }
  const long long gy = (p.M + TM - 1) / TM, gz = (long long)p.Z0 * p.Z1;
  if (gy > 65535 || gz > 65535) {
    set_error_message("gemm_simt: grid too large (M=%d, Z=%lld)", p.M, gz);
    return TTT_ERR_UNSUPPORTED;
  }
  SimtArgs a;
  a.M = p.M; a.N = p.N; a.K = p.K; a.Z0 = p.Z0;
  a.A = p.A.ptr; a.lda = p.A.ld; a.as0 = p.A.s0; a.as1 = p.A.s1; a.a_mn = p.A.mn_major;
  a.B = p.B.ptr; a.ldb = p.B.ld; a.bs0 = p.B.s0; a.bs1 = p.B.s1; a.b_mn = p.B.mn_major;
  a.C = p.C.ptr; a.ldc = p.C.ld; a.cs0 = p.C.s0; a.cs1 = p.C.s1;
  a.Cin = p.beta != 0.0f ? p.Cin.ptr : nullptr;
  a.ldi = p.Cin.ld; a.is0 = p.Cin.s0; a.is1 = p.Cin.s1;
  a.alpha = p.alpha; a.beta = p.beta;
  dim3 grid((p.N + TN - 1) / TN, (unsigned)gy, (unsigned)gz);
  const int key = (p.A.dtype << 2) | (p.B.dtype << 1) | p.C.dtype;
  using bf = __nv_bfloat16;
  switch (key) {
    case 0: launch_simt<float, float, float>(a, grid, stream); break;
    case 1: launch_simt<float, float, bf>(a, grid, stream); break;
    case 2: launch_simt<float, bf, float>(a, grid, stream); break;
    case 3: launch_simt<float, bf, bf>(a, grid, stream); break;
    case 4: launch_simt<bf, float, float>(a, grid, stream); break;
    case 5: launch_simt<bf, float, bf>(a, grid, stream); break;
    case 6: launch_simt<bf, bf, float>(a, grid, stream); break;
    default: launch_simt<bf, bf, bf>(a, grid, stream); break;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error_message("gemm_simt launch: %s", cudaGetErrorString(e));
    return TTT_ERR_CUDA;
  }
  return TTT_OK;
}

}  // namespace ttt
