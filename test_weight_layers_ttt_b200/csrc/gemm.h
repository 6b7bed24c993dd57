// Batched GEMM problem shared by the host orchestration and the two GEMM engines
// (tcgen05/TMA tensor-core engine for bf16 operands, CUDA-core engine for fp32).
//
//   C[z](i, j) = alpha * sum_k A[z](i, k) * B[z](j, k) + beta * Cin[z](i, j)
//
// for i < M, j < N, z = (z0, z1) in [0, Z0) x [0, Z1). Operand X in {A, B} with row index
// r (i for A, j for B) and reduction index k sits at
//   X.ptr + z0 * X.s0 + z1 * X.s1 + (mn_major ? k * X.ld + r : r * X.ld + k)   (elements).
// A batch stride of 0 broadcasts the operand over that batch index.
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace ttt {

struct GemmOperand {
  const void* ptr = nullptr;
  int dtype = DT_F32;
  bool mn_major = false;  // false: k contiguous ("K-major"); true: the row index contiguous
  long long ld = 0, s0 = 0, s1 = 0;
};

struct GemmOut {
  void* ptr = nullptr;
  int dtype = DT_F32;
  long long ld = 0, s0 = 0, s1 = 0;
  // fp32 C on the tensor-core engine only: a bf16 copy of the result with C's element
  // strides (e.g. the operand copy of a state kept in fp32), or null
  void* copy16 = nullptr;
};

struct GemmCin {
  const float* ptr = nullptr;  // fp32 addend, may alias C.ptr (same layout)
  long long ld = 0, s0 = 0, s1 = 0;
};

struct GemmProblem {
  int M = 0, N = 0, K = 0, Z0 = 1, Z1 = 1;
  GemmOperand A, B;
  GemmOut C;
  float alpha = 1.0f;
  float beta = 0.0f;
  GemmCin Cin;
  // tf32 engine only: per batch entry z0, alpha and beta further scaled by s^zpa and s^zpb
  // with s = 1 / (sqrt(zss[z0]) + zeps) (zss: sums of squares, e.g. of a Frobenius norm),
  // or null
  const float* zss = nullptr;
  float zeps = 0.0f;
  int zpa = 0, zpb = 0;
};

// CUDA-core engine: any strides, fp32 or bf16 operands, fp32 accumulation.
ttt_status gemm_simt(const GemmProblem& p, cudaStream_t stream);

// Tensor-core engine (tcgen05.mma kind::f16, TMEM accumulators, TMA operand loads).
// Requires bf16 A and B with 16-byte aligned bases and strides; see umma_supported.
bool umma_supported(const GemmProblem& p);
// Why the tensor-core engine cannot take `p` (a static string), or null when it can.
const char* umma_unsupported_reason(const GemmProblem& p);
ttt_status gemm_umma(const GemmProblem& p, cudaStream_t stream, unsigned* dev_err,
                     unsigned long long wait_ns);
// The same engine with fp32 A and B consumed as tf32 (tcgen05.mma kind::tf32: operands
// rounded toward zero to a 10-bit mantissa, fp32 accumulation); either major, fp32
// C. For bf16-mode products that need more than bf16 operand precision.
const char* umma_tf32_unsupported_reason(const GemmProblem& p);
ttt_status gemm_umma_tf32(const GemmProblem& p, cudaStream_t stream, unsigned* dev_err,
                          unsigned long long wait_ns);

// Feature GEMM with the SwiGLU applied in the epilogue. gemm.B holds the input-side
// weights as 128-row blocks [W0^T rows j..j+127 / 2 ; W2^T rows j..j+127] (256 rows per
// block, zero rows past m; see prep_wk_blocked), so gemm.N = 2 * ceil(m / 128) * 128 and
// every 256-wide output tile carries matching A/2 and B columns. With A = X W0 and
// B = X W2, the epilogue writes phi = silu(A) * B = (A/2) (1 + tanh(A/2)) B times
// rowscale[z0*rs0 + z1*rs1 + row] (or 1 when rowscale is null) to gemm.C (bf16, row stride
// gemm.C.ld, phi columns < n_valid) and, when out2 is set, the unscaled phi to out2.
//
// Gradient variant (grad = 1, recurrent form): with eta = rowscale and d = -eta * Dv, Dv =
// V W1^T given in `dv` (bf16 [rows, n_valid] with its own strides), the epilogue writes
// P = phi * eta to gemm.C (unless skip_out1), E2 = d * silu(A) to out2 (when set) and
// E0 = d * B * silu'(A) to out3 (when set). With rowscale = -1 and dv = dphi this is the
// SwiGLU backward: E0 = dA, E2 = dB.
struct SwigluGemm {
  GemmProblem gemm;
  void* out2 = nullptr;
  long long ld2 = 0, s20 = 0, s21 = 0;
  const float* rowscale = nullptr;
  long long rs0 = 0, rs1 = 0;
  int n_valid = 0;
  int grad = 0;
  int skip_out1 = 0;   // gradient variant: do not write P (gemm.C)
  void* out3 = nullptr;
  long long ld3 = 0, s30 = 0, s31 = 0;
  const void* dv = nullptr;
  long long ldd = 0, ds0 = 0, ds1 = 0;
};
// Query side of the parallel form fused (apply_fused.cu): out = phi(Q) S_c per 128-row tile
// with phi kept in shared memory. q [B,H,N,h] bf16; Wk the blocked [W0/2 ; W2] operand per
// head ([H, 2 * mpad, h], see prep_wk_blocked); Sc the bf16 chunk states [B*H, C, m, h];
// out [B,H,N,h] bf16. Needs h = 128 or 256 and chunk % 128 == 0.
bool fused_apply_supported(int dtype, int h, int m, int chunk, const void* q, const void* Wk,
                           const void* Sc, const void* out);
ttt_status fused_apply(const void* q, const void* Wk, const void* Sc, void* out, int B, int H,
                       int N, int h, int m, int chunk, unsigned* err,
                       unsigned long long wait_ns, cudaStream_t s);

// Key side of the parallel form fused (delta_fused.cu): dS[bh, c] = sign * phi(K_c)^T
// diag(eta_c) V_c per (batch, head) and chunk with phi kept in shared memory. k, v
// [B,H,N,h] bf16; eta [B,H,N] fp32; Wk the blocked [W0/2 ; W2] operand per head
// ([H, 2 * mpad, h]); dS [B*H, C, m, h] fp32, written. Needs h = 128 or 256.
bool fused_delta_supported(int dtype, int h, int m, const void* k, const void* v,
                           const float* eta, const void* Wk, const float* dS);
ttt_status fused_delta(const void* k, const void* v, const float* eta, const void* Wk, float* dS,
                       int B, int H, int N, int h, int m, int chunk, int sign, unsigned* err,
                       unsigned long long wait_ns, cudaStream_t s);

bool umma_swiglu_supported(const SwigluGemm& g);
const char* umma_swiglu_unsupported_reason(const SwigluGemm& g);
ttt_status gemm_simt_swiglu(const SwigluGemm& g, cudaStream_t stream);
ttt_status gemm_umma_swiglu(const SwigluGemm& g, cudaStream_t stream, unsigned* dev_err,
                            unsigned long long wait_ns);

// Error-word access (ttt_api.cu).
unsigned* device_error_word();
unsigned long long wait_limit_ns();
void set_error_message(const char* fmt, ...);

}  // namespace ttt
