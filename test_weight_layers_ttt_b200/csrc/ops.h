// Launch wrappers of the non-GEMM kernels of the TTT layer (ops.cu). All of them enqueue
// on `s` and return the launch status. OT is the operand element type of the dense
// contractions (bf16 in bf16 mode, fp32 in fp32 mode), passed as a DType tag.
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace ttt {

// Fast-weight input-side operand of the SwiGLU-epilogue GEMM, per entry e (source head
// e % src_heads; source layout 0: [h, m], 1: [m, h]): 128-row blocks
// [W0^T rows j..j+127 / 2 ; W2^T rows j..j+127] ([2 * ceil(m/128) * 128, h], K-major, zero
// rows past m). W0 enters halved (exact in binary floating point), so the GEMM's first
// half yields a/2 = (x W0)/2, the argument silu takes through tanh:
// silu(a) = (a/2) (1 + tanh(a/2)).
// Wk1, Wk2: further copies of the same operand, or null.
cudaError_t prep_wk_blocked(int ot, const float* W0, const float* W2, void* Wk, int n_entries,
                            int src_heads, int h, int m, int src_layout, cudaStream_t s,
                            void* Wk1 = nullptr, void* Wk2 = nullptr);

// Xs[r, :] = X[r, :] * eta[r] for `rows` rows of width w (OT in and out; eta fp32).
cudaError_t scale_rows(int ot, const void* X, const float* eta, void* Xs, long long rows, int w,
                       cudaStream_t s);

// Chunk prefix sums: S starts at W1[bh % H] (layout 0 [m,h] / 1 [h,m]; zero when W1 is
// null) plus the n_prior states prior[i, bh] (W1's layout, [n_prior, BH, ...]); for each
// chunk c the state read by chunk c is written to Sc[bh, c] (OT, [m,h]; skipped when Sc is
// null): inclusive of dS[bh, c] (order 0) or exclusive (order 1). The state after the last
// chunk goes to S_final (fp32, W1's layout) when non-null. With layout 1 and a scratch of
// (H + BH) * m * h floats, W1, the priors and S_final are transposed through it so the scan
// itself runs on 16-byte vectors.
cudaError_t chunk_scan(int ot, const float* dS, const float* W1, const float* prior, int n_prior,
                       void* Sc, float* S_final, int BH, int H, int C, int m, int h, int order,
                       int layout, float* scratch, cudaStream_t s);

// Recurrent-state helpers. Per (b, head) the fp32 state W_all holds the three fast
// matrices output-major, i.e. transposed: [W0^T (m x h) | W1^T (h x m) | W2^T (m x h)], each
// row one output unit over the input dimension (so the renormalisation is a row norm);
// momentum, the update buffer U and the split-K gradient partials use the same layout.
// rec_init transposes the per-head initial weights (original layouts W0, W2 [h, m], W1
// [m, h]) into W_all, writes W1t = the OT copy of W1^T [BH, h, m] (and the same into W1t1,
// W1t2 when not null) and, with momentum, M_all = M_in^T (M_in in the original part
// layouts) or 0.
cudaError_t rec_init(int ot, const float* W0, const float* W2, const float* W1, int BH, int H,
                     int h, int m, float* W_all, void* W1t, const float* M_in, float* M_all,
                     int momentum, cudaStream_t s, void* W1t1 = nullptr, void* W1t2 = nullptr);
// Column norms over the input dimension of the initial weights, per head:
// tnorm[head] = [W0 columns (m) | W1 columns (h) | W2 columns (m)].
cudaError_t col_norms(const float* W0, const float* W2, const float* W1, int H, int h, int m,
                      float* tnorm, cudaStream_t s);
// U = sum over `splits` partial gradients [split][BH][3hm] (parts ordered [W0^T | W2^T |
// W1^T] in the partials, [W0^T | W1^T | W2^T] in U); with momentum M <- alpha[bh, c] * M + U
// and U <- M. Only parts in `mask` are touched.
cudaError_t rec_reduce(const float* partials, int splits, float* U, float* M_all,
                       const float* alpha, int C, int c, int BH, int h, int m, int mask,
                       cudaStream_t s);
// Where the matrices of a batched Newton-Schulz live: matrix (part p, entry z) starts at
// U + z * zstride + p * pstride and is [R[p], C[p]] row-major (every part has R * C
// elements); parts not in `mask` are skipped.
struct NsLayout {
  int parts, mask;
  long long zstride, pstride;
  int R[3], C[3];
};
// The output-major recurrent state [W0^T (m x h) | W1^T (h x m) | W2^T (m x h)] of each
// (b, head).
inline NsLayout ns_layout_weights(int h, int m, int mask) {
  const long long hm = (long long)h * m;
  return NsLayout{3, mask, 3 * hm, hm, {m, h, m}, {h, m, h}};
}
// One [R, C] matrix per entry, entries R * C apart.
inline NsLayout ns_layout_single(int R, int C) {
  return NsLayout{1, 1, (long long)R * C, 0, {R, R, R}, {C, C, C}};
}

// Newton-Schulz set-up / tear-down for the batched paths: X = U / (||U||_F + eps) in the
// wide orientation ([min(R,C), max(R,C)]) into the scratch X (problem (z, p) at
// (z * parts + p) * R * C), with its transpose into Xt; either may be null (X null and Xt
// set: the scaled matrix in U's own orientation when R > C), and U <- X back
// in U's own orientation. Z entries. nrm: fp32 scratch of Z * parts sums of squares
// (already holding them when nrm_ready).
cudaError_t ns_normalize(const float* U, float* X, int Z, const NsLayout& L, float eps,
                         float* nrm, cudaStream_t s, float* Xt = nullptr,
                         bool nrm_ready = false);
cudaError_t ns_writeback(const float* X, float* U, int Z, const NsLayout& L, cudaStream_t s);
// The sums of squares alone (nrm[z * parts + p] = ||U_(z,p)||_F^2).
cudaError_t ns_sumsq(const float* U, int Z, const NsLayout& L, float* nrm, cudaStream_t s);

// The whole Newton-Schulz orthogonalisation of the matrices of L on the tensor cores
// (ns_mma.cu; operands split into bf16 hi + lo pairs, fp32 accumulation): normalise,
// `steps` iterations X <- a X + (b A + c A A) X with A = X X^T on the rows <= cols
// orientation, write back. Only for min(R, C) <= 128 and max(R, C) <= 256 for every part
// (ns_mma_supported). Bounded waits report through `err`.
bool ns_mma_supported(int R, int C);
cudaError_t ns_mma(float* U, int Z, const NsLayout& L, int steps, float eps, float a, float b,
                   float c, unsigned* err, unsigned long long wait_ns, cudaStream_t s);


// Backward of the prefix scan: R = dS_final[bh] (or 0 when null), then for c = C-1 .. 0:
// R += dSc[bh, c] and the gradient of chunk c's delta G[bh, c] (OT) is R (order 0) or the
// value before the addition (order 1); R0[bh] = the final R (fp32). [BH, C, n] / [BH, n].
cudaError_t suffix_scan(int ot, const float* dSc, const float* dS_final, void* G, float* R0,
                        int BH, int C, long long n, int order, cudaStream_t s);
// dv[r] = sign * eta[r] * T[r] (OT) and deta[r] = sign * <T[r], v[r]> for `rows` rows of
// width w (T fp32, v OT).
cudaError_t row_grads(int ot, const float* T, const void* v, const float* eta, int sign,
                      void* dv, float* deta, long long rows, int w, cudaStream_t s);
// out[i] = sum over b of X[b * stride + i] for i < n (fp32).
cudaError_t sum_batches(const float* X, int B, long long stride, long long n, float* out,
                        cudaStream_t s);
// Cast fp32 to OT (n elements).
cudaError_t cast_to(int ot, const float* X, void* out, long long n, cudaStream_t s);
// out[r] = [A[r] | B[r]] (OT) for `rows` rows of width w each (A, B fp32).
cudaError_t cat_cols(int ot, const float* A, const float* B, void* out, long long rows, int w,
                     cudaStream_t s);
// X [nb, rows, 2w] fp32 summed over nb: columns < w to out0 [rows, w], the rest to out1.
cudaError_t sum_split_cols(const float* X, int nb, long long rows, int w, float* out0,
                           float* out1, cudaStream_t s);

// Momentum over chunks, in place: D[bh, c] <- alpha[bh, c] * D[bh, c - 1] + D[bh, c] for
// c = 1 .. C-1 (D [BH, C, n] fp32, alpha [BH, C]). With nrm (only where
// momentum_scan_norms holds), also nrm[bh * C + c] = the sum of squares of the result
// D[bh, c] (the Frobenius norms the Newton-Schulz set-up needs).
bool momentum_scan_norms(int C, long long n, const float* D);
cudaError_t momentum_scan(float* D, const float* alpha, int BH, int C, long long n,
                          cudaStream_t s, float* nrm = nullptr);

// One step on the output-major state, one warp per row: the update is U when given, else
// the sum of the `splits` partials (parts ordered as for rec_reduce) with the momentum
// M <- alpha[bh, c] M + g folded in;
// W <- W - sign * u; optional renormalisation of each row (output unit) to its initial
// norm tnorm; refresh of the OT operand copies W1t [BH, h, m] and the blocked input-side
// operand Wk [BH, 2 * mpad, h] (see prep_wk_blocked). Only parts in `mask`.
cudaError_t rec_step(float* W_all, const float* U, const float* partials, int splits,
                     float* M_all, const float* alpha, int C, int c, const float* tnorm, int BH,
                     int H, int h, int m, int mask, int sign, int renorm, void* Wk, void* W1t,
                     int ot, cudaStream_t s);
// Final weights [B,H,...] in the original layouts (nullable outputs) and the momentum
// copy-out (original part layouts), transposed back from the output-major state.
cudaError_t rec_finish(const float* W_all, int BH, int H, int h, int m, float* W0_out,
                       float* W2_out, float* W1_out, const float* M_all, float* M_out,
                       cudaStream_t s);

// Causal depthwise 4-tap convolution: Xc[t, i] = sum_j conv_w[j, i] * X0[t - j, i] (bf16).
cudaError_t conv4_causal(const void* X0, const float* conv_w, void* Xc, int N, int d,
                         cudaStream_t s);

// Block that waits on an mbarrier nobody arrives at, bounded by `limit_ns`.
cudaError_t wait_timeout_probe(unsigned* err, unsigned long long limit_ns, cudaStream_t s);

cudaError_t fill_f32(float* p, long long n, float v, cudaStream_t s);

// Start of the parallel form's sequential schedule: master[bh] = W1[bh % H] (zero when null)
// + sum_i prior[i, bh] (fp32) and shadow = its bf16 copy; n elements per (b, head) entry.
cudaError_t seq_init(const float* W1, const float* prior, int n_prior, int BH, int H, long long n,
                     float* master, void* shadow, cudaStream_t s);

// Debug checks (checks.cu). Guards: kGuardBytes-long words written before a call's first
// kernel and compared after its last one (a change records DEVERR_BOUNDS); at most
// kMaxGuards per launch. finite_scan records DEVERR_NONFINITE when any of the n elements
// (fp32 or bf16, dt) is NaN or Inf.
constexpr int kGuardBytes = 256;
constexpr int kMaxGuards = 64;
struct GuardList {
  int n;
  unsigned* p[kMaxGuards];
};
cudaError_t guards_fill(const GuardList& g, cudaStream_t s);
cudaError_t guards_check(const GuardList& g, unsigned* err, cudaStream_t s);
cudaError_t finite_scan(int dt, const void* x, long long n, unsigned* err, cudaStream_t s);

}  // namespace ttt
