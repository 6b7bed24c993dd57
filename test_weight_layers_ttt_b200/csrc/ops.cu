// Non-GEMM kernels of the TTT layer: weight preparation (the blocked input-side operand),
// the chunk prefix scan over fp32 states, the recurrent update operators
// (momentum, Newton-Schulz set-up, step, per-column renormalisation), the causal Conv1D of
// the In-Place target, and the bounded-wait diagnostic.
#include "ops.h"
#include "umma.cuh"

namespace ttt {
namespace {

using bf16 = __nv_bfloat16;

// ------------------------------------------------------------------ weight preparation
// Tiled through shared memory so both the reads of W0/W2 (either layout) and the writes
// of the blocked operand are coalesced. grid (mpad/32, ceil(h/32), 2 * n_entries),
// block (32, 8); blockIdx.z = 2 * entry + which (0: W0, 1: W2).
template <typename OT>
__global__ void prep_wk_blocked_kernel(const float* W0, const float* W2, OT* Wk, OT* Wk1, OT* Wk2,
                                       int src_heads, int h, int m, int layout) {
  __shared__ float tile[32][33];
  const int mpad = (m + 127) / 128 * 128;
  const int j0 = blockIdx.x * 32, i0 = blockIdx.y * 32;
  const int e = blockIdx.z >> 1, which = blockIdx.z & 1;
  const float* src = (which ? W2 : W0) + (long long)(e % src_heads) * h * m;
  const int tx = threadIdx.x, ty = threadIdx.y;
  // tile[jj][ii] = W(i0 + ii, j0 + jj), zero past m (padding rows) or past h
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = ty + 8 * k;
    if (layout == 0) {  // [h, m]: consecutive tx -> consecutive j
      const int i = i0 + r, j = j0 + tx;
      tile[tx][r] = (i < h && j < m) ? src[(long long)i * m + j] : 0.0f;
    } else {            // [m, h]: consecutive tx -> consecutive i
      const int j = j0 + r, i = i0 + tx;
      tile[r][tx] = (i < h && j < m) ? src[(long long)j * h + i] : 0.0f;
    }
  }
  __syncthreads();
  const long long eo = (long long)e * 2 * mpad * h;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int jj = ty + 8 * k, j = j0 + jj, i = i0 + tx;
    if (j >= mpad || i >= h) continue;
    const long long row = (long long)(j >> 7) * 256 + (which ? 128 : 0) + (j & 127);
    const OT x = from_f32<OT>(which ? tile[jj][tx] : 0.5f * tile[jj][tx]);
    Wk[eo + row * h + i] = x;
    if (Wk1) Wk1[eo + row * h + i] = x;   // further copies of the same operand
    if (Wk2) Wk2[eo + row * h + i] = x;
  }
}

// ------------------------------------------------------------------ row scaling
template <typename OT>
__global__ void scale_rows_kernel(const OT* X, const float* eta, OT* Xs, long long rows, int w) {
  TTT_GRID_LOOP(idx, rows * w) {
    const long long r = idx / w;
    Xs[idx] = from_f32<OT>(to_f32(X[idx]) * eta[r]);
  }
}

// 16-byte version: one thread per 8 bf16 of a row (w % 8 == 0, 16-byte aligned rows).
__global__ void scale_rows8_kernel(const uint4* X, const float* eta, uint4* Xs, long long rows,
                                   int w8) {
  TTT_GRID_LOOP(idx, rows * w8) {
    const float e = eta[idx / w8];
    const uint4 u = X[idx];
    const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&u);
    uint4 o;
    __nv_bfloat162* ov = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(hv[q]);
      ov[q] = __floats2bfloat162_rn(f.x * e, f.y * e);
    }
    Xs[idx] = o;
  }
}

// ------------------------------------------------------------------ chunk prefix scan
// One thread per state element; the chunk axis (tens of chunks) is walked sequentially so
// every delta is read once and every chunk state written once.
// Initial state of (b, head) bh: W1[bh % H] (zero when W1 is null) plus the n_prior states
// prior[i, bh] ([n_prior, BH, ...] in W1's layout).
template <typename OT>
__global__ void chunk_scan_kernel(const float* __restrict__ dS, const float* __restrict__ W1,
                                  const float* __restrict__ prior, int n_prior,
                                  OT* __restrict__ Sc, float* __restrict__ S_final, int BH,
                                  int H, int C, int m, int h, int order, int layout) {
  const long long per = (long long)m * h;
  TTT_GRID_LOOP(idx, per * BH) {
    const long long bh = idx / per, e = idx - bh * per;
    const int k = (int)(e / h), j = (int)(e - (long long)k * h);
    const long long le = layout == 0 ? e : (long long)j * m + k;   // e in W1's layout
    float s = W1 ? W1[(bh % H) * per + le] : 0.0f;
    for (int i = 0; i < n_prior; ++i) s += prior[((long long)i * BH + bh) * per + le];
    const float* d = dS + bh * C * per + e;
    OT* out = Sc ? Sc + bh * C * per + e : nullptr;
    int c = 0;
    // Four chunks per step with the loads issued first, so each thread keeps four
    // independent loads in flight.
    for (; c + 4 <= C; c += 4) {
      float dv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) dv[u] = __ldcs(d + (long long)(c + u) * per);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (order == 1) {
          if (out) out[(long long)(c + u) * per] = from_f32<OT>(s);
          s += dv[u];
        } else {
          s += dv[u];
          if (out) out[(long long)(c + u) * per] = from_f32<OT>(s);
        }
      }
    }
    for (; c < C; ++c) {
      const float dv = __ldcs(d + (long long)c * per);
      if (order == 1) {
        if (out) out[(long long)c * per] = from_f32<OT>(s);
        s += dv;
      } else {
        s += dv;
        if (out) out[(long long)c * per] = from_f32<OT>(s);
      }
    }
    if (S_final) S_final[bh * per + (layout == 0 ? e : (long long)j * m + k)] = s;
  }
}

// Four consecutive state elements per thread (16-byte loads), for W1 in layout 0 and
// m*h divisible by 4; the chunk loop keeps four 16-byte loads in flight.
template <typename OT>
__global__ void chunk_scan4_kernel(const float4* __restrict__ dS, const float4* __restrict__ W1,
                                   const float4* __restrict__ prior, int n_prior,
                                   OT* __restrict__ Sc, float4* __restrict__ S_final, int BH,
                                   int H, int C, long long per4, int order) {
  TTT_GRID_LOOP(idx, per4 * BH) {
    const long long bh = idx / per4, e = idx - bh * per4;
    float4 s = W1 ? W1[(bh % H) * per4 + e] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int i = 0; i < n_prior; ++i) {
      const float4 p = prior[((long long)i * BH + bh) * per4 + e];
      s.x += p.x; s.y += p.y; s.z += p.z; s.w += p.w;
    }
    const float4* d = dS + bh * C * per4 + e;
    OT* out = Sc ? Sc + (bh * C * per4 + e) * 4 : nullptr;
    auto put = [&](int c, const float4& v) {
      if (!out) return;
      OT* o = out + (long long)c * per4 * 4;
      if constexpr (sizeof(OT) == 2) {
        uint2 pk;
        __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(o) = pk;
      } else {
        *reinterpret_cast<float4*>(o) = v;
      }
    };
    int c = 0;
    for (; c + 4 <= C; c += 4) {
      float4 dv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) dv[u] = __ldcs(d + (long long)(c + u) * per4);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (order == 1) put(c + u, s);
        s.x += dv[u].x; s.y += dv[u].y; s.z += dv[u].z; s.w += dv[u].w;
        if (order != 1) put(c + u, s);
      }
    }
    for (; c < C; ++c) {
      const float4 dv = __ldcs(d + (long long)c * per4);
      if (order == 1) put(c, s);
      s.x += dv.x; s.y += dv.y; s.z += dv.z; s.w += dv.w;
      if (order != 1) put(c, s);
    }
    if (S_final) S_final[bh * per4 + e] = s;
  }
}

// ------------------------------------------------------------------ sequential schedule
// Per (b, head) entry bh: master = W1[bh % H] (zero when W1 is null) + sum of the n_prior
// states prior[i, bh], and shadow = its bf16 copy; n elements per entry, any layout.
__global__ void seq_init_kernel(const float* W1, const float* prior, int n_prior, int BH, int H,
                                long long n, float* master, __nv_bfloat16* shadow) {
  TTT_GRID_LOOP(idx, (long long)BH * n) {
    const long long bh = idx / n, e = idx - bh * n;
    float v = W1 ? W1[(bh % H) * n + e] : 0.0f;
    for (int i = 0; i < n_prior; ++i) v += prior[((long long)i * BH + bh) * n + e];
    master[idx] = v;
    shadow[idx] = __float2bfloat16_rn(v);
  }
}

// ------------------------------------------------------------------ recurrent state
// Offset, in units of h*m, of part p of a (b, head) block of the split-K gradient partials,
// stored [W0^T | W2^T | W1^T] so the W0 and W2 gradients are one GEMM's contiguous output.
__device__ __forceinline__ int partial_part(int p) { return p == 0 ? 0 : p == 1 ? 2 : 1; }

// Part p of a (b, head) state: p = 0 W0 [h, m], p = 1 W1 [m, h], p = 2 W2 [h, m].
__device__ __forceinline__ void part_dims(int p, int h, int m, int& R, int& Cc) {
  if (p == 1) { R = m; Cc = h; } else { R = h; Cc = m; }
}

// Part p of a (b, head) state in the original (input-major) layout: W0 [h, m], W1 [m, h],
// W2 [h, m]; the recurrent state keeps each part output-major, i.e. transposed.
// grid (tiles of the largest part, 3, BH), block (32, 8): one 32 x 32 tile of part p through
// shared memory; both the original-layout side and the output-major side are accessed
// along their rows. dir 0 (set-up): W_all[bh] part p = W_p[head]^T (and W1t = bf16 of the
// W1 part, M_all = M_in^T or 0); dir 1 (tear-down): out_p[bh] = W_all[bh] part p^T (and
// M_out = M_all^T).
template <typename OT>
__global__ void rec_transpose_kernel(int dir, const float* W0, const float* W2, const float* W1,
                                     int H, int h, int m, float* W_all, OT* W1t, OT* W1t1,
                                     OT* W1t2, const float* M_in, float* M_all, int momentum,
                                     float* W0_out, float* W2_out, float* W1_out, float* M_out) {
  __shared__ float t[2][32][33];
  const int p = blockIdx.y, bh = blockIdx.z, head = bh % H;
  int R, Cc;   // original layout [R, Cc]; output-major [Cc, R]
  part_dims(p, h, m, R, Cc);
  const int tiles_c = (Cc + 31) / 32;
  if ((int)blockIdx.x >= tiles_c * ((R + 31) / 32)) return;
  const int r0 = (blockIdx.x / tiles_c) * 32, c0 = (blockIdx.x % tiles_c) * 32;
  const long long hm = (long long)h * m;
  const long long st = (long long)bh * 3 * hm + p * hm;   // part p of W_all / M_all
  const int tx = threadIdx.x, ty = threadIdx.y;
  if (dir == 0) {
    const float* src = (p == 0 ? W0 : p == 1 ? W1 : W2) + (long long)head * hm;
    const float* msrc = M_in ? M_in + st : nullptr;
    for (int k = ty; k < 32; k += 8) {
      const int r = r0 + k, c = c0 + tx;
      if (r < R && c < Cc) {
        t[0][k][tx] = src[(long long)r * Cc + c];
        if (momentum) t[1][k][tx] = msrc ? msrc[(long long)r * Cc + c] : 0.0f;
      }
    }
    __syncthreads();
    for (int k = ty; k < 32; k += 8) {
      const int c = c0 + k, r = r0 + tx;   // output-major [Cc, R]
      if (r < R && c < Cc) {
        const long long o = (long long)c * R + r;
        W_all[st + o] = t[0][tx][k];
        if (p == 1) {
          const OT x = from_f32<OT>(t[0][tx][k]);
          W1t[(long long)bh * hm + o] = x;
          if (W1t1) W1t1[(long long)bh * hm + o] = x;   // further operand copies
          if (W1t2) W1t2[(long long)bh * hm + o] = x;
        }
        if (momentum) M_all[st + o] = t[1][tx][k];
      }
    }
  } else {
    float* dst = p == 0 ? W0_out : p == 1 ? W1_out : W2_out;
    for (int k = ty; k < 32; k += 8) {
      const int c = c0 + k, r = r0 + tx;
      if (r < R && c < Cc) {
        const long long o = (long long)c * R + r;
        t[0][tx][k] = W_all[st + o];
        if (M_out) t[1][tx][k] = M_all[st + o];
      }
    }
    __syncthreads();
    for (int k = ty; k < 32; k += 8) {
      const int r = r0 + k, c = c0 + tx;
      if (r < R && c < Cc) {
        const long long o = (long long)r * Cc + c;
        if (dst) dst[(long long)bh * hm + o] = t[0][k][tx];
        if (M_out) M_out[st + o] = t[1][k][tx];
      }
    }
  }
}

// Column norms (over the input dimension) of the initial weights, per head:
// tnorm[head] = [ W0 columns (m) | W1 columns (h) | W2 columns (m) ].
// grid (ceil((2m + h) / 32), H), block (32, 8): threadIdx.x takes one of 32 consecutive
// columns (coalesced rows), threadIdx.y every 8th row of it; the 8 partial sums (fp64) are
// added in shared memory.
__global__ void col_norms_kernel(const float* W0, const float* W2, const float* W1, int H, int h,
                                 int m, float* tnorm) {
  __shared__ double part[8][33];
  const int per = 2 * m + h, hd = blockIdx.y;
  const int c = blockIdx.x * 32 + threadIdx.x, ty = threadIdx.y;
  const long long hm = (long long)h * m;
  double ss = 0.0;
  if (c < per) {
    const float* base;
    int rows, ld;
    if (c < m) { base = W0 + hd * hm + c; rows = h; ld = m; }
    else if (c < m + h) { base = W1 + hd * hm + (c - m); rows = m; ld = h; }
    else { base = W2 + hd * hm + (c - m - h); rows = h; ld = m; }
#pragma unroll 4
    for (int r = ty; r < rows; r += 8) {
      const float w = base[(long long)r * ld];
      ss += (double)w * w;
    }
  }
  part[ty][threadIdx.x] = ss;
  __syncthreads();
  if (ty == 0 && c < per) {
    double t = 0.0;
#pragma unroll
    for (int y = 0; y < 8; ++y) t += part[y][threadIdx.x];
    tnorm[(long long)hd * per + c] = (float)sqrt(t);
  }
}

// Four consecutive elements per thread (requires h*m divisible by 4 and 16-byte bases).
__global__ void rec_reduce4_kernel(const float4* __restrict__ partials, int splits,
                                   float4* __restrict__ U, float4* __restrict__ M_all,
                                   const float* __restrict__ alpha, int C, int c, int BH,
                                   long long hm4, int mask) {
  const long long per4 = 3 * hm4, total4 = per4 * BH;
  TTT_GRID_LOOP(idx, total4) {
    const long long bh = idx / per4;
    const int p = (int)((idx - bh * per4) / hm4);
    if (!(mask & (1 << p))) continue;
    const long long pi = idx + (partial_part(p) - p) * hm4;
    float4 g = partials[pi];
    for (int s = 1; s < splits; ++s) {
      const float4 q = partials[(long long)s * total4 + pi];
      g.x += q.x; g.y += q.y; g.z += q.z; g.w += q.w;
    }
    if (M_all) {
      const float a = alpha[bh * C + c];
      float4 mv = M_all[idx];
      mv.x = fmaf(a, mv.x, g.x); mv.y = fmaf(a, mv.y, g.y);
      mv.z = fmaf(a, mv.z, g.z); mv.w = fmaf(a, mv.w, g.w);
      M_all[idx] = mv;
      g = mv;
    }
    U[idx] = g;
  }
}

__global__ void rec_reduce_kernel(const float* partials, int splits, float* U, float* M_all,
                                  const float* alpha, int C, int c, int BH, int h, int m,
                                  int mask) {
  const long long hm = (long long)h * m, per = 3 * hm, total = per * BH;
  TTT_GRID_LOOP(idx, total) {
    const long long bh = idx / per;
    const int p = (int)((idx - bh * per) / hm);
    if (!(mask & (1 << p))) continue;
    const long long pi = idx + (partial_part(p) - p) * hm;
    float g = 0.0f;
    for (int s = 0; s < splits; ++s) g += partials[(long long)s * total + pi];
    if (M_all) {
      const float mv = alpha[bh * C + c] * M_all[idx] + g;
      M_all[idx] = mv;
      g = mv;
    }
    U[idx] = g;
  }
}

// One block per (part, bh): Frobenius norm, then the normalised update in the orientation
// with rows <= cols.
// ||U||_F of every (part, entry) problem: grid (parts, Z, NS_SLABS) blocks of 256 threads,
// each adding its slab's sum of squares into nrm[z * parts + p] (zeroed first).
constexpr int NS_SLABS = 16;

__global__ void ns_sumsq_kernel(const float* U, NsLayout L, float* nrm) {
  const int p = blockIdx.x, z = blockIdx.y;
  if (!(L.mask & (1 << p))) return;
  const long long n = (long long)L.R[p] * L.C[p];
  const float* u = U + z * L.zstride + p * L.pstride;
  __shared__ float red[8];
  float ss = 0.0f;
  for (long long e = blockIdx.z * 256LL + threadIdx.x; e < n; e += 256LL * NS_SLABS)
    ss = fmaf(u[e], u[e], ss);
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.0f;
    for (int w = 0; w < 8; ++w) t += red[w];
    atomicAdd(&nrm[(long long)z * L.parts + p], t);
  }
}

// X (wide orientation) = U * scale and / or Xt = X^T (either may be null), 16 bytes per
// access: one 32 x 32 tile per block of 256 threads, each thread one float4 of a tile row
// (rows and columns multiples of 4, 16-byte aligned matrices); the transposed side goes
// through shared memory. grid (tiles of the problem, parts, Z).
__global__ void ns_norm4_kernel(const float* U, float* X, float* Xt, NsLayout L,
                                const float* nrm, float eps) {
  const int p = blockIdx.y, z = blockIdx.z;
  if (!(L.mask & (1 << p))) return;
  const int R = L.R[p], Cc = L.C[p];
  const int tc = (Cc + 31) / 32, tr_ = (R + 31) / 32;
  if ((int)blockIdx.x >= tc * tr_) return;
  const int i0 = (blockIdx.x / tc) * 32, j0 = (blockIdx.x % tc) * 32;   // tile of U [R, Cc]
  const long long n = (long long)R * Cc;
  const float* u = U + z * L.zstride + p * L.pstride;
  float* x = X ? X + ((long long)z * L.parts + p) * n : nullptr;
  float* xt = Xt ? Xt + ((long long)z * L.parts + p) * n : nullptr;
  const bool tr = R > Cc;
  float* same = tr ? xt : x;     // U's orientation [R, Cc]
  float* other = tr ? x : xt;    // the transposed one [Cc, R]
  const float scale = 1.0f / (sqrtf(nrm[(long long)z * L.parts + p]) + eps);
  __shared__ float t[32][33];
  const int r = threadIdx.x >> 3, q = (threadIdx.x & 7) * 4;
  const int i = i0 + r, j = j0 + q;
  float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  if (i < R && j < Cc) {
    v = *reinterpret_cast<const float4*>(u + (long long)i * Cc + j);
    v.x *= scale; v.y *= scale; v.z *= scale; v.w *= scale;
  }
  if (same && i < R && j < Cc) *reinterpret_cast<float4*>(same + (long long)i * Cc + j) = v;
  if (!other) return;
  t[r][q] = v.x; t[r][q + 1] = v.y; t[r][q + 2] = v.z; t[r][q + 3] = v.w;
  __syncthreads();
  const int jt = j0 + r, it = i0 + q;   // row jt of the transposed side, columns it .. it + 3
  if (jt < Cc && it < R)
    *reinterpret_cast<float4*>(other + (long long)jt * R + it) =
        make_float4(t[q][r], t[q + 1][r], t[q + 2][r], t[q + 3][r]);
}

// X (wide orientation) = U * scale and / or Xt = X^T (either may be null), or U <- X back
// (to_u): 32 x 32 tiles through shared memory so every side is read and written along rows.
// grid (tiles of the problem, parts, Z), block (32, 8).
__global__ void ns_copy_kernel(const float* U_in, float* X, float* U_out, NsLayout L,
                               const float* nrm, float eps, int to_u, float* Xt) {
  const int p = blockIdx.y, z = blockIdx.z;
  if (!(L.mask & (1 << p))) return;
  const int R = L.R[p], Cc = L.C[p];
  const int tc = (Cc + 31) / 32, tr_ = (R + 31) / 32;
  if ((int)blockIdx.x >= tc * tr_) return;
  const int i0 = (blockIdx.x / tc) * 32, j0 = (blockIdx.x % tc) * 32;   // tile of U [R, Cc]
  const long long n = (long long)R * Cc;
  const long long uoff = z * L.zstride + p * L.pstride;
  float* x = X ? X + ((long long)z * L.parts + p) * n : nullptr;
  const bool tr = R > Cc;
  __shared__ float t[32][33];
  const int tx = threadIdx.x, ty = threadIdx.y;
  if (!to_u) {
    const float scale = 1.0f / (sqrtf(nrm[(long long)z * L.parts + p]) + eps);
    const float* u = U_in + uoff;
    for (int k = ty; k < 32; k += 8) {
      const int i = i0 + k, j = j0 + tx;
      t[k][tx] = (i < R && j < Cc) ? u[(long long)i * Cc + j] * scale : 0.0f;
    }
    __syncthreads();
    float* xt = Xt ? Xt + ((long long)z * L.parts + p) * n : nullptr;
    for (int k = ty; k < 32; k += 8) {
      // U's own orientation [R, Cc] and the transposed one [Cc, R]
      const int i = i0 + k, j = j0 + tx;
      const int jt = j0 + k, it = i0 + tx;
      float* same = tr ? xt : x;
      float* other = tr ? x : xt;
      if (same && i < R && j < Cc) same[(long long)i * Cc + j] = t[k][tx];
      if (other && it < R && jt < Cc) other[(long long)jt * R + it] = t[tx][k];
    }
  } else {
    float* u = U_out + uoff;
    for (int k = ty; k < 32; k += 8) {
      if (!tr) {
        const int i = i0 + k, j = j0 + tx;
        t[k][tx] = (i < R && j < Cc) ? x[(long long)i * Cc + j] : 0.0f;
      } else {
        const int j = j0 + k, i = i0 + tx;
        t[tx][k] = (i < R && j < Cc) ? x[(long long)j * R + i] : 0.0f;
      }
    }
    __syncthreads();
    for (int k = ty; k < 32; k += 8) {
      const int i = i0 + k, j = j0 + tx;
      if (i < R && j < Cc) u[(long long)i * Cc + j] = t[k][tx];
    }
  }
}


// out[z] = in[z]^T for Z row-major [rows, cols] fp32 matrices: 32 x 32 tiles through shared
// memory, both sides along rows. grid (ceil(cols/32), ceil(rows/32), Z), block (32, 8).
__global__ void transpose_kernel(const float* in, float* out, int rows, int cols) {
  __shared__ float t[32][33];
  const long long z = blockIdx.z, n = (long long)rows * cols;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32, tx = threadIdx.x, ty = threadIdx.y;
  for (int k = ty; k < 32; k += 8) {
    const int r = r0 + k, c = c0 + tx;
    if (r < rows && c < cols) t[k][tx] = in[z * n + (long long)r * cols + c];
  }
  __syncthreads();
  for (int k = ty; k < 32; k += 8) {
    const int c = c0 + k, r = r0 + tx;   // out [cols, rows]
    if (r < rows && c < cols) out[z * n + (long long)c * rows + r] = t[tx][k];
  }
}

// out[z] = sum_{i < n_in} in[i * Z + z]^T for Z matrices [rows, cols] per input (the same
// tiling as transpose_kernel); grid (ceil(cols/32), ceil(rows/32), Z).
__global__ void transpose_sum_kernel(const float* in, int n_in, float* out, int rows, int cols) {
  __shared__ float t[32][33];
  const long long z = blockIdx.z, Z = gridDim.z, n = (long long)rows * cols;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32, tx = threadIdx.x, ty = threadIdx.y;
  for (int k = ty; k < 32; k += 8) {
    const int r = r0 + k, c = c0 + tx;
    if (r < rows && c < cols) {
      float acc = 0.0f;
      for (int i = 0; i < n_in; ++i) acc += in[((long long)i * Z + z) * n + (long long)r * cols + c];
      t[k][tx] = acc;
    }
  }
  __syncthreads();
  for (int k = ty; k < 32; k += 8) {
    const int c = c0 + k, r = r0 + tx;   // out [cols, rows]
    if (r < rows && c < cols) out[z * n + (long long)c * rows + r] = t[tx][k];
  }
}

// ------------------------------------------------------------------ backward helpers
template <typename OT>
__global__ void suffix_scan_kernel(const float* dSc, const float* dS_final, OT* G, float* R0,
                                   int BH, int C, long long n, int order) {
  TTT_GRID_LOOP(idx, (long long)BH * n) {
    const long long bh = idx / n, e = idx - bh * n;
    float r = dS_final ? dS_final[idx] : 0.0f;
    for (int c = C - 1; c >= 0; --c) {
      const long long o = (bh * C + c) * n + e;
      if (order == 1) G[o] = from_f32<OT>(r);
      r += dSc[o];
      if (order != 1) G[o] = from_f32<OT>(r);
    }
    R0[idx] = r;
  }
}

// The same with 4 elements per thread (16-byte loads of dSc, eight chunks' loads issued
// together; n a multiple of 4, 16-byte aligned buffers).
template <typename OT>
__global__ void suffix_scan4_kernel(const float4* dSc, const float4* dS_final, OT* G, float4* R0,
                                    int BH, int C, long long n4, int order) {
  TTT_GRID_LOOP(idx, (long long)BH * n4) {
    const long long bh = idx / n4, e = idx - bh * n4;
    float4 r = dS_final ? dS_final[idx] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    auto put = [&](long long o, const float4& x) {
      OT* g = G + o * 4;
      g[0] = from_f32<OT>(x.x); g[1] = from_f32<OT>(x.y);
      g[2] = from_f32<OT>(x.z); g[3] = from_f32<OT>(x.w);
    };
    for (int c0 = C - 1; c0 >= 0; c0 -= 8) {
      float4 x[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (c0 - k >= 0) x[k] = dSc[(bh * C + c0 - k) * n4 + e];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (c0 - k < 0) break;
        const long long o = (bh * C + c0 - k) * n4 + e;
        if (order == 1) put(o, r);
        r.x += x[k].x; r.y += x[k].y; r.z += x[k].z; r.w += x[k].w;
        if (order != 1) put(o, r);
      }
    }
    R0[idx] = r;
  }
}

// one warp per row
template <typename OT>
__global__ void row_grads_kernel(const float* T, const OT* v, const float* eta, float sgn,
                                 OT* dv, float* deta, long long rows, int w) {
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    const int lane = threadIdx.x & 31;
    const float se = sgn * eta[r];
    float acc = 0.0f;
    for (int j = lane; j < w; j += 32) {
      const float t = T[r * w + j];
      acc = fmaf(t, to_f32(v[r * w + j]), acc);
      dv[r * w + j] = from_f32<OT>(se * t);
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) deta[r] = sgn * acc;
  }
}

// The same for bf16 v / dv with w a multiple of 8: each lane moves 8 elements per step (two
// 16-byte loads of T, one of v, one 16-byte store of dv).
__global__ void row_grads8_kernel(const float4* T, const uint4* v, const float* eta, float sgn,
                                  uint4* dv, float* deta, long long rows, int w8) {
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    const int lane = threadIdx.x & 31;
    const float se = sgn * eta[r];
    float acc = 0.0f;
    for (int j = lane; j < w8; j += 32) {
      const float4 t0 = T[(r * w8 + j) * 2], t1 = T[(r * w8 + j) * 2 + 1];
      const uint4 vv = v[r * w8 + j];
      const __nv_bfloat162* vb = reinterpret_cast<const __nv_bfloat162*>(&vv);
      const float2 v0 = __bfloat1622float2(vb[0]), v1 = __bfloat1622float2(vb[1]);
      const float2 v2 = __bfloat1622float2(vb[2]), v3 = __bfloat1622float2(vb[3]);
      acc = fmaf(t0.x, v0.x, acc); acc = fmaf(t0.y, v0.y, acc);
      acc = fmaf(t0.z, v1.x, acc); acc = fmaf(t0.w, v1.y, acc);
      acc = fmaf(t1.x, v2.x, acc); acc = fmaf(t1.y, v2.y, acc);
      acc = fmaf(t1.z, v3.x, acc); acc = fmaf(t1.w, v3.y, acc);
      uint4 o;
      const __nv_bfloat162 o0 = __floats2bfloat162_rn(se * t0.x, se * t0.y);
      const __nv_bfloat162 o1 = __floats2bfloat162_rn(se * t0.z, se * t0.w);
      const __nv_bfloat162 o2 = __floats2bfloat162_rn(se * t1.x, se * t1.y);
      const __nv_bfloat162 o3 = __floats2bfloat162_rn(se * t1.z, se * t1.w);
      o.x = *reinterpret_cast<const uint32_t*>(&o0); o.y = *reinterpret_cast<const uint32_t*>(&o1);
      o.z = *reinterpret_cast<const uint32_t*>(&o2); o.w = *reinterpret_cast<const uint32_t*>(&o3);
      dv[r * w8 + j] = o;
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) deta[r] = sgn * acc;
  }
}

__global__ void sum_batches4_kernel(const float4* X, int B, long long stride4, long long n4,
                                    float4* out) {
  TTT_GRID_LOOP(i, n4) {
    float4 acc = X[i];
    for (int b = 1; b < B; ++b) {
      const float4 x = X[b * stride4 + i];
      acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
    }
    out[i] = acc;
  }
}

__global__ void sum_batches_kernel(const float* X, int B, long long stride, long long n,
                                   float* out) {
  TTT_GRID_LOOP(i, n) {
    float acc = 0.0f;
    for (int b = 0; b < B; ++b) acc += X[b * stride + i];
    out[i] = acc;
  }
}

template <typename OT>
__global__ void cast_kernel(const float* X, OT* out, long long n) {
  TTT_GRID_LOOP(i, n) out[i] = from_f32<OT>(X[i]);
}

template <typename OT>
__global__ void cat_cols_kernel(const float* A, const float* B, OT* out, long long rows, int w) {
  TTT_GRID_LOOP(i, rows * 2 * w) {
    const long long r = i / (2 * w);
    const int c = (int)(i - r * 2 * w);
    out[i] = from_f32<OT>(c < w ? A[r * w + c] : B[r * w + c - w]);
  }
}

__global__ void sum_split_cols_kernel(const float* X, int nb, long long rows, int w,
                                      float* out0, float* out1) {
  TTT_GRID_LOOP(i, rows * 2 * w) {
    const long long r = i / (2 * w);
    const int c = (int)(i - r * 2 * w);
    float acc = 0.0f;
    for (int b = 0; b < nb; ++b) acc += X[(long long)b * rows * 2 * w + i];
    if (c < w) out0[r * w + c] = acc;
    else out1[r * w + c - w] = acc;
  }
}

// One thread per 4 elements, chunks in order; the loads of eight chunks are issued
// together before their updates (the chunk axis is short, the values are independent).
// With nrm, the sum of squares of every (b, head, chunk) matrix M_c is accumulated into
// nrm[bh * C + c] (block sums, one atomic add per block and chunk; n4 a multiple of the
// block size, so a block never spans two (b, head) entries).
__global__ void momentum_scan4_kernel(float4* D, const float* alpha, int BH, int C,
                                      long long n4, float* nrm) {
  __shared__ float red[8];
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)BH * n4) return;
  const long long bh = idx / n4, e = idx - bh * n4;
  float4* d = D + bh * C * n4 + e;
  auto block_sum = [&](float v, int c) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
      float t = 0.0f;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
      atomicAdd(&nrm[bh * C + c], t);
    }
    __syncthreads();
  };
  float4 mv = d[0];
  if (nrm) block_sum(mv.x * mv.x + mv.y * mv.y + mv.z * mv.z + mv.w * mv.w, 0);
  for (int c0 = 1; c0 < C; c0 += 8) {
    float4 x[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (c0 + k < C) x[k] = d[(long long)(c0 + k) * n4];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (c0 + k >= C) break;
      const float a = alpha[bh * C + c0 + k];
      mv.x = fmaf(a, mv.x, x[k].x); mv.y = fmaf(a, mv.y, x[k].y);
      mv.z = fmaf(a, mv.z, x[k].z); mv.w = fmaf(a, mv.w, x[k].w);
      d[(long long)(c0 + k) * n4] = mv;
      if (nrm) block_sum(mv.x * mv.x + mv.y * mv.y + mv.z * mv.z + mv.w * mv.w, c0 + k);
    }
  }
}

// One thread per element, chunks in order (the chunk axis is short).
__global__ void momentum_scan_kernel(float* D, const float* alpha, int BH, int C, long long n) {
  TTT_GRID_LOOP(idx, (long long)BH * n) {
    const long long bh = idx / n, e = idx - bh * n;
    float* d = D + bh * C * n + e;
    float mv = d[0];
    for (int c = 1; c < C; ++c) {
      mv = fmaf(alpha[bh * C + c], mv, d[(long long)c * n]);
      d[(long long)c * n] = mv;
    }
  }
}

// One warp per row of the output-major state (one output unit of a fast matrix, over its
// input dimension): the update u = U (Newton-Schulz path) or the sum of the split-K partial
// gradients with the momentum M <- alpha M + g folded in (written back); w <- w - sign u;
// with renormalisation the row's norm is reduced across the warp and the row rescaled to
// the initial column norm; the fp32 master and the bf16 / fp32 operand copy are written
// (W1 rows to W1t [h, m], W0 / W2 rows to their rows of the blocked operand Wk, W0 halved).
// Rows per (b, head): m of W0^T (length h), h of W1^T (length m), m of W2^T (length h).
// VEC: rows in 16-byte vectors (h, m multiples of 4); NV: the most vectors (elements without
// VEC) a lane holds, ceil(max(h, m) / 128) (/ 32).
template <typename OT, bool VEC, int NV>
__global__ void __launch_bounds__(256) rec_step_rows_kernel(float* W_all, const float* U, const float* partials,
                                     int splits, float* M_all, const float* alpha, int C, int c,
                                     const float* tnorm, int BH, int H, int h, int m, int mask,
                                     int sign, int renorm, OT* Wk, OT* W1t) {
  const long long rows_bh = 2LL * m + h, rows = rows_bh * BH;
  const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= rows) return;
  const int bh = (int)(wid / rows_bh);
  int r = (int)(wid - (long long)bh * rows_bh), p = 0;
  if (r >= m + h) { p = 2; r -= m + h; } else if (r >= m) { p = 1; r -= m; }
  if (!(mask & (1 << p))) return;
  const int len = p == 1 ? m : h;
  const long long hm = (long long)h * m;
  const long long off = (long long)bh * 3 * hm + p * hm + (long long)r * len;
  const long long poff = off + (partial_part(p) - p) * hm;   // the row in the partials
  const long long pstride = (long long)BH * 3 * hm;
  const float sg = (float)sign;
  const float a = (M_all && !U) ? alpha[(long long)bh * C + c] : 0.0f;
  constexpr int MAXV = NV;
  float v[VEC ? MAXV * 4 : MAXV];
  float ss = 0.0f;
  const int n = VEC ? len / 4 : len;
  if constexpr (VEC) {
    // every 16-byte load of the row first (predicated, no early exit), so all of a lane's
    // loads are in flight together; then the update
    float4 wv[MAXV], uv[MAXV];
    const float4 z4 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    const float4* usrc = reinterpret_cast<const float4*>(U ? U + off : partials + poff);
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int q = lane + 32 * i;
      wv[i] = q < n ? reinterpret_cast<const float4*>(W_all + off)[q] : z4;
      uv[i] = q < n ? usrc[q] : z4;
    }
    if (!U) {
      for (int s2 = 1; s2 < splits; ++s2) {
        const float4* src = reinterpret_cast<const float4*>(partials + s2 * pstride + poff);
        float4 xv[MAXV];
#pragma unroll
        for (int i = 0; i < MAXV; ++i) xv[i] = lane + 32 * i < n ? src[lane + 32 * i] : z4;
#pragma unroll
        for (int i = 0; i < MAXV; ++i) {
          uv[i].x += xv[i].x; uv[i].y += xv[i].y; uv[i].z += xv[i].z; uv[i].w += xv[i].w;
        }
      }
      if (M_all) {
        float4 mv[MAXV];
#pragma unroll
        for (int i = 0; i < MAXV; ++i)
          mv[i] = lane + 32 * i < n ? reinterpret_cast<float4*>(M_all + off)[lane + 32 * i] : z4;
#pragma unroll
        for (int i = 0; i < MAXV; ++i) {
          const int q = lane + 32 * i;
          if (q >= n) break;
          mv[i].x = fmaf(a, mv[i].x, uv[i].x); mv[i].y = fmaf(a, mv[i].y, uv[i].y);
          mv[i].z = fmaf(a, mv[i].z, uv[i].z); mv[i].w = fmaf(a, mv[i].w, uv[i].w);
          reinterpret_cast<float4*>(M_all + off)[q] = mv[i];
          uv[i] = mv[i];
        }
      }
    }
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      v[4 * i] = wv[i].x - sg * uv[i].x; v[4 * i + 1] = wv[i].y - sg * uv[i].y;
      v[4 * i + 2] = wv[i].z - sg * uv[i].z; v[4 * i + 3] = wv[i].w - sg * uv[i].w;
      if (lane + 32 * i < n) {
        ss = fmaf(v[4 * i], v[4 * i], ss); ss = fmaf(v[4 * i + 1], v[4 * i + 1], ss);
        ss = fmaf(v[4 * i + 2], v[4 * i + 2], ss); ss = fmaf(v[4 * i + 3], v[4 * i + 3], ss);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int q = lane + 32 * i;
    if (q >= n) break;
    if constexpr (VEC) {
      break;   // done above
    } else {
      float u;
      if (U) {
        u = U[off + q];
      } else {
        u = partials[poff + q];
        for (int s2 = 1; s2 < splits; ++s2) u += partials[s2 * pstride + poff + q];
        if (M_all) {
          const float mv = fmaf(a, M_all[off + q], u);
          M_all[off + q] = mv;
          u = mv;
        }
      }
      v[i] = W_all[off + q] - sg * u;
      ss = fmaf(v[i], v[i], ss);
    }
  }
  float scale = 1.0f;
  if (renorm) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float* tn = tnorm + (long long)(bh % H) * (2 * m + h) + (p == 0 ? 0 : p == 1 ? m : m + h);
    scale = tn[r] / sqrtf(ss);
  }
  const int mpad = (m + 127) / 128 * 128;
  OT* orow = p == 1 ? W1t + (long long)bh * hm + (long long)r * len
                    : Wk + ((long long)bh * 2 * mpad + (r >> 7) * 256 + (p == 2 ? 128 : 0) +
                            (r & 127)) * h;
  const float f = p == 0 ? 0.5f : 1.0f;   // the blocked operand holds W0 / 2
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int q = lane + 32 * i;
    if (q >= n) break;
    if constexpr (VEC) {
      const float4 w = make_float4(v[4 * i] * scale, v[4 * i + 1] * scale, v[4 * i + 2] * scale,
                                   v[4 * i + 3] * scale);
      reinterpret_cast<float4*>(W_all + off)[q] = w;
      if constexpr (sizeof(OT) == 2) {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(f * w.x, f * w.y);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(f * w.z, f * w.w);
        uint2 pk;
        pk.x = *reinterpret_cast<const uint32_t*>(&lo);
        pk.y = *reinterpret_cast<const uint32_t*>(&hi);
        reinterpret_cast<uint2*>(orow)[q] = pk;
      } else {
        reinterpret_cast<float4*>(orow)[q] = make_float4(f * w.x, f * w.y, f * w.z, f * w.w);
      }
    } else {
      const float w = v[i] * scale;
      W_all[off + q] = w;
      orow[q] = from_f32<OT>(f * w);
    }
  }
}

// ------------------------------------------------------------------ In-Place target conv
__global__ void conv4_kernel(const bf16* X0, const float* w, bf16* Xc, int N, int d) {
  TTT_GRID_LOOP(idx, (long long)N * d) {
    const long long t = idx / d;
    const int i = (int)(idx - t * d);
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (t - j >= 0) acc += w[j * d + i] * __bfloat162float(X0[(t - j) * d + i]);
    Xc[idx] = __float2bfloat16_rn(acc);
  }
}

// 16-byte version: a thread owns 8 channels over a run of CONV_RUN tokens and slides a
// window of the last three input rows through registers, so every input row is read once
// per run (plus a three-row halo) and every load and store is a coalesced 16-byte access.
// grid (ceil(d / 8 / 128), ceil(N / CONV_RUN)), block 128. Needs d % 8 == 0 and 16-byte
// aligned X0 / Xc.
constexpr int CONV_RUN = 32;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 v = __bfloat1622float2(h[q]);
    f[2 * q] = v.x;
    f[2 * q + 1] = v.y;
  }
}

__global__ void __launch_bounds__(128) conv4_vec_kernel(const bf16* X0, const float* w, bf16* Xc,
                                                        int N, int d) {
  const int g = blockIdx.x * 128 + threadIdx.x;   // channel group
  if (g * 8 >= d) return;
  const int c = g * 8;
  const long long t0 = (long long)blockIdx.y * CONV_RUN;
  float wt[4][8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 a = *reinterpret_cast<const float4*>(w + (long long)j * d + c);
    const float4 b = *reinterpret_cast<const float4*>(w + (long long)j * d + c + 4);
    wt[j][0] = a.x; wt[j][1] = a.y; wt[j][2] = a.z; wt[j][3] = a.w;
    wt[j][4] = b.x; wt[j][5] = b.y; wt[j][6] = b.z; wt[j][7] = b.w;
  }
  float win[3][8];   // win[j - 1] = X0[t - j]
#pragma unroll
  for (int j = 1; j <= 3; ++j) {
    const long long t = t0 - j;
    if (t >= 0) {
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(X0 + t * d + c), win[j - 1]);
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) win[j - 1][q] = 0.0f;
    }
  }
  const long long t_end = min((long long)N, t0 + CONV_RUN);
  for (long long t = t0; t < t_end; ++t) {
    float x[8];
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(X0 + t * d + c), x);
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 8; q += 2) {
      float r[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int k = q + u;
        r[u] = wt[0][k] * x[k] + wt[1][k] * win[0][k] + wt[2][k] * win[1][k] +
               wt[3][k] * win[2][k];
      }
      const __nv_bfloat162 pk = __floats2bfloat162_rn(r[0], r[1]);
      o[q / 2] = *reinterpret_cast<const uint32_t*>(&pk);
    }
    *reinterpret_cast<uint4*>(Xc + t * d + c) = make_uint4(o[0], o[1], o[2], o[3]);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      win[2][q] = win[1][q];
      win[1][q] = win[0][q];
      win[0][q] = x[q];
    }
  }
}

// ------------------------------------------------------------------ diagnostics
__global__ void wait_timeout_kernel(unsigned* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    umma::mbar_init(umma::smem_u32(&bar), 1);
    umma::mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nobody arrives on `bar`: the wait must run out and report it.
    umma::mbar_wait(umma::smem_u32(&bar), 0, &abort_flag, err, limit_ns);
  }
  __syncthreads();
}

__global__ void fill_kernel(float* p, long long n, float v) {
  TTT_GRID_LOOP(i, n) p[i] = v;
}

template <typename F>
cudaError_t by_ot(int ot, F&& f) {
  if (ot == DT_BF16) return f(bf16{});
  return f(float{});
}

}  // namespace

cudaError_t prep_wk_blocked(int ot, const float* W0, const float* W2, void* Wk, int n_entries,
                            int src_heads, int h, int m, int src_layout, cudaStream_t s,
                            void* Wk1, void* Wk2) {
  return by_ot(ot, [&](auto tag) {
    using OT = decltype(tag);
    const int mpad = (m + 127) / 128 * 128;
    dim3 grid(mpad / 32, (h + 31) / 32, 2 * n_entries);
    prep_wk_blocked_kernel<OT><<<grid, dim3(32, 8), 0, s>>>(
        W0, W2, static_cast<OT*>(Wk), static_cast<OT*>(Wk1), static_cast<OT*>(Wk2), src_heads,
        h, m, src_layout);
    return cudaGetLastError();
  });
}

cudaError_t scale_rows(int ot, const void* X, const float* eta, void* Xs, long long rows, int w,
                       cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const bool vec = ot == DT_BF16 && w % 8 == 0 &&
                   ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(Xs)) & 15) == 0;
  if (vec) {
    scale_rows8_kernel<<<grid_for(rows * (w / 8), 256), 256, 0, s>>>(
        static_cast<const uint4*>(X), eta, static_cast<uint4*>(Xs), rows, w / 8);
    return cudaGetLastError();
  }
  return by_ot(ot, [&](auto tag) {
    using OT = decltype(tag);
    scale_rows_kernel<OT><<<grid_for(rows * w, 256), 256, 0, s>>>(
        static_cast<const OT*>(X), eta, static_cast<OT*>(Xs), rows, w);
    return cudaGetLastError();
  });
}

cudaError_t chunk_scan(int ot, const float* dS, const float* W1, const float* prior, int n_prior,
                       void* Sc, float* S_final, int BH, int H, int C, int m, int h, int order,
                       int layout, float* scratch, cudaStream_t s) {
  const long long per = (long long)m * h;
  if (layout == 1 && scratch) {
    // transposed W1 / S_final: transpose once on each side and scan in the [m, h] layout;
    // the prior states (W1's layout) are summed and transposed into the region of the
    // transposed final state (each element is read there before the scan writes it)
    float* W1t = W1 ? scratch : nullptr;
    float* Sft = scratch + (long long)H * per;
    if (W1)
      transpose_kernel<<<dim3((m + 31) / 32, (h + 31) / 32, H), dim3(32, 8), 0, s>>>(W1, W1t, h,
                                                                                    m);
    if (n_prior > 0)
      transpose_sum_kernel<<<dim3((m + 31) / 32, (h + 31) / 32, BH), dim3(32, 8), 0, s>>>(
          prior, n_prior, Sft, h, m);
    cudaError_t e = chunk_scan(ot, dS, W1t, n_prior > 0 ? Sft : nullptr, n_prior > 0 ? 1 : 0, Sc,
                               S_final ? Sft : nullptr, BH, H, C, m, h, order, 0, nullptr, s);
    if (e != cudaSuccess || !S_final) return e;
    transpose_kernel<<<dim3((h + 31) / 32, (m + 31) / 32, BH), dim3(32, 8), 0, s>>>(Sft, S_final,
                                                                                  m, h);
    return cudaGetLastError();
  }
  const bool vec = layout == 0 && per % 4 == 0 &&
                   ((reinterpret_cast<uintptr_t>(dS) | reinterpret_cast<uintptr_t>(W1) |
                     reinterpret_cast<uintptr_t>(prior) | reinterpret_cast<uintptr_t>(Sc) |
                     reinterpret_cast<uintptr_t>(S_final)) & 15) == 0;
  return by_ot(ot, [&](auto tag) {
    using OT = decltype(tag);
    if (vec) {
      const long long n4 = per / 4 * BH;
      chunk_scan4_kernel<OT><<<grid_for(n4, 256, 148 * 16), 256, 0, s>>>(
          reinterpret_cast<const float4*>(dS), reinterpret_cast<const float4*>(W1),
          reinterpret_cast<const float4*>(prior), n_prior, static_cast<OT*>(Sc),
          reinterpret_cast<float4*>(S_final), BH, H, C, per / 4, order);
    } else {
      chunk_scan_kernel<OT><<<grid_for(per * BH, 256, 148 * 64), 256, 0, s>>>(
          dS, W1, prior, n_prior, static_cast<OT*>(Sc), S_final, BH, H, C, m, h, order, layout);
    }
    return cudaGetLastError();
  });
}

cudaError_t rec_init(int ot, const float* W0, const float* W2, const float* W1, int BH, int H,
                     int h, int m, float* W_all, void* W1t, const float* M_in, float* M_all,
                     int momentum, cudaStream_t s, void* W1t1, void* W1t2) {
  return by_ot(ot, [&](auto tag) {
    using OT = decltype(tag);
    const int tiles = ((h + 31) / 32) * ((m + 31) / 32);
    rec_transpose_kernel<OT><<<dim3(tiles, 3, BH), dim3(32, 8), 0, s>>>(
        0, W0, W2, W1, H, h, m, W_all, static_cast<OT*>(W1t), static_cast<OT*>(W1t1),
        static_cast<OT*>(W1t2), M_in, M_all, momentum, nullptr, nullptr, nullptr, nullptr);
    return cudaGetLastError();
  });
}

cudaError_t col_norms(const float* W0, const float* W2, const float* W1, int H, int h, int m,
                      float* tnorm, cudaStream_t s) {
  if (H <= 0) return cudaSuccess;
  col_norms_kernel<<<dim3((2 * m + h + 31) / 32, H), dim3(32, 8), 0, s>>>(W0, W2, W1, H, h, m,
                                                                          tnorm);
  return cudaGetLastError();
}

cudaError_t rec_reduce(const float* partials, int splits, float* U, float* M_all,
                       const float* alpha, int C, int c, int BH, int h, int m, int mask,
                       cudaStream_t s) {
  const long long hm = (long long)h * m, n = 3 * hm * BH;
  const bool vec = hm % 4 == 0 &&
                   ((reinterpret_cast<uintptr_t>(partials) | reinterpret_cast<uintptr_t>(U) |
                     reinterpret_cast<uintptr_t>(M_all)) & 15) == 0;
  if (vec) {
    rec_reduce4_kernel<<<grid_for(n / 4, 256), 256, 0, s>>>(
        reinterpret_cast<const float4*>(partials), splits, reinterpret_cast<float4*>(U),
        reinterpret_cast<float4*>(M_all), alpha, C, c, BH, hm / 4, mask);
  } else {
    rec_reduce_kernel<<<grid_for(n, 256), 256, 0, s>>>(partials, splits, U, M_all, alpha, C, c,
                                                       BH, h, m, mask);
  }
  return cudaGetLastError();
}

cudaError_t ns_sumsq(const float* U, int Z, const NsLayout& L, float* nrm, cudaStream_t s) {
  if (Z <= 0) return cudaSuccess;
  cudaError_t e = fill_f32(nrm, (long long)Z * L.parts, 0.0f, s);
  if (e != cudaSuccess) return e;
  ns_sumsq_kernel<<<dim3(L.parts, Z, NS_SLABS), 256, 0, s>>>(U, L, nrm);
  return cudaGetLastError();
}

cudaError_t ns_normalize(const float* U, float* X, int Z, const NsLayout& L, float eps,
                         float* nrm, cudaStream_t s, float* Xt, bool nrm_ready) {
  if (Z <= 0) return cudaSuccess;
  if (!nrm_ready) {
    cudaError_t e = ns_sumsq(U, Z, L, nrm, s);
    if (e != cudaSuccess) return e;
  }
  int tiles = 0;
  for (int p = 0; p < L.parts; ++p)
    tiles = max(tiles, ((L.R[p] + 31) / 32) * ((L.C[p] + 31) / 32));
  bool vec = ((reinterpret_cast<uintptr_t>(U) | reinterpret_cast<uintptr_t>(X) |
               reinterpret_cast<uintptr_t>(Xt)) & 15) == 0 &&
             L.zstride % 4 == 0 && L.pstride % 4 == 0;
  for (int p = 0; p < L.parts; ++p) vec = vec && L.R[p] % 4 == 0 && L.C[p] % 4 == 0;
  if (vec)
    ns_norm4_kernel<<<dim3(tiles, L.parts, Z), 256, 0, s>>>(U, X, Xt, L, nrm, eps);
  else
    ns_copy_kernel<<<dim3(tiles, L.parts, Z), dim3(32, 8), 0, s>>>(U, X, nullptr, L, nrm, eps, 0,
                                                                   Xt);
  return cudaGetLastError();
}

cudaError_t ns_writeback(const float* X, float* U, int Z, const NsLayout& L, cudaStream_t s) {
  if (Z <= 0) return cudaSuccess;
  int tiles = 0;
  for (int p = 0; p < L.parts; ++p)
    tiles = max(tiles, ((L.R[p] + 31) / 32) * ((L.C[p] + 31) / 32));
  ns_copy_kernel<<<dim3(tiles, L.parts, Z), dim3(32, 8), 0, s>>>(
      nullptr, const_cast<float*>(X), U, L, nullptr, 0.0f, 1, nullptr);
  return cudaGetLastError();
}



cudaError_t suffix_scan(int ot, const float* dSc, const float* dS_final, void* G, float* R0,
                        int BH, int C, long long n, int order, cudaStream_t s) {
  if (BH <= 0 || n <= 0) return cudaSuccess;
  const bool vec = n % 4 == 0 &&
                   ((reinterpret_cast<uintptr_t>(dSc) | reinterpret_cast<uintptr_t>(dS_final) |
                     reinterpret_cast<uintptr_t>(R0)) & 15) == 0;
  return by_ot(ot, [&](auto tag) {
    using OT = decltype(tag);
    if (vec)
      suffix_scan4_kernel<OT><<<grid_for((long long)BH * n / 4, 256), 256, 0, s>>>(
          reinterpret_cast<const float4*>(dSc), reinterpret_cast<const float4*>(dS_final),
          static_cast<OT*>(G), reinterpret_cast<float4*>(R0), BH, C, n / 4, order);
    else
      suffix_scan_kernel<OT><<<grid_for((long long)BH * n, 256), 256, 0, s>>>(
          dSc, dS_final, static_cast<OT*>(G), R0, BH, C, n, order);
    return cudaGetLastError();
  });
}

cudaError_t row_grads(int ot, const float* T, const void* v, const float* eta, int sign,
                      void* dv, float* deta, long long rows, int w, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const long long blocks = (rows + 7) / 8;
  const unsigned grid = (unsigned)(blocks < 148 * 32 ? blocks : 148 * 32);
  if (ot == DT_BF16 && w % 8 == 0 &&
      ((reinterpret_cast<uintptr_t>(T) | reinterpret_cast<uintptr_t>(v) |
        reinterpret_cast<uintptr_t>(dv)) & 15) == 0) {
    row_grads8_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(T),
                                           static_cast<const uint4*>(v), eta, (float)sign,
                                           static_cast<uint4*>(dv), deta, rows, w / 8);
    return cudaGetLastError();
  }
  return by_ot(ot, [&](auto tag) {
    using OT = decltype(tag);
    row_grads_kernel<OT><<<grid, 256, 0, s>>>(T, static_cast<const OT*>(v), eta, (float)sign,
                                              static_cast<OT*>(dv), deta, rows, w);
    return cudaGetLastError();
  });
}

cudaError_t sum_batches(const float* X, int B, long long stride, long long n, float* out,
                        cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  if (B >= 1 && n % 4 == 0 && stride % 4 == 0 &&
      ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(out)) & 15) == 0)
    sum_batches4_kernel<<<grid_for(n / 4, 256), 256, 0, s>>>(
        reinterpret_cast<const float4*>(X), B, stride / 4, n / 4, reinterpret_cast<float4*>(out));
  else
    sum_batches_kernel<<<grid_for(n, 256), 256, 0, s>>>(X, B, stride, n, out);
  return cudaGetLastError();
}

cudaError_t cast_to(int ot, const float* X, void* out, long long n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  return by_ot(ot, [&](auto tag) {
    using OT = decltype(tag);
    cast_kernel<OT><<<grid_for(n, 256), 256, 0, s>>>(X, static_cast<OT*>(out), n);
    return cudaGetLastError();
  });
}

cudaError_t cat_cols(int ot, const float* A, const float* B, void* out, long long rows, int w,
                     cudaStream_t s) {
  if (rows <= 0 || w <= 0) return cudaSuccess;
  return by_ot(ot, [&](auto tag) {
    using OT = decltype(tag);
    cat_cols_kernel<OT><<<grid_for(rows * 2 * w, 256), 256, 0, s>>>(A, B, static_cast<OT*>(out),
                                                                   rows, w);
    return cudaGetLastError();
  });
}

cudaError_t sum_split_cols(const float* X, int nb, long long rows, int w, float* out0,
                           float* out1, cudaStream_t s) {
  if (rows <= 0 || w <= 0) return cudaSuccess;
  sum_split_cols_kernel<<<grid_for(rows * 2 * w, 256), 256, 0, s>>>(X, nb, rows, w, out0, out1);
  return cudaGetLastError();
}

bool momentum_scan_norms(int C, long long n, const float* D) {
  return C > 1 && n % 1024 == 0 && (reinterpret_cast<uintptr_t>(D) & 15) == 0;
}

cudaError_t momentum_scan(float* D, const float* alpha, int BH, int C, long long n,
                          cudaStream_t s, float* nrm) {
  if (BH <= 0 || C <= 1 || n <= 0) return cudaSuccess;
  if (nrm && !momentum_scan_norms(C, n, D)) return cudaErrorInvalidValue;
  if (nrm) {
    cudaError_t e = fill_f32(nrm, (long long)BH * C, 0.0f, s);
    if (e != cudaSuccess) return e;
  }
  if (n % 4 == 0 && (reinterpret_cast<uintptr_t>(D) & 15) == 0)
    momentum_scan4_kernel<<<(unsigned)(((long long)BH * n / 4 + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<float4*>(D), alpha, BH, C, n / 4, nrm);
  else
    momentum_scan_kernel<<<grid_for((long long)BH * n, 256), 256, 0, s>>>(D, alpha, BH, C, n);
  return cudaGetLastError();
}

cudaError_t rec_step(float* W_all, const float* U, const float* partials, int splits,
                     float* M_all, const float* alpha, int C, int c, const float* tnorm, int BH,
                     int H, int h, int m, int mask, int sign, int renorm, void* Wk, void* W1t,
                     int ot, cudaStream_t s) {
  return by_ot(ot, [&](auto tag) {
    using OT = decltype(tag);
    const long long rows = (2LL * m + h) * BH;
    const unsigned grid = (unsigned)((rows * 32 + 255) / 256);
    const bool vec = h % 4 == 0 && m % 4 == 0;
    const int len = h > m ? h : m;
    auto go = [&](auto kern) {
      kern<<<grid, 256, 0, s>>>(W_all, U, partials, splits, M_all, alpha, C, c, tnorm, BH, H, h,
                                m, mask, sign, renorm, static_cast<OT*>(Wk),
                                static_cast<OT*>(W1t));
    };
    if (vec && len <= 256) go(rec_step_rows_kernel<OT, true, 2>);
    else if (vec && len <= 512) go(rec_step_rows_kernel<OT, true, 4>);
    else if (vec) go(rec_step_rows_kernel<OT, true, 12>);
    else if (len <= 128) go(rec_step_rows_kernel<OT, false, 4>);
    else go(rec_step_rows_kernel<OT, false, 48>);
    return cudaGetLastError();
  });
}

cudaError_t rec_finish(const float* W_all, int BH, int H, int h, int m, float* W0_out,
                       float* W2_out, float* W1_out, const float* M_all, float* M_out,
                       cudaStream_t s) {
  const int tiles = ((h + 31) / 32) * ((m + 31) / 32);
  rec_transpose_kernel<float><<<dim3(tiles, 3, BH), dim3(32, 8), 0, s>>>(
      1, nullptr, nullptr, nullptr, H, h, m, const_cast<float*>(W_all), nullptr, nullptr,
      nullptr, nullptr, const_cast<float*>(M_all), 0, W0_out, W2_out, W1_out, M_out);
  return cudaGetLastError();
}

cudaError_t conv4_causal(const void* X0, const float* conv_w, void* Xc, int N, int d,
                         cudaStream_t s) {
  const bool vec = d % 8 == 0 && ((reinterpret_cast<uintptr_t>(X0) | reinterpret_cast<uintptr_t>(Xc) |
                                    reinterpret_cast<uintptr_t>(conv_w)) & 15) == 0 &&
                   (N + CONV_RUN - 1) / CONV_RUN <= 65535;
  if (vec) {
    const dim3 grid((unsigned)((d / 8 + 127) / 128), (unsigned)((N + CONV_RUN - 1) / CONV_RUN));
    conv4_vec_kernel<<<grid, 128, 0, s>>>(static_cast<const bf16*>(X0), conv_w,
                                          static_cast<bf16*>(Xc), N, d);
  } else {
    conv4_kernel<<<grid_for((long long)N * d, 256), 256, 0, s>>>(
        static_cast<const bf16*>(X0), conv_w, static_cast<bf16*>(Xc), N, d);
  }
  return cudaGetLastError();
}

cudaError_t wait_timeout_probe(unsigned* err, unsigned long long limit_ns, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(err, limit_ns);
  return cudaGetLastError();
}

cudaError_t fill_f32(float* p, long long n, float v, cudaStream_t s) {
  fill_kernel<<<grid_for(n, 256), 256, 0, s>>>(p, n, v);
  return cudaGetLastError();
}

cudaError_t seq_init(const float* W1, const float* prior, int n_prior, int BH, int H, long long n,
                     float* master, void* shadow, cudaStream_t s) {
  if (BH <= 0 || n <= 0) return cudaSuccess;
  seq_init_kernel<<<grid_for((long long)BH * n, 256), 256, 0, s>>>(
      W1, prior, n_prior, BH, H, n, master, static_cast<__nv_bfloat16*>(shadow));
  return cudaGetLastError();
}

}  // namespace ttt
