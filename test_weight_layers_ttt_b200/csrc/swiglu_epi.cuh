// SwiGLU epilogue math shared by the tensor-core kernels: the accumulator halves hold
// h = A/2 (the input-side operand carries W0 / 2) and B, and
// silu(A) B = A sigmoid(A) B = h (1 + tanh(h)) B.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace ttt {
namespace umma {

__device__ __forceinline__ float tanh_fast(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(x));
  return t;
}

// Two SwiGLU outputs from the half pre-activations h = A/2 (the operand holds W0 / 2) and
// B: silu(A) B = A sigmoid(A) B = h (1 + tanh(h)) B, so with p = h B the result is
// p + p tanh(h); `s` scales it (the row's eta, or 1). One MUFU tanh.approx per element
// (relative error about 2^-11, below the bf16 rounding of the result) and the rest as
// packed fp32x2 multiplies / fma.
__device__ __forceinline__ void swiglu2(uint32_t h0, uint32_t h1, uint32_t b0, uint32_t b1,
                                        float s, float& o0, float& o1) {
  const float t0 = tanh_fast(__uint_as_float(h0)), t1 = tanh_fast(__uint_as_float(h1));
  asm("{\n\t.reg .b64 H, B, P, T, S;\n\t"
      "mov.b64 H, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "mov.b64 T, {%6, %7};\n\tmov.b64 S, {%8, %9};\n\t"
      "mul.rn.f32x2 P, H, B;\n\tmul.rn.f32x2 P, P, S;\n\t"
      "fma.rn.f32x2 P, P, T, P;\n\tmov.b64 {%0, %1}, P;\n\t}"
      : "=f"(o0), "=f"(o1)
      : "r"(h0), "r"(h1), "r"(b0), "r"(b1), "f"(t0), "f"(t1), "f"(s), "f"(s));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}

// 32 SwiGLU outputs of one TMEM row slice (h = A/2 and B, 32 columns each), scaled by `sc`,
// packed to bf16 and written as 16-byte chunks c0 .. c0 + 3 of this lane's 128-byte row of
// a 128-byte-swizzled staging box.
__device__ __forceinline__ void swiglu_piece(const uint32_t (&ra)[32], const uint32_t (&rb)[32],
                                             float sc, uint32_t box, int lane, int c0) {
  uint32_t pk[16];
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    float f0, f1;
    swiglu2(ra[j], ra[j + 1], rb[j], rb[j + 1], sc, f0, f1);
    pk[j / 2] = pack_bf16x2(f0, f1);
  }
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const uint32_t addr = box + lane * 128 + (((c0 + cc) ^ (lane & 7)) << 4);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * cc]),
                 "r"(pk[4 * cc + 1]), "r"(pk[4 * cc + 2]), "r"(pk[4 * cc + 3])
                 : "memory");
  }
}

}  // namespace umma
}  // namespace ttt
