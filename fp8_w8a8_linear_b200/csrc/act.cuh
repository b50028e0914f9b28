// act.cuh - the expert MLP's activation, shared by the GeGLU kernel and the
// GeGLU epilogue of the grouped gate/up GEMM so that both evaluate it with
// the same fp32 operations (and give the same bits).
//
// Expert MLP (dev.to "Gemma 4 From E2B to 31B on an AMD MI300X", sections
// "Step 1 - Build the Larger Repacks" and "Why the Mixture-of-Experts Model
// Sits Lower"): per expert a gate, an up and a down FP8 linear; the pages
// name no activation, and the GELU-tanh gated unit is the reading used here.
#pragma once

namespace fp8k {

// h = gelu_tanh(g) * up for g, up that are bf16 values held in fp32, in fp32,
// within one bf16 ulp of the exact product for every bf16 g and every
// |up| <= 2^40 (the caller rounds h to bf16 once): geglu8_f32 below.
//
// gelu_tanh(g) = 0.5 g (1 + tanh(v)), v = sqrt(2/pi) (g + 0.044715 g^3),
// evaluated through 0.5 (1 + tanh(v)) = sigmoid(2v) = 1 / (1 + exp(-2v)).
// With a = -2|v| <= 0 and e = exp(a) in (0, 1] (no overflow for any g):
//   g >= 0:  sigmoid(2v) = 1 / (1 + e),   gelu = g / (1 + e);
//   g <  0:  sigmoid(2v) = e / (1 + e),   gelu = g e / (1 + e).
// On the common path -2|v| <= 86 (every g >= -9.9), e >= 4e-38 is a normal
// number and 1 + e lies in [1, 2]: the hardware exponential and division
// keep a relative error below 1e-5 there (no flush to zero, no huge divisor),
// far inside one bf16 ulp (2^-8).
// In the far negative tail (g < -9.9, -2v > 86) e is near or below the
// smallest normal fp32 value and 1 + e == 1, so h = g e up, taken in the log
// domain as exp(L), L = 2v + ln|g| + ln|up|: that neither flushes through a
// subnormal intermediate nor depends on how small e is. exp(L) is evaluated
// as exp(L + 64 ln 2) * 2^-64, so the hardware exponential always returns a
// normal number (L >= -131.7) or underflows only where exp(L) < 1e-57, far
// below the smallest bf16 subnormal; the multiply by 2^-64 is exact but for
// one rounding onto the fp32 grid (2^-149). Relative error: below 2e-5.
//
// This runs for every element in the gate/up GEMM's epilogue, so the common
// path is branch-free over a group of eight values (their dependency chains
// interleave) and the rare tail values are redone afterwards, behind one
// branch per group.
constexpr float kGeluA = -1.5957691216057308f;  // -2 sqrt(2/pi)
constexpr float kGeluB = -1.5957691216057308f * 0.044715f;

__device__ __forceinline__ float gelu_m2v(float g) {  // -2v, sign opposite to g
  return __fmul_rn(g, __fmaf_rn(kGeluB, __fmul_rn(g, g), kGeluA));
}

__device__ __forceinline__ bool geglu_in_tail(float g, float m2v) { return g < 0.0f && m2v > 86.0f; }

__device__ __forceinline__ float geglu_main(float g, float up, float m2v) {
  const float e = __expf(-fabsf(m2v));
  const float num = g < 0.0f ? __fmul_rn(g, e) : g;
  return __fmul_rn(__fdividef(num, __fadd_rn(1.0f, e)), up);
}

__device__ __forceinline__ float geglu_tail(float g, float up, float m2v) {
  constexpr float k64Ln2 = 44.3614195558365f;  // 64 ln 2
  const float L = __fadd_rn(__fadd_rn(-m2v, __logf(-g)), __logf(fabsf(up)));
  return copysignf(__fmul_rn(__expf(__fadd_rn(L, k64Ln2)), 0x1p-64f), -up);  // sign of g up
}

// h[i] = gelu_tanh(g[i]) * u[i] for eight values (bf16 numbers held in fp32).
__device__ __forceinline__ void geglu8_f32(const float (&g)[8], const float (&u)[8], float (&h)[8]) {
  float m2v[8];
  bool tail = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    m2v[i] = gelu_m2v(g[i]);
    h[i] = geglu_main(g[i], u[i], m2v[i]);
    tail |= geglu_in_tail(g[i], m2v[i]);
  }
  if (tail) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (geglu_in_tail(g[i], m2v[i])) h[i] = geglu_tail(g[i], u[i], m2v[i]);
  }
}

}  // namespace fp8k
