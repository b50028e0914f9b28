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

// gelu_tanh(x) = 0.5 x (1 + tanh(u)), u = sqrt(2/pi) (x + 0.044715 x^3), in
// fp32 through the identity 0.5 (1 + tanh(u)) = 1 / (1 + exp(-2u)):
// gelu_tanh(x) = x / (1 + exp(-2u)). For x -> -inf, exp(-2u) overflows to
// +inf and the quotient is -0 (the limit); for x -> +inf it is x.
__device__ __forceinline__ float gelu_tanh_f32(float x) {
  constexpr float kA = -1.5957691216057308f;            // -2 sqrt(2/pi)
  constexpr float kB = -1.5957691216057308f * 0.044715f;
  const float m2u = x * __fmaf_rn(kB, x * x, kA);       // -2u
  return __fdividef(x, 1.0f + __expf(m2u));
}

// h = bf16(gelu_tanh(g) * u) for g, u that are bf16 values held in fp32.
__device__ __forceinline__ float geglu_f32(float g, float u) {
  return __fmul_rn(gelu_tanh_f32(g), u);
}

}  // namespace fp8k
