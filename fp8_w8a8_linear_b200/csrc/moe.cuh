// moe.cuh - the mixture-of-experts pieces around the grouped FP8 GEMM:
// deterministic routing (tokens grouped by expert in ascending (token, slot)
// order), gather of quantized rows, GeGLU + per-row quantization, combine.
//
// Layer (dev.to "Gemma 4 From E2B to 31B on an AMD MI300X", section "Step 1 -
// Build the Larger Repacks": 128 experts per layer, one gate/up/down FP8
// linear per expert, bf16 router; section "Why the Mixture-of-Experts Model
// Sits Lower": the fp8_w8a8 fused-MoE path for E=128, N=704).
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"
#include "quant.cuh"

namespace fp8k {

// ------------------------------------------------------------------ routing
// counts[e] (written to offsets[e + 1]) = number of flat entries equal to e.
__global__ void __launch_bounds__(256) moe_count_kernel(const int32_t* __restrict__ ids,
                                                         int64_t n, int32_t* __restrict__ offsets) {
  pdl_launch_dependents();
  __shared__ int red[8];
  const int e = blockIdx.x;
  int c = 0;
  bool bad = false;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
    const int32_t v = ids[i];
    c += v == e;
    bad |= e == 0 && (v < 0 || v >= static_cast<int>(gridDim.x));
  }
  if (bad) report(FP8_DEV_BAD_INDEX);
  c = __reduce_add_sync(0xFFFFFFFFu, c);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < 8; ++w) t += red[w];
    offsets[e + 1] = t;
  }
}

// Block e writes the flat indices of its entries, in index order, to
// perm[off_e ...] and their positions to inv[]; off_e = sum of counts < e.
// Each thread takes 8 consecutive entries per 2048-entry chunk; a block-wide
// exclusive scan of the per-thread match counts keeps the order.
__global__ void __launch_bounds__(256) moe_scatter_kernel(const int32_t* __restrict__ ids,
                                                           int64_t n,
                                                           const int32_t* __restrict__ counts1,
                                                           int32_t* __restrict__ perm,
                                                           int32_t* __restrict__ inv) {
  pdl_launch_dependents();
  pdl_wait();  // counts come from the preceding count grid
  __shared__ int wsum[8];
  __shared__ int base_s;
  const int e = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid < 32) {
    int s = 0;
    for (int i = tid; i < e; i += 32) s += counts1[i];  // counts1[i] = count of expert i
    s = __reduce_add_sync(0xFFFFFFFFu, s);
    if (tid == 0) base_s = s;
  }
  __syncthreads();
  int base = base_s;
  for (int64_t c0 = 0; c0 < n; c0 += 2048) {
    const int64_t i0 = c0 + static_cast<int64_t>(tid) * 8;
    uint32_t mask = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (i0 + j < n && ids[i0 + j] == e) mask |= 1u << j;
    const int cnt = __popc(mask);
    int incl = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, d);
      if (lane >= d) incl += v;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    int wpre = 0, total = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int v = wsum[k];
      wpre += k < w ? v : 0;
      total += v;
    }
    int pos = base + wpre + incl - cnt;
    while (mask) {
      const int j = __ffs(mask) - 1;
      mask &= mask - 1;
      perm[pos] = static_cast<int32_t>(i0 + j);
      inv[i0 + j] = pos;
      ++pos;
    }
    base += total;
    __syncthreads();
  }
}

// offsets[0] = 0, offsets[e + 1] = counts[0] + ... + counts[e], in place
// (offsets[e + 1] holds counts[e] on entry). One warp.
__global__ void moe_offsets_kernel(int32_t* __restrict__ offsets, int E) {
  pdl_launch_dependents();
  pdl_wait();  // counts come from the count grid, and the scatter grid reads them
  const int lane = threadIdx.x;
  const int per = (E + 31) / 32;
  int sum = 0;
  for (int i = 0; i < per; ++i) {
    const int e = lane * per + i;
    if (e < E) sum += offsets[e + 1];
  }
  int incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, d);
    if (lane >= d) incl += v;
  }
  int run = incl - sum;
  for (int i = 0; i < per; ++i) {
    const int e = lane * per + i;
    if (e < E) {
      const int c = offsets[e + 1];
      run += c;
      offsets[e + 1] = run;
    }
  }
  if (lane == 0) offsets[0] = 0;
}

// ------------------------------------------------------------------ gather
// rows_out[i] = x8[perm[i] / top_k], s_out[i] = s_tok[perm[i] / top_k].
// One warp per row, 16-byte copies (K % 16 == 0).
__global__ void __launch_bounds__(256) moe_gather_kernel(const uint8_t* __restrict__ x8,
                                                          const float* __restrict__ s_tok,
                                                          const int32_t* __restrict__ perm,
                                                          int64_t rows, int64_t K, int top_k,
                                                          uint8_t* __restrict__ x8_out,
                                                          float* __restrict__ s_out) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int64_t src = perm[row] / top_k;
  const uint4* a = reinterpret_cast<const uint4*>(x8 + src * K);
  uint4* b = reinterpret_cast<uint4*>(x8_out + row * K);
  for (int64_t j = lane; j < K / 16; j += 32) b[j] = __ldg(a + j);
  if (lane == 0) s_out[row] = s_tok[src];
}

// ------------------------------------------------------------------ GeGLU + quant
// gelu_tanh(x) = 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))) in fp32.
__device__ __forceinline__ float gelu_tanh_f32(float x) {
  const float inner = 0.7978845608028654f * __fmaf_rn(0.044715f * x, x * x, x);
  return 0.5f * x * (1.0f + tanhf(inner));
}

// Eight bf16 h values (packed) from eight gate and eight up values.
__device__ __forceinline__ uint4 geglu8(const uint4& g, const uint4& u) {
  const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, uw[4] = {u.x, u.y, u.z, u.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float g0 = __uint_as_float(gw[i] << 16), g1 = __uint_as_float(gw[i] & 0xFFFF0000u);
    const float u0 = __uint_as_float(uw[i] << 16), u1 = __uint_as_float(uw[i] & 0xFFFF0000u);
    const float h0 = gelu_tanh_f32(g0) * u0, h1 = gelu_tanh_f32(g1) * u1;
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(h1), "f"(h0));
    o[i] = r;
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// One warp per row of gate_up [M, 2*I] (gate | up); writes h8 [M, I] and
// s_h [M] with the same per-row quantization as the activation quantizer.
// h is recomputed for the second pass (identical arithmetic, so identical
// values). Requires I % 8 == 0.
__global__ void __launch_bounds__(256) moe_geglu_quant_kernel(const uint16_t* __restrict__ gu,
                                                               int64_t M, int64_t I,
                                                               uint8_t* __restrict__ h8,
                                                               float* __restrict__ s_h,
                                                               uint16_t* __restrict__ h_out) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const uint4* g = reinterpret_cast<const uint4*>(gu + row * 2 * I);
  const uint4* u = reinterpret_cast<const uint4*>(gu + row * 2 * I + I);
  const int64_t nvec = I / 8;
  // h of up to kCache vectors per lane stays in registers between the amax
  // pass and the quantize pass; longer rows recompute it (same arithmetic,
  // same values).
  constexpr int kCache = 4;
  uint4 hc[kCache];
  uint32_t mx = 0;
  auto amax_of = [&](const uint4& h, int64_t j) {
    if (h_out) reinterpret_cast<uint4*>(h_out + row * I)[j] = h;
    mx = __vmaxu2(mx, h.x & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, h.y & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, h.z & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, h.w & 0x7FFF7FFFu);
  };
#pragma unroll
  for (int i = 0; i < kCache; ++i) {
    const int64_t j = lane + 32 * i;
    if (j < nvec) {
      hc[i] = geglu8(__ldg(g + j), __ldg(u + j));
      amax_of(hc[i], j);
    }
  }
  for (int64_t j = lane + 32 * kCache; j < nvec; j += 32) amax_of(geglu8(__ldg(g + j), __ldg(u + j)), j);
  mx = max(mx & 0xFFFFu, mx >> 16);
  const uint32_t amax_bits = __reduce_max_sync(0xFFFFFFFFu, mx);
  if (amax_bits >= 0x7F80u && lane == 0) report(FP8_DEV_NONFINITE);
  const float amax = __uint_as_float(amax_bits << 16);
  const float s = __fdiv_rn(amax, kE4M3Max);
  if (lane == 0) s_h[row] = s;
  const RowDivisor dv = make_divisor(s, amax);
  uint2* dst = reinterpret_cast<uint2*>(h8 + row * I);
  auto quant = [&](const uint4& h) -> uint2 {
    if (s == 0.0f) return make_uint2(0, 0);
    const uint32_t wv[4] = {h.x, h.y, h.z, h.w};
    float f[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      f[2 * q] = div_rn(dv, __uint_as_float(wv[q] << 16));
      f[2 * q + 1] = div_rn(dv, __uint_as_float(wv[q] & 0xFFFF0000u));
    }
    return make_uint2(pack4_e4m3(f[0], f[1], f[2], f[3]), pack4_e4m3(f[4], f[5], f[6], f[7]));
  };
#pragma unroll
  for (int i = 0; i < kCache; ++i) {
    const int64_t j = lane + 32 * i;
    if (j < nvec) dst[j] = quant(hc[i]);
  }
  for (int64_t j = lane + 32 * kCache; j < nvec; j += 32) dst[j] = quant(geglu8(__ldg(g + j), __ldg(u + j)));
}

// ------------------------------------------------------------------ combine
// out[t] = sum_{j < k} w[t, j] * rows[inv[t*k + j]] with fp32 products and
// sums in slot order (w = 1/k when weights is null), rounded once to bf16.
// One warp per token, 16-byte accesses (H % 8 == 0).
__global__ void __launch_bounds__(256) moe_combine_kernel(const uint16_t* __restrict__ rows,
                                                           const int32_t* __restrict__ inv,
                                                           int64_t T, int top_k, int64_t H,
                                                           const float* __restrict__ weights,
                                                           uint16_t* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const float wu = __fdiv_rn(1.0f, static_cast<float>(top_k));
  for (int64_t j = lane; j < H / 8; j += 32) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int s = 0; s < top_k; ++s) {
      const int64_t r = inv[t * top_k + s];
      const float w = weights ? weights[t * top_k + s] : wu;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(rows + r * H) + j);
      const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(w, __uint_as_float(vw[i] << 16)));
        acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(w, __uint_as_float(vw[i] & 0xFFFF0000u)));
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t r;
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(acc[2 * i + 1]), "f"(acc[2 * i]));
      o[i] = r;
    }
    reinterpret_cast<uint4*>(out + t * H)[j] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace fp8k
