// quant.cuh - HBM-streaming FP8 quantizers for sm_100a:
//   * per-token activation quantization (bf16 -> E4M3 + fp32 scale),
//   * QAT q4_0 -> per-channel E4M3 repack,
//   * E4M3FNUZ -> E4M3 load conversion,
//   * the element-wise fp32 -> E4M3 cast.
//
// Arithmetic contract (model card "Gemma 4 31B-it QAT, FP8 E4M3 W8A8",
// header paragraph: one fp32 scale per output channel, per-token activation
// quantization): per row, amax = max|v|, s = fp32(amax / 448) and
// code = E4M3_RNE_SATFINITE(fp32(v / s)), with IEEE round-to-nearest
// division (__fdiv_rn) and multiplication (__fmul_rn, never contracted into
// an FMA); zero results are +0, an all-zero row gets s = 0.
//
// Layout: rows are contiguous in HBM; one row is handled by a fixed group of
// threads (TPR threads) that first reduces amax over the row with integer
// max on the magnitude bit patterns (which orders non-negative floats and
// puts NaN above Inf, so non-finite rows are detected for free), then
// quantizes the row from registers when it fits (V vectors per thread) or
// re-reads it from L1/L2 otherwise. Loads and stores are 16-byte vectors,
// consecutive threads on consecutive vectors.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace fp8k {

constexpr float kE4M3Max = 448.0f;

// Reduction of a 32-bit unsigned max across the TPR threads of one row.
// TPR is 32 (one warp per row) or a multiple of 32 up to the block size (a
// whole block per row); `red` holds one word per warp of the block.
template <int TPR>
__device__ __forceinline__ uint32_t row_max_u32(uint32_t v, uint32_t* red) {
  v = __reduce_max_sync(0xFFFFFFFFu, v);
  if constexpr (TPR == 32) {
    return v;
  } else {
    constexpr int WPR = TPR / 32;
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    const int w0 = (w / WPR) * WPR;
    uint32_t m = red[w0];
#pragma unroll
    for (int i = 1; i < WPR; ++i) m = max(m, red[w0 + i]);
    __syncthreads();
    return m;
  }
}

// ----------------------------------------------------------- activation quant
// x: [M, ldx] bf16, K % 8 == 0 (16-byte vectors of 8 values).
template <int TPR, int V>
__global__ void __launch_bounds__(256) quant_act_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                         int64_t K, int64_t ldx,
                                                         uint8_t* __restrict__ x8,
                                                         float* __restrict__ s_tok) {
  pdl_launch_dependents();
  __shared__ uint32_t red[8];
  constexpr int RPB = 256 / TPR;  // rows per block
  const int64_t row = static_cast<int64_t>(blockIdx.x) * RPB + threadIdx.x / TPR;
  const int t = threadIdx.x % TPR;
  const bool active = row < M;
  const int64_t nvec = K / 8;
  const uint4* src = reinterpret_cast<const uint4*>(x + (active ? row : 0) * ldx);

  uint4 cache[V > 0 ? V : 1];
  uint32_t mx = 0;  // running max of |bf16| bit patterns, two lanes per word
  if (V > 0 && nvec <= static_cast<int64_t>(V) * TPR) {
#pragma unroll
    for (int i = 0; i < (V > 0 ? V : 1); ++i) {
      const int64_t j = t + static_cast<int64_t>(i) * TPR;
      if (active && j < nvec) {
        cache[i] = __ldg(src + j);
      } else {
        cache[i] = make_uint4(0, 0, 0, 0);
      }
      mx = __vmaxu2(mx, cache[i].x & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, cache[i].y & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, cache[i].z & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, cache[i].w & 0x7FFF7FFFu);
    }
  } else {
    for (int64_t j = t; active && j < nvec; j += TPR) {
      const uint4 u = __ldg(src + j);
      mx = __vmaxu2(mx, u.x & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, u.y & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, u.z & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, u.w & 0x7FFF7FFFu);
    }
  }
  mx = max(mx & 0xFFFFu, mx >> 16);
  const uint32_t amax_bits = row_max_u32<TPR>(mx, red);
  if (!active) return;
  if (amax_bits >= 0x7F80u) {  // Inf or NaN in the row
    if (t == 0) report(FP8_DEV_NONFINITE);
  }
  const float amax = __uint_as_float(amax_bits << 16);
  const float s = __fdiv_rn(amax, kE4M3Max);
  if (t == 0) s_tok[row] = s;
  uint2* dst = reinterpret_cast<uint2*>(x8 + row * K);

  auto quant8 = [&](const uint4& u) -> uint2 {
    if (s == 0.0f) return make_uint2(0, 0);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __fdiv_rn(__uint_as_float(w[i] << 16), s);
      f[2 * i + 1] = __fdiv_rn(__uint_as_float(w[i] & 0xFFFF0000u), s);
    }
    return make_uint2(pack4_e4m3(f[0], f[1], f[2], f[3]), pack4_e4m3(f[4], f[5], f[6], f[7]));
  };

  if (V > 0 && nvec <= static_cast<int64_t>(V) * TPR) {
#pragma unroll
    for (int i = 0; i < (V > 0 ? V : 1); ++i) {
      const int64_t j = t + static_cast<int64_t>(i) * TPR;
      if (j < nvec) dst[j] = quant8(cache[i]);
    }
  } else {
    for (int64_t j = t; j < nvec; j += TPR) dst[j] = quant8(__ldg(src + j));
  }
}

// ----------------------------------------------------------- QAT repack
// One q4_0 group = 32 values = one 16-byte vector of packed nibbles + one
// fp32 scale. Because every value in a group is d * q with q in [-8, 7], the
// group's codes come from a 16-entry table indexed by the nibble: the table
// holds code(d * q) for q = 1..8 (8 divisions) and its sign-flipped copies,
// which is exact because IEEE multiplication, division and the E4M3 RNE
// encoding are all symmetric under negation. Bytes are then gathered four at
// a time with byte permutes.
struct GroupLUT {
  uint32_t t0, t1, t2, t3;  // table bytes for nibbles 0..15
};

__device__ __forceinline__ GroupLUT group_lut(float d, float s) {
  // c[q] = code(fp32(fp32(d*q) / s)) for q = 1..8; code(0) = 0.
  float f[8];
#pragma unroll
  for (int q = 1; q <= 8; ++q) f[q - 1] = __fdiv_rn(__fmul_rn(d, static_cast<float>(q)), s);
  const uint32_t p0 = pack4_e4m3(f[0], f[1], f[2], f[3]);  // codes of q = 1..4
  const uint32_t p1 = pack4_e4m3(f[4], f[5], f[6], f[7]);  // codes of q = 5..8
  // Negation flips bit 7 of every nonzero code (d may be negative, so the
  // codes of q = 1..8 can carry either sign).
  const uint32_t n0 = p0 ^ (0x80808080u & ~__vcmpeq4(p0, 0u));
  const uint32_t n1 = p1 ^ (0x80808080u & ~__vcmpeq4(p1, 0u));
  GroupLUT L;
  // nibble 0..7 -> q = 0..7: [0, c1, c2, c3 | c4, c5, c6, c7]
  L.t0 = (p0 << 8);
  L.t1 = (p0 >> 24) | (p1 << 8);
  // nibble 8..15 -> q = -8..-1: [-c8, -c7, -c6, -c5 | -c4, -c3, -c2, -c1]
  L.t2 = __byte_perm(n1, 0, 0x0123);
  L.t3 = __byte_perm(n0, 0, 0x0123);
  return L;
}

// Four nibbles (the low 16 bits of `chunk`, nibble i -> output byte i).
__device__ __forceinline__ uint32_t lut4(const GroupLUT& L, uint32_t chunk) {
  const uint32_t idx = chunk & 0x7777u;
  const uint32_t lo = __byte_perm(L.t0, L.t1, idx);
  const uint32_t hi = __byte_perm(L.t2, L.t3, idx);
  const uint32_t sel = __byte_perm(0x0000FF00u, 0u, (chunk >> 3) & 0x1111u);  // 0xFF if nibble >= 8
  return lo ^ ((lo ^ hi) & sel);
}

// Largest |q| over the 8 nibbles of a word, as a byte-wise running max.
__device__ __forceinline__ uint32_t nib_absmax(uint32_t w, uint32_t acc) {
  const uint32_t a = w & 0x0F0F0F0Fu;
  const uint32_t b = (w >> 4) & 0x0F0F0F0Fu;
  acc = __vmaxu4(acc, __vminu4(a, __vsub4(0x10101010u, a)));
  acc = __vmaxu4(acc, __vminu4(b, __vsub4(0x10101010u, b)));
  return acc;
}

template <int TPR, int V>
__global__ void __launch_bounds__(256) repack_qat_kernel(const uint8_t* __restrict__ q4,
                                                          const float* __restrict__ d, int64_t N,
                                                          int64_t K, uint8_t* __restrict__ w8,
                                                          float* __restrict__ s_ch) {
  __shared__ uint32_t red[8];
  constexpr int RPB = 256 / TPR;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * RPB + threadIdx.x / TPR;
  const int t = threadIdx.x % TPR;
  const bool active = row < N;
  const int64_t ng = K / 32;
  const uint4* qsrc = reinterpret_cast<const uint4*>(q4 + (active ? row : 0) * (K / 2));
  const float* dsrc = d + (active ? row : 0) * ng;
  const bool cached = V > 0 && ng <= static_cast<int64_t>(V) * TPR;

  uint4 qc[V > 0 ? V : 1];
  float dc[V > 0 ? V : 1];
  uint32_t mbits = 0;  // max over groups of the bit pattern of fp32(|d| * max|q|)
  auto group_amax = [&](const uint4& u, float dg) {
    uint32_t acc = 0;
    acc = nib_absmax(u.x, acc);
    acc = nib_absmax(u.y, acc);
    acc = nib_absmax(u.z, acc);
    acc = nib_absmax(u.w, acc);
    acc = __vmaxu4(acc, acc >> 16);
    acc = __vmaxu4(acc, acc >> 8);
    const float qmax = static_cast<float>(acc & 0xFFu);
    // max_k |fp32(d*q_k)| = fp32(|d| * max_k |q_k|): rounding is monotone.
    return __float_as_uint(__fmul_rn(fabsf(dg), qmax));
  };
  if (cached) {
#pragma unroll
    for (int i = 0; i < (V > 0 ? V : 1); ++i) {
      const int64_t g = t + static_cast<int64_t>(i) * TPR;
      if (active && g < ng) {
        qc[i] = __ldg(qsrc + g);
        dc[i] = __ldg(dsrc + g);
        mbits = max(mbits, group_amax(qc[i], dc[i]));
      } else {
        qc[i] = make_uint4(0, 0, 0, 0);
        dc[i] = 0.0f;
      }
    }
  } else {
    for (int64_t g = t; active && g < ng; g += TPR)
      mbits = max(mbits, group_amax(__ldg(qsrc + g), __ldg(dsrc + g)));
  }
  const uint32_t amax_bits = row_max_u32<TPR>(mbits, red);
  if (!active) return;
  if (amax_bits >= 0x7F800000u) {
    if (t == 0) report(FP8_DEV_NONFINITE);
  }
  const float amax = __uint_as_float(amax_bits);
  const float s = __fdiv_rn(amax, kE4M3Max);
  if (t == 0) s_ch[row] = s;
  uint4* dst = reinterpret_cast<uint4*>(w8 + row * K);

  auto emit = [&](int64_t g, const uint4& u, float dg) {
    uint4 o0, o1;
    if (s == 0.0f) {
      o0 = make_uint4(0, 0, 0, 0);
      o1 = o0;
    } else {
      const GroupLUT L = group_lut(dg, s);
      o0.x = lut4(L, u.x);
      o0.y = lut4(L, u.x >> 16);
      o0.z = lut4(L, u.y);
      o0.w = lut4(L, u.y >> 16);
      o1.x = lut4(L, u.z);
      o1.y = lut4(L, u.z >> 16);
      o1.z = lut4(L, u.w);
      o1.w = lut4(L, u.w >> 16);
    }
    dst[2 * g] = o0;
    dst[2 * g + 1] = o1;
  };
  if (cached) {
#pragma unroll
    for (int i = 0; i < (V > 0 ? V : 1); ++i) {
      const int64_t g = t + static_cast<int64_t>(i) * TPR;
      if (g < ng) emit(g, qc[i], dc[i]);
    }
  } else {
    for (int64_t g = t; g < ng; g += TPR) emit(g, __ldg(qsrc + g), __ldg(dsrc + g));
  }
}

// ----------------------------------------------------------- FNUZ -> E4M3
// E4M3FNUZ code -> fp32 value (exact). Bias 8; e == 0 holds m/8 * 2^-7.
__device__ __forceinline__ float dec_fnuz(uint32_t b) {
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  const float mag = (e == 0) ? static_cast<float>(m) * 0x1p-10f
                             : __uint_as_float(((e + 127u - 8u) << 23) | (m << 20));
  return (b & 0x80u) ? -mag : mag;
}
// E4M3 code -> fp32 value (exact, finite codes). Bias 7; e == 0 holds m/8 * 2^-6.
__device__ __forceinline__ float dec_e4m3(uint32_t b) {
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  const float mag = (e == 0) ? static_cast<float>(m) * 0x1p-9f
                             : __uint_as_float(((e + 127u - 7u) << 23) | (m << 20));
  return (b & 0x80u) ? -mag : mag;
}

template <int TPR>
__global__ void __launch_bounds__(256) convert_fnuz_kernel(const uint8_t* src,
                                                            const float* s_src,
                                                            int64_t N, int64_t K, uint8_t* dst,
                                                            float* s_dst) {
  __shared__ uint32_t red[8];
  constexpr int RPB = 256 / TPR;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * RPB + threadIdx.x / TPR;
  const int t = threadIdx.x % TPR;
  const bool active = row < N;
  const int64_t nvec = K / 16;
  const uint4* in = reinterpret_cast<const uint4*>(src + (active ? row : 0) * K);
  // Read the scale before the row-wide reduction below, so that an in-place
  // conversion (s_dst == s_src) cannot overwrite it before every thread of
  // the row has read it.
  const float s_in = active ? s_src[row] : 0.0f;
  uint32_t flags = 0;  // bit 0: a 0x80 code, bit 1: a +-240 code
  for (int64_t j = t; active && j < nvec; j += TPR) {
    const uint4 u = in[j];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (__vcmpeq4(w[i], 0x80808080u)) flags |= 1u;
      if (__vcmpeq4(w[i] & 0x7F7F7F7Fu, 0x7F7F7F7Fu)) flags |= 2u;
    }
  }
  flags = row_max_u32<TPR>(__reduce_or_sync(0xFFFFFFFFu, flags), red);
  if (!active) return;
  const float half = __fmul_rn(s_in, 0.5f);
  const bool finite = isfinite(s_in);
  const bool keep = !(flags & 2u) && finite && __fmul_rn(half, 2.0f) == s_in;
  if (t == 0) {
    if (flags & 1u) report(FP8_DEV_NAN_CODE);
    if (!finite) report(FP8_DEV_NONFINITE);
  }
  uint4* out = reinterpret_cast<uint4*>(dst + row * K);
  bool inexact = false;
  if (keep) {
    if (dst != src)
      for (int64_t j = t; j < nvec; j += TPR) out[j] = in[j];
  } else {
    for (int64_t j = t; j < nvec; j += TPR) {
      const uint4 u = in[j];
      uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float f[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) f[b] = dec_fnuz((w[i] >> (8 * b)) & 0xFFu);
        const uint32_t c = pack4_e4m3(f[0], f[1], f[2], f[3]);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const uint32_t cb = (c >> (8 * b)) & 0xFFu;
          const uint32_t ib = (w[i] >> (8 * b)) & 0xFFu;
          if (ib != 0x80u && dec_e4m3(cb) != f[b]) inexact = true;
        }
        w[i] = c;
      }
      out[j] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  if (__any_sync(0xFFFFFFFFu, inexact) && (t & 31) == 0) report(FP8_DEV_INEXACT);
  if (t == 0) s_dst[row] = keep ? half : s_in;
}

// ----------------------------------------------------------- cast
__global__ void __launch_bounds__(256) cast_e4m3_kernel(const float* __restrict__ x, int64_t n,
                                                         uint8_t* __restrict__ out) {
  const int64_t i4 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
  const int64_t base = i4 * 4;
  if (base >= n) return;
  float f[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) f[i] = (base + i < n) ? x[base + i] : 0.0f;
  uint32_t c = pack4_e4m3(f[0], f[1], f[2], f[3]);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (isnan(f[i])) c = (c & ~(0xFFu << (8 * i))) | (0x7Fu << (8 * i));
  }
  if (base + 4 <= n) {
    *reinterpret_cast<uint32_t*>(out + base) = c;
  } else {
    for (int i = 0; base + i < n; ++i) out[base + i] = (c >> (8 * i)) & 0xFFu;
  }
}

}  // namespace fp8k
