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

#include "act.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace fp8k {

// ------------------------------------------------------------------ router
// Top-k expert choice from the bf16 router's logits (the router, router.proj,
// stays bf16 in every build: sizes article, "Step 1 - Build the Larger
// Repacks"). One warp per token: each lane holds the logits of experts lane,
// lane + 32, ... (at most kTopkMaxE / 32 each); k rounds of a warp-wide
// maximum pick the largest logits, ties to the lower expert index, so the
// choice is unique. The weights are the softmax over the k chosen logits,
// w_j = exp(l_j - l_max) / sum_i exp(l_i - l_max), in fp32 with IEEE
// division (the pages give no router weights; the renormalized top-k softmax
// is the reading). A NaN or infinite logit sets FP8_DEV_NONFINITE (a NaN
// ranks lowest); that token's outputs are unspecified.
constexpr int kTopkMaxE = 1024;
constexpr int kTopkMaxK = 16;

// Each logit travels as one 32-bit key whose unsigned order is the choice
// order: the bf16 pattern made order-preserving (negative values bit-flipped,
// positive ones with the sign bit set; -0 taken as +0; NaN mapped to 0,
// below -inf) in the
// high half and 0xFFFF - expert in the low half (ties go to the lower
// expert). A round is then one warp-wide unsigned max (redux.sync); a chosen
// key is replaced by 0.
__device__ __forceinline__ uint32_t topk_key(uint16_t b, int e) {
  if ((b & 0x7FFFu) == 0u) b = 0u;  // -0 ranks as +0 (equal values tie by index)
  const uint32_t ord = (b & 0x7FFFu) > 0x7F80u ? 0u : ((b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u));
  return (ord << 16) | (0xFFFFu - static_cast<uint32_t>(e));
}

__device__ __forceinline__ float topk_key_value(uint32_t key) {
  const uint32_t ord = key >> 16;
  const uint32_t b = (ord & 0x8000u) ? (ord & 0x7FFFu) : (~ord & 0xFFFFu);
  return __uint_as_float(b << 16);
}

template <int PER_LANE>  // logits held per lane: E <= 32 * PER_LANE
__global__ void __launch_bounds__(256) moe_topk_kernel(const uint16_t* __restrict__ logits,
                                                        int64_t T, int E, int k,
                                                        int32_t* __restrict__ ids,
                                                        float* __restrict__ weights) {
  pdl_launch_dependents();
  pdl_wait();  // the logits come from the preceding router GEMM
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  const uint16_t* row = logits + t * E;
  uint32_t key[PER_LANE];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0u;
    if (e < E) {
      const uint16_t bits = __ldg(row + e);
      bad |= (bits & 0x7FFFu) >= 0x7F80u;  // NaN or +-inf
      key[i] = topk_key(bits, e);
    }
  }
  if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) report(FP8_DEV_NONFINITE);
  int my_id = 0;
  float my_val = 0.0f;
  for (int r = 0; r < k; ++r) {
    uint32_t best = 0u;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) best = max(best, key[i]);
    const uint32_t win = __reduce_max_sync(0xFFFFFFFFu, best);
    const int e = static_cast<int>(0xFFFFu - (win & 0xFFFFu));
    if ((e & 31) == lane) {
#pragma unroll
      for (int i = 0; i < PER_LANE; ++i)
        if (i == (e >> 5)) key[i] = 0u;
    }
    if (lane == r) {
      my_id = e;
      my_val = topk_key_value(win);
    }
  }
  // softmax over the chosen logits: lane 0 holds the largest
  const float vmax = __shfl_sync(0xFFFFFFFFu, my_val, 0);
  const float ex = lane < k ? expf(__fsub_rn(my_val, vmax)) : 0.0f;
  float sum = 0.0f;
  for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, __shfl_sync(0xFFFFFFFFu, ex, j));
  if (lane < k) {
    ids[t * k + lane] = my_id;
    weights[t * k + lane] = __fdiv_rn(ex, sum);
  }
}

// ------------------------------------------------------------------ routing
// One block per expert e over the n = tokens * top_k flat ids:
//   pass 1: base = #{ids < e}, cnt = #{ids == e}; offsets[e + 1] = base + cnt;
//   pass 2: the entries equal to e, in index order, go to perm[base ...] and
//           their positions to inv[]: each thread takes kRouteIds consecutive
//           ids of a chunk, and a block-wide exclusive scan of the per-thread
//           match counts keeps the order. The next chunk's ids are loaded
//           before the current one is scanned.
// Positions are decided by counts alone (no atomics), so the result is unique.
// Out-of-range ids are counted in no expert and set FP8_DEV_BAD_INDEX; every
// position written is still < n.
constexpr int kRouteThreads = 512;
constexpr int kRouteIds = 32;                          // ids per thread per chunk
constexpr int kRouteChunk = kRouteThreads * kRouteIds;

__global__ void __launch_bounds__(kRouteThreads) moe_route_kernel(const int32_t* __restrict__ ids,
                                                                   int64_t n, int E,
                                                                   int32_t* __restrict__ perm,
                                                                   int32_t* __restrict__ inv,
                                                                   int32_t* __restrict__ offsets) {
  pdl_launch_dependents();
  pdl_wait();  // the ids may come from a preceding grid
  constexpr int kWarps = kRouteThreads / 32;
  __shared__ int wsum[kWarps];
  __shared__ int wsum2[kWarps];
  const int e = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  // 16-byte loads when every int4 lies inside the ids.
  const bool vec = (reinterpret_cast<uintptr_t>(ids) & 15) == 0 && n % 4 == 0;
  const int4* ids4 = reinterpret_cast<const int4*>(ids);

  // ---- pass 1
  int lt = 0, eq = 0;
  bool bad = false;
  auto tally = [&](int v) {
    lt += v < e;
    eq += v == e;
    bad |= static_cast<unsigned>(v) >= static_cast<unsigned>(E);
  };
  const int64_t nv = vec ? n / 4 : 0;
  for (int64_t b0 = tid; b0 < nv; b0 += int64_t(kRouteThreads) * 8) {
    int4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t j = b0 + int64_t(i) * kRouteThreads;
      v[i] = j < nv ? __ldg(ids4 + j) : make_int4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (b0 + int64_t(i) * kRouteThreads < nv) {
        tally(v[i].x);
        tally(v[i].y);
        tally(v[i].z);
        tally(v[i].w);
      }
    }
  }
  for (int64_t i = nv * 4 + tid; i < n; i += kRouteThreads) tally(__ldg(ids + i));
  if (e == 0 && bad) report(FP8_DEV_BAD_INDEX);
  lt = __reduce_add_sync(0xFFFFFFFFu, lt);
  eq = __reduce_add_sync(0xFFFFFFFFu, eq);
  if (lane == 0) {
    wsum[w] = lt;
    wsum2[w] = eq;
  }
  __syncthreads();
  int base = 0, cnt = 0;
#pragma unroll
  for (int k = 0; k < kWarps; ++k) {
    base += wsum[k];
    cnt += wsum2[k];
  }
  if (tid == 0) {
    offsets[e + 1] = base + cnt;
    if (e == 0) offsets[0] = 0;
  }
  __syncthreads();  // wsum is reused below
  if (cnt == 0) return;

  // ---- pass 2
  int4 cur[kRouteIds / 4], nxt[kRouteIds / 4];
  auto load = [&](int64_t c0, int4* v) {
    const int64_t i0 = c0 + int64_t(tid) * kRouteIds;
#pragma unroll
    for (int q = 0; q < kRouteIds / 4; ++q) {
      const int64_t i = i0 + 4 * q;
      if (vec) {
        v[q] = i < n ? __ldg(ids4 + i / 4) : make_int4(-1, -1, -1, -1);
      } else {
        v[q].x = i < n ? __ldg(ids + i) : -1;
        v[q].y = i + 1 < n ? __ldg(ids + i + 1) : -1;
        v[q].z = i + 2 < n ? __ldg(ids + i + 2) : -1;
        v[q].w = i + 3 < n ? __ldg(ids + i + 3) : -1;
      }
    }
  };
  load(0, cur);
  for (int64_t c0 = 0; c0 < n; c0 += kRouteChunk) {
    if (c0 + kRouteChunk < n) load(c0 + kRouteChunk, nxt);
    uint32_t mask = 0;
#pragma unroll
    for (int q = 0; q < kRouteIds / 4; ++q) {
      mask |= static_cast<uint32_t>(cur[q].x == e) << (4 * q);
      mask |= static_cast<uint32_t>(cur[q].y == e) << (4 * q + 1);
      mask |= static_cast<uint32_t>(cur[q].z == e) << (4 * q + 2);
      mask |= static_cast<uint32_t>(cur[q].w == e) << (4 * q + 3);
    }
    const int c = __popc(mask);
    int incl = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, d);
      if (lane >= d) incl += v;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    int wpre = 0, total = 0;
#pragma unroll
    for (int k = 0; k < kWarps; ++k) {
      const int v = wsum[k];
      wpre += k < w ? v : 0;
      total += v;
    }
    int pos = base + wpre + incl - c;
    const int64_t i0 = c0 + int64_t(tid) * kRouteIds;
    while (mask) {
      const int j = __ffs(mask) - 1;
      mask &= mask - 1;
      perm[pos] = static_cast<int32_t>(i0 + j);
      inv[i0 + j] = pos;
      ++pos;
    }
    base += total;
    __syncthreads();  // wsum is rewritten by the next chunk
#pragma unroll
    for (int q = 0; q < kRouteIds / 4; ++q) cur[q] = nxt[q];
  }
}

// ------------------------------------------------------------------ weight layout
// Gate/up weights of the GeGLU-fused grouped GEMM: per expert, row
// t*256 + s*128 + j of the output is row s*I + t*128 + j of the input
// (s = 0 gate, 1 up; features t*128 + j >= I give zero rows with scale 0).
// One warp per output row, 16-byte copies (K % 16 == 0).
__global__ void __launch_bounds__(256) moe_interleave_gate_up_kernel(
    const uint8_t* __restrict__ w8, const float* __restrict__ s_ch, int64_t E, int64_t I, int64_t K,
    int64_t tiles, uint8_t* __restrict__ w_il, float* __restrict__ s_il) {
  const int64_t orow = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t per = 256 * tiles;
  if (orow >= E * per) return;
  const int64_t e = orow / per, r = orow % per;
  const int64_t t = r / 256, sg = (r % 256) / 128, j = r % 128;
  const int64_t feat = t * 128 + j;
  const bool live = feat < I;
  const int64_t irow = e * 2 * I + sg * I + feat;
  const uint4* src = reinterpret_cast<const uint4*>(w8 + irow * K);
  uint4* dst = reinterpret_cast<uint4*>(w_il + orow * K);
  for (int64_t v = lane; v < K / 16; v += 32) dst[v] = live ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
  if (lane == 0) s_il[orow] = live ? s_ch[irow] : 0.0f;
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
  const int32_t p = perm[row];
  // not a flat (token, slot) index: a zero row and scale, flagged
  const bool ok = p >= 0 && p < rows;
  if (!ok && lane == 0) report(FP8_DEV_BAD_INDEX);
  const int64_t src = ok ? p / top_k : 0;
  uint4* b = reinterpret_cast<uint4*>(x8_out + row * K);
  const uint4* a = reinterpret_cast<const uint4*>(x8 + src * K);
  // four 16-byte vectors per lane in flight before their stores
  for (int64_t j0 = lane; j0 < K / 16; j0 += 128) {
    uint4 v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      v[i] = ok && j0 + 32 * i < K / 16 ? __ldg(a + j0 + 32 * i) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (j0 + 32 * i < K / 16) b[j0 + 32 * i] = v[i];
  }
  if (lane == 0) s_out[row] = ok ? s_tok[src] : 0.0f;
}

// ------------------------------------------------------------------ GeGLU + quant
// Eight bf16 h values (packed) from eight gate and eight up values.
__device__ __forceinline__ uint4 geglu8(const uint4& g, const uint4& u) {
  const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, uw[4] = {u.x, u.y, u.z, u.w};
  float gf[8], uf[8], hf[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    gf[2 * i] = __uint_as_float(gw[i] << 16);
    gf[2 * i + 1] = __uint_as_float(gw[i] & 0xFFFF0000u);
    uf[2 * i] = __uint_as_float(uw[i] << 16);
    uf[2 * i + 1] = __uint_as_float(uw[i] & 0xFFFF0000u);
  }
  geglu8_f32(gf, uf, hf);
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hf[2 * i + 1]), "f"(hf[2 * i]));
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
// One warp per token, 16-byte accesses (H % 8 == 0). The token's k row
// indices and weights are read once into lanes; for each 16-byte column
// vector all k rows are loaded before the ordered sum (k <= kCombineMaxK).
constexpr int kCombineMaxK = 16;

template <int KMAX>  // slots held per column vector (top_k <= KMAX <= kCombineMaxK)
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
  int r_l = lane < top_k ? inv[t * top_k + lane] : 0;
  if (r_l < 0 || r_l >= T * top_k) {  // not a row of `rows`: contributes nothing, flagged
    report(FP8_DEV_BAD_INDEX);
    r_l = -1;
  }
  const float w_l = lane < top_k ? (weights ? weights[t * top_k + lane] : wu) : 0.0f;
  // Warp-uniform trip count: every lane takes part in the shuffles.
  for (int64_t j0 = 0; j0 < H / 8; j0 += 32) {
    const int64_t j = j0 + lane;
    const bool live = j < H / 8;
    uint4 v[KMAX];
#pragma unroll
    for (int s = 0; s < KMAX; ++s) {
      const int64_t r = __shfl_sync(0xFFFFFFFFu, r_l, s);
      v[s] = make_uint4(0, 0, 0, 0);
      if (s < top_k && live && r >= 0) v[s] = __ldg(reinterpret_cast<const uint4*>(rows + r * H) + j);
    }
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int s = 0; s < KMAX; ++s) {
      const float w = __shfl_sync(0xFFFFFFFFu, w_l, s);
      if (s < top_k) {
        const uint32_t vw[4] = {v[s].x, v[s].y, v[s].z, v[s].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(w, __uint_as_float(vw[i] << 16)));
          acc[2 * i + 1] =
              __fadd_rn(acc[2 * i + 1], __fmul_rn(w, __uint_as_float(vw[i] & 0xFFFF0000u)));
        }
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t r;
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(acc[2 * i + 1]), "f"(acc[2 * i]));
      o[i] = r;
    }
    if (live) reinterpret_cast<uint4*>(out + t * H)[j] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace fp8k
