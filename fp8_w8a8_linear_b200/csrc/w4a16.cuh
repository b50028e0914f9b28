// w4a16.cuh - the W4A16 build: int4 weights that hold the QAT q4_0 grid
// exactly (one fp32 scale per 32 values along K), bf16 activations.
//
// Sizes article ("Gemma 4 From E2B to 31B on an AMD MI300X"), section "The
// Sizes and the Builds" (q4w4a16: int4 holding the QAT grid exactly, bf16
// activations) and section "The 4-Bit Builds Stay Slow at Every Size" (the
// kernel unpacks the weights to bf16 before each multiply); E2B article,
// section "十种构建" (the 4-bit repack keeps each group's trained step and
// stores int4 without rounding again).
//
// Unpacked weight: w = bf16_rn(fp32(d * q)) - the QAT value fp32(d * q) (as
// the FP8 repack reads it) rounded once to bf16, so that it feeds a bf16
// tensor-core MMA (kind::f16) against the bf16 activations.
//
// * w4a16_dequant_kernel: q4 [N, K/2] + d [N, K/32] -> w [N, K] bf16, an HBM
//   streaming kernel (32 groups per warp: 16 + 4 bytes in, 64 out per group).
// * gemm_w4_decode_kernel (M <= 128): swap-AB like the FP8 decode GEMM, with
//   the weight operand unpacked on chip. Warp 0 streams the packed weights
//   and scales (0.625 bytes per weight) into a ring of raw stages with TMA;
//   the last warp streams the token tiles into the operand ring (a thread of
//   its own, so that no token-tile load waits behind a raw-stage refill);
//   the warps from 2 on - sixteen with the deep rings (one CTA per SM), eight
//   with the shallow ones - unpack each raw stage into two 128-row x 64-value
//   bf16 operand blocks in the 128-byte swizzled K-major layout the MMA reads
//   (one 32-value group per thread: the unpacking is a chain of dependent
//   integer and fp32 steps whose latency the other warps hide); warp 1 issues
//   tcgen05.mma.kind::f16 into a TMEM accumulator. K may be split across a thread-block cluster with
//   the partial tiles summed in rank order through distributed shared memory,
//   as in the FP8 decode GEMM. The epilogue stores y = bf16(acc).
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "gemm.cuh"
#include "ptx.cuh"

namespace fp8k {

// Eight int4 values (one 32-bit word of q4, element i in nibble i, two's
// complement) times the group scale d, each rounded to fp32 and then to
// bf16: four bf16x2 words. q + 8 (the nibble XOR 8) is placed in the low
// mantissa bits of 2^23, so 2^23 + (q + 8) - (2^23 + 8) = q exactly.
__device__ __forceinline__ uint4 unpack8_bf16(uint32_t word, float d) {
  const uint32_t u = word ^ 0x88888888u;
  const uint32_t lo = u & 0x0F0F0F0Fu;         // nibbles 0, 2, 4, 6 in bytes 0..3
  const uint32_t hi = (u >> 4) & 0x0F0F0F0Fu;  // nibbles 1, 3, 5, 7
  constexpr uint32_t kTop = 0x4B000000u;       // 2^23
  float q[8];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    // byte b of lo / hi as the low byte of the fp32 pattern 0x4B0000xx
    q[2 * b] = __uint_as_float(__byte_perm(lo, kTop, 0x7540u + b));
    q[2 * b + 1] = __uint_as_float(__byte_perm(hi, kTop, 0x7540u + b));
  }
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float w0, w1;
    asm("{\n\t.reg .b64 v, c, s;\n\t"
        "mov.b64 v, {%2, %3};\n\t"
        "mov.b64 c, {%4, %4};\n\t"
        "mov.b64 s, {%5, %5};\n\t"
        "add.rn.f32x2 v, v, c;\n\t"
        "mul.rn.f32x2 v, v, s;\n\t"
        "mov.b64 {%0, %1}, v;\n\t}"
        : "=f"(w0), "=f"(w1)
        : "f"(q[2 * i]), "f"(q[2 * i + 1]), "f"(-8388616.0f), "f"(d));
    out[i] = pack_bf16x2(w0, w1);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// w [N, K] bf16 from q4 [N, K/2] and d [N, K/32]; K % 32 == 0. A warp takes
// 32 consecutive groups (2 KB of output) at a time: in step j lane l unpacks
// 16-byte piece l % 4 of group 8j + l / 4, so that each store instruction of
// the warp writes 512 contiguous bytes and each load reads 128 contiguous
// bytes of q4 (one whole-line store per lane and piece, not four partial
// ones per 64-byte group).
__global__ void __launch_bounds__(256) w4a16_dequant_kernel(const uint8_t* __restrict__ q4,
                                                             const float* __restrict__ d,
                                                             int64_t groups,
                                                             uint16_t* __restrict__ w) {
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t chunks = (groups + 31) / 32;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const uint32_t* qw = reinterpret_cast<const uint32_t*>(q4);
  uint4* dst = reinterpret_cast<uint4*>(w);
  for (int64_t c = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; c < chunks;
       c += nwarps) {
    const int64_t g0 = 32 * c;
    uint32_t qv[4];
    float dv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t g = g0 + 8 * j + (lane >> 2);
      qv[j] = g < groups ? __ldg(qw + 4 * g + (lane & 3)) : 0u;
      dv[j] = g < groups ? __ldg(d + g) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t g = g0 + 8 * j + (lane >> 2);
      if (g < groups) dst[4 * g0 + 32 * j + lane] = unpack8_bf16(qv[j], dv[j]);
    }
  }
}

// ============================================================== fused decode
// One pipeline step covers 128 values of K: two 64-value k-blocks.
//   raw stage: q4 box [128 rows][64 bytes] then d box [128 rows][4 floats];
//   operand stage: two bf16 weight blocks [128 rows][128 bytes] (128B
//   swizzle) then two token tiles [BNT rows][128 bytes].
template <int BNT, int RS, int AS>
struct W4DecodeCfg {
  static constexpr int kQBytes = kBM * 64;
  static constexpr int kDBytes = kBM * 16;
  static constexpr int kRawBytes = kQBytes + kDBytes;
  static constexpr int kABlock = kBM * kBK;   // 16 KB: 128 rows x 64 bf16
  static constexpr int kXBlock = BNT * kBK;   // BNT rows x 64 bf16
  static constexpr int kStageBytes = 2 * kABlock + 2 * kXBlock;
  static constexpr int kTmemCols = tmem_cols_for(BNT);
  static constexpr int kOpRing = AS * kStageBytes;
  static constexpr int kRawRing = RS * kRawBytes;
  static constexpr int kYBytes = BNT * kBM * 2;  // bf16 output tile, reuses the operand ring
  static constexpr int kBarBytes = 8 * (2 * RS + 2 * AS + 1) + 16;
  static constexpr int kRedBytes = BNT * kBM * 4;
  static constexpr int kFixed = kOpRing + kRawRing + kBarBytes;
  static constexpr int kRedOff = (kFixed + 127) / 128 * 128;  // 16-byte vector accesses
  static constexpr size_t kSmemSingle = 1024 + static_cast<size_t>(kFixed);
  static constexpr size_t kSmemSplit = 1024 + static_cast<size_t>(kRedOff) + kRedBytes;
  static_assert(BNT % 16 == 0 && BNT >= 16 && BNT <= 128, "BNT");
  static_assert(kXBlock % 1024 == 0 && kRawBytes % 1024 == 0, "1024-byte alignment of blocks");
  static_assert(kYBytes <= kOpRing, "output tile must fit in the operand ring");
};

// Unpacking warps: 16 in the deep-ring variants (one CTA per SM), 8 in the
// shallow ones, which must leave room - registers included - for a second
// CTA on the SM.
__host__ __device__ constexpr int w4_unpack_warps(int rs) { return rs >= 4 ? 16 : 8; }
__host__ __device__ constexpr int w4_threads(int rs) { return 32 * (3 + w4_unpack_warps(rs)); }

template <int BNT, int RS, int AS>
__global__ void __launch_bounds__(w4_threads(RS), RS >= 4 ? 1 : 2)
    gemm_w4_decode_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmD,
                          const __grid_constant__ CUtensorMap tmX,
                          const __grid_constant__ CUtensorMap tmY, uint16_t* __restrict__ y, int M,
                          int N, int K, int splits, int st_per_split, int use_tma_store) {
  using C = W4DecodeCfg<BNT, RS, AS>;
  constexpr int kW4DequantWarps = w4_unpack_warps(RS);
  constexpr int kW4XWarp = 2 + kW4DequantWarps;  // the token-tile producer
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* ops = smem;                          // AS operand stages
  uint8_t* raws = smem + C::kOpRing;            // RS raw stages
  uint16_t* ytile = reinterpret_cast<uint16_t*>(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(raws + C::kRawRing);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * RS + 2 * AS + 1);
  float* red = reinterpret_cast<float*>(smem + C::kRedOff);  // split only
  const uint32_t rfull0 = smem_u32(bars);
  const uint32_t rempty0 = smem_u32(bars + RS);
  const uint32_t ofull0 = smem_u32(bars + 2 * RS);
  const uint32_t oempty0 = smem_u32(bars + 2 * RS + AS);
  const uint32_t tfull = smem_u32(bars + 2 * RS + 2 * AS);

  const int warp = warp_id(), lane = lane_id();
  const int tile_n = blockIdx.x / splits;
  const int rank = blockIdx.x % splits;  // == %cluster_ctarank for cluster dims (splits,1,1)
  const int num_st = (K + 127) / 128;
  const int st0 = rank * st_per_split;
  const int st1 = min(num_st, st0 + st_per_split);
  const int nst = max(0, st1 - st0);
  const bool split = splits > 1;
  const int rows = kBM / splits;
  bool have_acc = nst > 0;
  const int pre = min(RS, nst);

  if (split) cluster_arrive_relaxed();
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < RS; ++s) {
      mbar_init(rfull0 + 8 * s, 1);
      mbar_init(rempty0 + 8 * s, kW4DequantWarps);
    }
    for (int s = 0; s < AS; ++s) {
      mbar_init(ofull0 + 8 * s, kW4DequantWarps + 1);  // the unpacking warps + the token tiles
      mbar_init(oempty0 + 8 * s, 1);
    }
    mbar_init(tfull, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmD);
    tma_prefetch_desc(&tmX);
    // The packed weights depend on nothing a preceding grid writes: start
    // the raw ring now.
    const uint64_t pol_w = l2_policy_evict_first();
    for (int i = 0; i < pre; ++i) {
      const uint32_t fb = rfull0 + 8 * i;
      uint8_t* r = raws + i * C::kRawBytes;
      mbar_arrive_expect_tx(fb, C::kRawBytes);
      tma_load_2d(smem_u32(r), &tmQ, fb, (st0 + i) * 64, tile_n * kBM, pol_w);
      tma_load_2d(smem_u32(r + C::kQBytes), &tmD, fb, (st0 + i) * 4, tile_n * kBM, pol_w);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0 && have_acc) {
      // refill the raw stage step i used with step i + RS, once it is unpacked
      const uint64_t pol_w = l2_policy_evict_first();
      for (int i = 0; i + RS < nst; ++i) {
        const int rs = i % RS;
        if (!mbar_wait(rempty0 + 8 * rs, (i / RS) & 1)) break;
        const uint32_t rb = rfull0 + 8 * rs;
        uint8_t* r = raws + rs * C::kRawBytes;
        mbar_arrive_expect_tx(rb, C::kRawBytes);
        tma_load_2d(smem_u32(r), &tmQ, rb, (st0 + i + RS) * 64, tile_n * kBM, pol_w);
        tma_load_2d(smem_u32(r + C::kQBytes), &tmD, rb, (st0 + i + RS) * 4, tile_n * kBM, pol_w);
      }
    }
  } else if (warp == kW4XWarp) {
    if (lane == 0 && have_acc) {
      const uint64_t pol_x = l2_policy_evict_last();
      pdl_wait();  // the activations may come from the preceding grid
      for (int i = 0; i < nst; ++i) {
        // token tiles of step i into operand stage i % AS
        const int os = i % AS;
        if (!mbar_wait(oempty0 + 8 * os, ((i / AS) & 1) ^ 1)) break;
        const uint32_t fb = ofull0 + 8 * os;
        uint8_t* x0 = ops + os * C::kStageBytes + 2 * C::kABlock;
        mbar_arrive_expect_tx(fb, 2 * C::kXBlock);
        tma_load_2d(smem_u32(x0), &tmX, fb, (st0 + i) * 256, 0, pol_x);
        tma_load_2d(smem_u32(x0 + C::kXBlock), &tmX, fb, (st0 + i) * 256 + 128, 0, pol_x);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && have_acc) {
      constexpr uint32_t idesc = idesc_kind<kKindBF16>(kBM, BNT);
      for (int i = 0; i < nst; ++i) {
        const int os = i % AS;
        if (!mbar_wait(ofull0 + 8 * os, (i / AS) & 1)) break;
        tc_fence_after();
        const uint8_t* st = ops + os * C::kStageBytes;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t a0 = smem_u32(st + j * C::kABlock);
          const uint32_t b0 = smem_u32(st + 2 * C::kABlock + j * C::kXBlock);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            umma_kind<kKindBF16>(tmem_base, sw128_kmajor_desc(a0 + 32 * k),
                                 sw128_kmajor_desc(b0 + 32 * k), idesc, (i | j | k) != 0);
        }
        umma_commit(oempty0 + 8 * os);
      }
      umma_commit(tfull);
    }
  } else {
    // The unpacking warps: unit (r, c) turns 16-byte piece c of row r's
    // packed step (32 values, one group; k-block j = c / 2) into four
    // 16-byte pieces of row r of weight block j, piece p of a row stored at
    // p ^ (r & 7) (the 128-byte swizzle). 512 units per step, one or two per
    // thread. Explicit shared-memory accesses.
    const int t = threadIdx.x - 64;
    for (int i = 0; have_acc && i < nst; ++i) {
      const int rs = i % RS, os = i % AS;
      const bool ok = mbar_wait(rfull0 + 8 * rs, (i / RS) & 1) &&
                      mbar_wait(oempty0 + 8 * os, ((i / AS) & 1) ^ 1);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      const uint32_t raw = smem_u32(raws + rs * C::kRawBytes);
#pragma unroll
      for (int u = t; u < 512; u += 32 * kW4DequantWarps) {
        const int r = u & 127, c = u >> 7;
        const int j = c >> 1, p0 = (c & 1) * 4;
        uint32_t q[4];
        float dg;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(q[0]), "=r"(q[1]), "=r"(q[2]), "=r"(q[3])
                     : "r"(raw + r * 64 + c * 16));
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(dg) : "r"(raw + C::kQBytes + r * 16 + c * 4));
        const uint32_t arow = smem_u32(ops + os * C::kStageBytes + j * C::kABlock + r * 128);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const uint4 v = unpack8_bf16(q[w], dg);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(arow + (((p0 + w) ^ (r & 7)) << 4)),
                       "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                       : "memory");
        }
      }
      fence_proxy_async_shared();  // the generic writes -> visible to the tensor core
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(rempty0 + 8 * rs);
        mbar_arrive(ofull0 + 8 * os);
      }
    }
  }

  // ---- epilogue: warps 2..5 (TMEM lane quadrants); the other warps only wait
  const bool epi = warp >= 2 && warp < 6;
  if (epi) {
    const int et = threadIdx.x - 64;  // 0..127
    const int quad = warp & 3;
    const int ch = quad * 32 + lane;
    if (have_acc && !mbar_wait(tfull, 0)) have_acc = false;
    __syncwarp();
    tc_fence_after();
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    uint32_t dst = 0;
    if (split) {
      cluster_wait_acquire();  // every CTA of the cluster has started
      // owner's buffer [rank][channel in slice][token], 16-byte stores
      dst = mapa_shared(smem_u32(red) + static_cast<uint32_t>(((rank * rows + ch % rows) * BNT) * 4),
                        ch / rows);
    }
    (void)et;
#pragma unroll 1
    for (int c = 0; c < BNT / 16; ++c) {
      uint32_t rr[16];
      tmem_ld16(t_row + c * 16, rr);
      tmem_ld_wait();
      float acc[16];
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) acc[jj] = have_acc ? __uint_as_float(rr[jj]) : 0.0f;
      if (!split) {
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) ytile[(c * 16 + jj) * kBM + ch] = f32_to_bf16_rn(acc[jj]);
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (c * 16 + 4 * q < M)
            asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(
                             dst + static_cast<uint32_t>((c * 16 + 4 * q) * 4)),
                         "f"(acc[4 * q]), "f"(acc[4 * q + 1]), "f"(acc[4 * q + 2]), "f"(acc[4 * q + 3])
                         : "memory");
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  if (split) {
    if (!epi) cluster_wait_acquire();  // the first barrier phase, for the other warps
    cluster_arrive_release();          // this CTA's partials are in their owners' buffers
    cluster_wait_acquire();
    if (epi) {
      // four tokens of one channel per thread and step, summed over the ranks
      // in rank order (tokens past M are left out: the store clips them)
      const int et = threadIdx.x - 64;
      constexpr int kTG = BNT / 4;
      const uint32_t red_s = smem_u32(red);
      for (int e = et; e < rows * kTG; e += 128) {
        const int rl = e / kTG, tg = e % kTG;
        if (4 * tg >= M) continue;
        float4 sum;
        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(sum.x), "=f"(sum.y), "=f"(sum.z), "=f"(sum.w)
                     : "r"(red_s + static_cast<uint32_t>((rl * BNT + 4 * tg) * 4)));
        for (int s = 1; s < splits; ++s) {
          float4 v;
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                       : "r"(red_s + static_cast<uint32_t>(((s * rows + rl) * BNT + 4 * tg) * 4)));
          sum.x = __fadd_rn(sum.x, v.x);
          sum.y = __fadd_rn(sum.y, v.y);
          sum.z = __fadd_rn(sum.z, v.z);
          sum.w = __fadd_rn(sum.w, v.w);
        }
        ytile[(4 * tg) * rows + rl] = f32_to_bf16_rn(sum.x);
        ytile[(4 * tg + 1) * rows + rl] = f32_to_bf16_rn(sum.y);
        ytile[(4 * tg + 2) * rows + rl] = f32_to_bf16_rn(sum.z);
        ytile[(4 * tg + 3) * rows + rl] = f32_to_bf16_rn(sum.w);
      }
    }
  }
  const int rows_out = split ? rows : kBM;
  const int n0 = tile_n * kBM + (split ? rank * rows : 0);
  if (use_tma_store) {
    if (epi) {
      fence_proxy_async_shared();
      named_bar_sync(1, 128);
      if (threadIdx.x == 64) {
        tma_store_2d(&tmY, smem_u32(ytile), n0, 0);
        bulk_commit_group();
        bulk_wait_group_all();
      }
    }
  } else if (epi) {
    named_bar_sync(1, 128);
    const int et = threadIdx.x - 64;
    for (int e = et; e < rows_out * BNT; e += 128) {
      const int tok = e / rows_out, rl = e % rows_out;
      if (tok < M && n0 + rl < N) y[static_cast<int64_t>(tok) * N + n0 + rl] = ytile[tok * rows_out + rl];
    }
  }
}

}  // namespace fp8k
