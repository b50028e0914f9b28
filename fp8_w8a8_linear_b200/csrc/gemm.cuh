// gemm.cuh - row-wise scaled FP8 GEMM on sm_100a tensor cores.
//
//   y[m, n] = bf16_rn( fp32( acc[m, n] * s_tok[m] ) * s_ch[n] ),
//   acc[m, n] = sum_k e4m3(x8[m, k]) * e4m3(w8[n, k])   (fp32, in TMEM)
//
// The row-wise scaled FP8 GEMM of the W8A8 scheme (E2B MI300X article, step 3
// boot log and the E4M3/E4M3FNUZ tip: RowWiseTorchFP8ScaledMMLinearKernel for
// CompressedTensorsW8A8Fp8; 31B model card header: per-output-channel fp32
// weight scales, per-token activation scales, bf16 output).
//
// Two kernels share one pipeline design:
//
// * gemm_prefill_kernel (M > 128): persistent, one CTA per SM, warp
//   specialised. Warp 0 lane 0 streams 128x128-byte A tiles (activations)
//   and BNx128-byte B tiles (weights) with TMA into a STAGES-deep ring of
//   128B-swizzled shared-memory buffers; warp 1 lane 0 issues
//   tcgen05.mma.kind::f8f6f4 (M=128, N=BN, K=32 per instruction) into one of
//   two TMEM accumulators; warps 2-5 drain the other accumulator (tcgen05.ld),
//   apply both scales and store bf16, so the epilogue of tile i overlaps the
//   main loop of tile i+1. Tiles are walked in groups of `group_m` row tiles
//   so that a wave of CTAs shares A and B tiles in L2.
//
// * gemm_decode_kernel (M <= 128): swap-AB. The weight tile is the MMA's A
//   operand (128 output channels per CTA) and the tokens are its N (16..128),
//   so a single token does not waste the 128-row MMA. K is split across the
//   CTAs of a thread-block cluster (splits = cluster size, 1..8). Each CTA
//   owns one slice of the 128 output rows; every CTA stores its fp32 partials
//   for each slice straight into the owner's shared memory (distributed
//   shared memory), and after one cluster barrier each owner sums its slice
//   in rank order - deterministic, no global workspace, no spin-waits. The
//   weight stream uses an L2 evict-first policy, the activation tile
//   evict-last.
//
// Every mbarrier wait is bounded (ptx.cuh); the only unbounded waits are the
// hardware cluster barriers, which every thread reaches on every path.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "act.cuh"
#include "ptx.cuh"

namespace fp8k {

constexpr int kBM = 128;  // MMA M (rows of operand A)
constexpr int kBK = 128;  // K bytes per pipeline stage (= one 128B swizzle row)

__host__ __device__ constexpr int tmem_cols_for(int cols) {
  return cols <= 32 ? 32 : cols <= 64 ? 64 : cols <= 128 ? 128 : cols <= 256 ? 256 : 512;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Two IEEE fp32 products, each rounded to nearest even (one packed
// instruction; per lane identical to __fmul_rn).
__device__ __forceinline__ void fmul2_rn(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 pa, pb, pd;\n\t"
      "mov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t"
      "mul.rn.f32x2 pd, pa, pb;\n\tmov.b64 {%0, %1}, pd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Two fp32 -> bf16 (round to nearest even), `lo` in bits [0,16).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Epilogue store of one 32-row x 32-column bf16 chunk that a warp holds one
// row per lane (pk = the lane's 64 bytes), through the warp's 2 KB staging
// buffer: written row per lane, read back so that each global store
// instruction covers 8 rows x 64 contiguous bytes (instead of 32 rows x 16
// bytes). The 16-byte pieces of row r sit at piece index q ^ ((r >> 1) & 3),
// which keeps both the writes and the reads free of bank conflicts. Rows at
// or past row_end and columns at or past N (N % 8 == 0) are not written.
constexpr int kStageChunkBytes = 32 * 64;
// Epilogue staging of the single-SM tile kernel: one chunk per epilogue warp,
// then the tile's column scales for each of the two accumulators (the pair
// kernel stages 128 column scales per warp instead).
constexpr int kEpiStgBytes = 8 * kStageChunkBytes + 2 * 256 * 4;

__device__ __forceinline__ void store_chunk_coalesced(uint8_t* stg, const uint4 (&pk)[4],
                                                      uint16_t* __restrict__ y, int64_t row0,
                                                      int64_t row_end, int N, int n0, int lane) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(stg + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4)) = pk[q];
  __syncwarp();
  const int q = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = i * 8 + (lane >> 2);
    const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * 64 + ((q ^ ((rr >> 1) & 3)) << 4));
    const int64_t row = row0 + rr;
    if (row < row_end && n0 + q * 8 < N)
      *reinterpret_cast<uint4*>(y + row * static_cast<int64_t>(N) + n0 + q * 8) = v;
  }
  __syncwarp();  // the buffer is rewritten by the next chunk
}

// A warp's epilogue staging buffers (one, or two used in turn): `last` is
// the buffer the most recently committed TMA store reads (-1: none yet).
struct StgRing {
  uint8_t* base;
  int nbuf;
  int turn;
  int last;
  __device__ __forceinline__ uint8_t* buf(int b) const { return base + b * kStageChunkBytes; }
};

// Store of one 32 x 32 bf16 chunk a warp holds one row per lane (pk = the
// lane's 64 bytes; `row` = this lane's row): one TMA store of the swizzled
// staging buffer when tma_ok (warp-uniform: the map covers y and all 32 rows
// belong to the tile's rows; the map clips columns at N), else through
// store_chunk_coalesced. A buffer is rewritten only after every store that
// reads it has done so: with two buffers, when the latest store reads the
// other one, every store but that latest one - so staging a chunk overlaps
// the previous chunk's store.
__device__ __forceinline__ void epi_store_chunk(const uint4 (&pk)[4], StgRing& ring,
                                                uint16_t* __restrict__ y, int row, int64_t row_end,
                                                int N, int n0, int lane, const CUtensorMap* tmY,
                                                bool tma_ok) {
  const int b = ring.turn;
  uint8_t* stg = ring.buf(b);
  if (lane == 0) {
    if (ring.nbuf > 1 && ring.last != b)
      bulk_wait_group_read_but_last();
    else
      bulk_wait_group_read_all();
  }
  __syncwarp();
  if (tma_ok) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      *reinterpret_cast<uint4*>(stg + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4)) = pk[q];
    fence_proxy_async_shared();  // generic writes -> visible to the TMA store
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmY, smem_u32(stg), n0, row - lane);
      bulk_commit_group();
    }
    ring.last = b;
    if (ring.nbuf > 1) ring.turn ^= 1;
  } else {
    store_chunk_coalesced(stg, pk, y, row - lane, row_end, N, n0, lane);
  }
}

// One 32-column chunk of the epilogue: a warp's 32 accumulator rows (r =
// this lane's row `row`), scaled by s_a of the row and the chunk's 32 column
// scales (sb_chunk, staged in shared memory), rounded to bf16 and stored -
// through store_chunk_coalesced when rows are 16-byte storable (warp-uniform
// vec_ok), else element by element.
//
// With tma_ok (warp-uniform: a store tensor map over y exists and all 32
// rows of the chunk belong to the tile's row range) the staged chunk leaves
// by one TMA store instead (the staging layout is the map's 64-byte swizzle;
// the map clips columns at N); the buffer is reused only after the previous
// store from it has read it.
__device__ __forceinline__ void epi_chunk(const uint32_t (&r)[32], const float* sb_chunk,
                                          float sa, bool vec_ok,
                                          StgRing& stg, uint16_t* __restrict__ y, int row,
                                          int64_t row_end, int N, int n0, int lane,
                                          const CUtensorMap* tmY, bool tma_ok) {
  if (n0 >= N) return;
  if (vec_ok) {
    uint4 pk[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 b0 = reinterpret_cast<const float4*>(sb_chunk)[2 * q];
      const float4 b1 = reinterpret_cast<const float4*>(sb_chunk)[2 * q + 1];
      const float sb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {  // v = (acc * s_a) * s_b, two values per instruction
        fmul2_rn(v[i], v[i + 1], __uint_as_float(r[8 * q + i]), __uint_as_float(r[8 * q + i + 1]), sa, sa);
        fmul2_rn(v[i], v[i + 1], v[i], v[i + 1], sb[i], sb[i + 1]);
      }
      pk[q] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                         pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
    }
    epi_store_chunk(pk, stg, y, row, row_end, N, n0, lane, tmY, tma_ok);
  } else if (row < row_end) {
    uint16_t* yrow = y + static_cast<int64_t>(row) * N;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (n0 + j < N) {
        const float v = __fmul_rn(__fmul_rn(__uint_as_float(r[j]), sa), sb_chunk[j]);
        yrow[n0 + j] = f32_to_bf16_rn(v);
      }
    }
  }
}

// K blocking of the prefill kernels: 128-byte k-blocks, each four 32-deep
// MMA k-steps. When K is not a multiple of 128 but is one of 32 (and
// K > 128), the last k-block is loaded at K - 128, wholly inside the operands,
// and its first k-steps - the columns the previous block already covered -
// are not issued. Every column enters the sum once, in the same order, and
// the partly out-of-range TMA box (whose zero fill costs more than a full
// box) is never requested.
struct KBlocking {
  int num_kb;
  int last_x;   // K coordinate of the last k-block
  int last_k0;  // first MMA k-step of the last k-block
  __device__ __forceinline__ int x(int kb) const { return kb == num_kb - 1 ? last_x : kb * kBK; }
};

__device__ __forceinline__ KBlocking k_blocking(int K) {
  KBlocking b;
  b.num_kb = (K + kBK - 1) / kBK;
  const int tail = K % kBK;
  if (tail != 0 && tail % 32 == 0 && K > kBK) {
    b.last_x = K - kBK;
    b.last_k0 = (kBK - tail) / 32;
  } else {
    b.last_x = (b.num_kb - 1) * kBK;
    b.last_k0 = 0;
  }
  return b;
}

// Tile order: groups of `group_m` row tiles; inside a group, row tiles vary
// fastest, then column tiles.
__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int group_m,
                                            int& tm, int& tn) {
  const int per_group = group_m * tiles_n;
  const int g = tile / per_group;
  const int first_m = g * group_m;
  const int gm = min(tiles_m - first_m, group_m);
  const int local = tile - g * per_group;
  tm = first_m + local % gm;
  tn = local / gm;
}

// ============================================================== prefill
template <int BN, int STAGES>
struct PrefillCfg {
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = BN * kBK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = tmem_cols_for(2 * BN);
  static constexpr int kBarBytes = 8 * (2 * STAGES + 4) + 16;
  static constexpr int kStgBytes = kEpiStgBytes;  // epilogue staging (chunks, column scales)
  static constexpr size_t kSmem =
      1024 + static_cast<size_t>(STAGES) * kStageBytes + kStgBytes + kBarBytes;
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
};

// Largest number of experts the grouped GEMM handles (its m-tile prefix
// lives in shared memory).
constexpr int kMaxExperts = 1024;
// Dynamic shared memory a grouped launch adds for E experts: the m-tile
// prefix and a copy of the row offsets, E + 1 ints each.
constexpr size_t grouped_smem_bytes(int E) { return 8 * (static_cast<size_t>(E) + 1); }

// Arguments shared by the dense and the grouped (per-expert) GEMM.
//  dense:   A rows [0, M), B rows [0, N); tiles walked in groups of group_m.
//  grouped: expert e owns A rows offsets[e]..offsets[e+1] and B rows
//           e*N..e*N+N (weights stacked [E*N, K], scales [E*N]).
struct GemmArgs {
  const float* s_a;
  const float* s_b;
  uint16_t* y;
  int M, N, K;
  int tiles_m, tiles_n, group_m;
  const int* offsets;  // grouped only
  int num_experts;     // grouped only
  int use_tma_store;   // tmY is a 32 x 32 bf16 store map over y (64-byte swizzle)
  int n_out;           // GeGLU epilogue only: columns of h (the features)
  // Split (stream-K) launches of the dense pair GEMM only: the last
  // sk_tiles tiles are shared out by k-blocks (see PairItems), partial
  // accumulators passing through ws_part with per-warp flags ws_flag.
  int sk_tiles;
  uint32_t* ws_part;
  int* ws_flag;
};

struct Tile {
  int a_row;    // first A row (TMA coordinate)
  int row_end;  // rows >= row_end belong to another expert / are out of range
  int b_row;    // first B row (TMA coordinate)
  int col0;     // first output column
  int sb_off;   // offset of this tile's expert in s_b
};

// Tile t of the grouped problem: m-tiles of tile_rows rows are numbered
// expert by expert (mt_off[e] = first m-tile of expert e), n-tiles vary
// fastest. The experts' row offsets are read from their shared-memory copy
// (row_off = mt_off + E + 1), so decoding a tile touches no global memory.
// Each thread decodes its tiles in increasing order, so the expert index only
// moves forward: `e` carries it from one call to the next (start at 0) and is
// advanced to the expert with mt_off[e] <= m-tile < mt_off[e + 1] - usually a
// step or two, at most E steps over all of a thread's tiles.
__device__ __forceinline__ Tile grouped_tile(const GemmArgs& g, const int* mt_off, int t, int BN,
                                             int tile_rows, int& e) {
  const int* row_off = mt_off + g.num_experts + 1;
  const int gmt = t / g.tiles_n, tn = t - (t / g.tiles_n) * g.tiles_n;
  while (mt_off[e + 1] <= gmt) ++e;  // t < mt_off[E] * tiles_n, so this stops at e < E
  Tile T;
  T.a_row = row_off[e] + (gmt - mt_off[e]) * tile_rows;
  T.row_end = row_off[e + 1];
  T.b_row = e * g.N + tn * BN;
  T.col0 = tn * BN;
  T.sb_off = e * g.N;
  return T;
}

// mt_off[e] = number of tile_rows-row m-tiles of experts 0..e-1 (mt_off[E]
// = total), from the row offsets, and mt_off[E + 1 + e] = offsets[e] (e = 0..E,
// the copy grouped_tile reads); one warp. The offsets may come from a
// preceding routing grid, so the warp waits for it first. An expert whose
// row range is not inside [0, M) (or runs backwards) gets no tiles and sets
// FP8_DEV_BAD_INDEX, so no tile can read or write outside x, s_a or y.
__device__ __forceinline__ int grouped_expert_rows(const GemmArgs& g, int e) {
  const int lo = g.offsets[e], hi = g.offsets[e + 1];
  if (lo < 0 || hi < lo || hi > g.M) {
    report(FP8_DEV_BAD_INDEX);
    return 0;
  }
  return hi - lo;
}

__device__ __forceinline__ void grouped_prefix(const GemmArgs& g, int* mt_off, int tile_rows,
                                               int lane) {
  pdl_wait();
  const int E = g.num_experts;
  const int per = (E + 31) / 32;
  int sum = 0;
  for (int i = 0; i < per; ++i) {
    const int e = lane * per + i;
    if (e < E) sum += (grouped_expert_rows(g, e) + tile_rows - 1) / tile_rows;
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
      mt_off[e] = run;
      run += (grouped_expert_rows(g, e) + tile_rows - 1) / tile_rows;
    }
  }
  if (lane == 31) mt_off[E] = incl;
  for (int e = lane; e <= E; e += 32) mt_off[E + 1 + e] = g.offsets[e];
}

__device__ __forceinline__ Tile dense_tile(const GemmArgs& g, int t, int BN) {
  int tm, tn;
  tile_coords(t, g.tiles_m, g.tiles_n, g.group_m, tm, tn);
  Tile T;
  T.a_row = tm * kBM;
  T.row_end = g.M;
  T.b_row = tn * BN;
  T.col0 = tn * BN;
  T.sb_off = 0;
  return T;
}

// Warps: 0 = TMA producer, 1 = MMA issuer + TMEM owner, 2..9 = epilogue (two
// warps per TMEM lane quadrant, each draining half of the tile's columns).
constexpr int kEpiWarps = 8;
constexpr int kPrefillThreads = 64 + 32 * kEpiWarps;

template <int BN, int STAGES, bool GROUPED, int KD = kKindE4M3>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    gemm_prefill_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmY, const GemmArgs g) {
  using C = PrefillCfg<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::kABytes;
  uint8_t* stg_all = sB + STAGES * C::kBBytes;  // epilogue staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg_all + C::kStgBytes);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  // grouped: 2 * (E + 1) ints after the barriers and the TMEM holder (the
  // launch adds grouped_smem_bytes(E) of dynamic shared memory for them)
  int* mt_off = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(bars) + C::kBarBytes);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * STAGES);
  const uint32_t tempty0 = smem_u32(bars + 2 * STAGES + 2);

  const int warp = warp_id(), lane = lane_id();
  const KBlocking kblk = k_blocking(g.K);
  const int num_kb = kblk.num_kb;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, kEpiWarps);
    }
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  if constexpr (GROUPED) {
    if (warp == 2) grouped_prefix(g, mt_off, kBM, lane);  // m-tiles of 128 rows
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int num_tiles = GROUPED ? mt_off[g.num_experts] * g.tiles_n : g.tiles_m * g.tiles_n;
  int e_seen = 0;  // this thread's expert cursor (tiles are decoded in increasing order)
  auto tile_of = [&](int t) {
    return GROUPED ? grouped_tile(g, mt_off, t, BN, kBM, e_seen) : dense_tile(g, t, BN);
  };

  if (warp == 0) {
    if (lane == 0) {
      pdl_wait();  // activations may come from a preceding quantizer grid
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const Tile T = tile_of(tile);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1)) { ok = false; break; }
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, C::kStageBytes);
          tma_load_2d(smem_u32(sA + stage * C::kABytes), &tmA, fb, kblk.x(kb), T.a_row, 0ull);
          tma_load_2d(smem_u32(sB + stage * C::kBBytes), &tmB, fb, kblk.x(kb), T.b_row, 0ull);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_kind<KD>(kBM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        // one k-block's MMAs from k-step k0 on (k0 > 0 only for a shifted last block)
        auto kblock = [&](int kb, int k0) {
          if (!mbar_wait(full0 + 8 * stage, phase)) return false;
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::kABytes);
          const uint32_t b0 = smem_u32(sB + stage * C::kBBytes);
#pragma unroll
          for (int k = k0; k < kBK / 32; ++k) {
            umma_kind<KD>(d_tmem, sw128_kmajor_desc(a0 + 32 * k), sw128_kmajor_desc(b0 + 32 * k),
                          idesc, (kb | k) != 0);
          }
          umma_commit(empty0 + 8 * stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
          return true;
        };
        // the hot loop keeps constant k-steps; a shifted last block is peeled off
        const int kb_full = kblk.last_k0 != 0 ? num_kb - 1 : num_kb;
        for (int kb = 0; ok && kb < kb_full; ++kb) ok = kblock(kb, 0);
        if (ok && kb_full < num_kb) ok = kblock(num_kb - 1, kblk.last_k0);
        umma_commit(tfull0 + 8 * acc);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else {
    // Epilogue warps 2..9; a warp may only touch TMEM lanes 32*(warp%4)..+31,
    // and warps w and w+4 share a quadrant, splitting its column chunks.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    StgRing stg = {stg_all + (warp - 2) * kStageChunkBytes, 1, 0, -1};  // this warp's staging chunk
    float* sb_tile = reinterpret_cast<float*>(stg_all + 8 * kStageChunkBytes);  // [2][256]
    const int N = g.N;
    // 16-byte stores of y rows and 16-byte loads of the column scales
    const bool vec_ok = (N % 8) == 0 && (reinterpret_cast<uintptr_t>(g.s_b) & 15) == 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool waited = false;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const Tile T = tile_of(tile);
      {
        // The tile's column scales into this accumulator's buffer, one per
        // epilogue thread (weight-side data, read before the tile is done;
        // every warp left the buffer's previous tile before the last barrier).
        const int col = T.col0 + (threadIdx.x - 64);
        sb_tile[acc * 256 + (threadIdx.x - 64)] =
            col < N ? (g.s_b ? __ldg(g.s_b + T.sb_off + col) : 1.0f) : 0.0f;
      }
      const bool got = mbar_wait(tfull0 + 8 * acc, acc_phase);
      // all epilogue warps: scales visible; leave together if any wait failed
      if (named_bar_or(2, 32 * kEpiWarps, !got)) break;
      tc_fence_after();
      if (!waited) { pdl_wait(); waited = true; }
      const int row = T.a_row + quad * 32 + lane;
      const float sa = row < T.row_end ? (g.s_a ? __ldg(g.s_a + row) : 1.0f) : 0.0f;
      // whole 32-row chunk inside the tile's rows: one TMA store per chunk
      const bool tma_rows = g.use_tma_store && (row - lane) + 32 <= T.row_end;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN;
      constexpr int kCh = BN / 64;  // 32-column chunks per warp
#pragma unroll 1
      for (int c = half * kCh; c < (half + 1) * kCh; ++c) {
        uint32_t r[32];
        tmem_ld32(t_row + c * 32, r);
        tmem_ld_wait();
        acc_to_f32<KD>(r);
        epi_chunk(r, sb_tile + acc * 256 + c * 32, sa, vec_ok, stg, g.y, row, T.row_end, N,
                  T.col0 + c * 32, lane, &tmY, tma_rows);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (lane == 0) bulk_wait_group_all();  // this warp's TMA stores of y are complete
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Work items of one CTA pair of a persistent pair GEMM, in the order the
// pair takes them. Tiles [0, T_dp) are whole tiles dealt round-robin (tile
// p, p + P, ...). With a split, the last T - T_dp tiles (a full wave and
// the partial last one) are cut into k-blocks, U in all, and pair p takes
// the run [U p / P, U (p + 1) / P) of them in tile order, so every pair
// does the same number of k-blocks (to one) instead of the last wave
// leaving most pairs idle. A run of at least one tile's k-blocks (T - T_dp
// >= P) starts with the end of one tile (a part: its fp32 or int32
// accumulator goes to the workspace), then whole tiles, then the start of
// another tile (owned: this pair adds the parts of the later k-blocks,
// written by the next pair(s), and stores the tile). The owned piece is
// the pair's last item and a part its first, so an owner's parts have
// usually been written by the time it needs them.
struct WorkItem {
  int tile, kb0, kb1;  // k-blocks [kb0, kb1) of the tile
  int role;            // kWhole, kOwned or kPart
};
constexpr int kWhole = 0, kOwned = 1, kPart = 2;

struct PairItems {
  int P, T_dp, nkb, U;
  int dp, u, u_end;
  __device__ __forceinline__ int u_lo(int q) const {
    return static_cast<int>((static_cast<long long>(U) * q) / P);
  }
  __device__ __forceinline__ void init(int p, int P_, int T, int sk_tiles, int nkb_) {
    P = P_;
    nkb = nkb_;
    T_dp = T - sk_tiles;
    U = sk_tiles * nkb;
    dp = p;
    u = u_lo(p);
    u_end = u_lo(p + 1);
  }
  __device__ __forceinline__ bool next(WorkItem& w) {
    if (dp < T_dp) {
      w.tile = dp;
      w.kb0 = 0;
      w.kb1 = nkb;
      w.role = kWhole;
      dp += P;
      return true;
    }
    if (u >= u_end) return false;
    const int ts = u / nkb;
    w.tile = T_dp + ts;
    w.kb0 = u - ts * nkb;
    w.kb1 = min(nkb, w.kb0 + (u_end - u));
    w.role = w.kb0 > 0 ? kPart : (w.kb1 == nkb ? kWhole : kOwned);
    u += w.kb1 - w.kb0;
    return true;
  }
};

// Workspace of a split launch: per pair q, CTA rank r and epilogue warp w
// one flag, and per (q, r) a 128 x 256 word accumulator part (16 KB per
// epilogue warp, laid out so that the warp's accesses are contiguous).
__host__ __device__ constexpr size_t split_flag_bytes(int pairs) {
  return (static_cast<size_t>(pairs) * 2 * 8 * 4 + 255) / 256 * 256;
}
__host__ __device__ constexpr size_t split_ws_bytes(int pairs) {
  return split_flag_bytes(pairs) + static_cast<size_t>(pairs) * 2 * 128 * 256 * 4;
}

// Bounded wait for a flag another CTA sets with release semantics (acquire
// load); false (and FP8_DEV_TIMEOUT) when the limit runs out.
__device__ __forceinline__ bool wait_flag_set(const int* flag) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
  if (v != 0) return true;
  const long long lim = *const_cast<volatile long long*>(&g_wait_limit);
  const long long t0 = clock64();
  for (;;) {
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v != 0) return true;
    if (clock64() - t0 > lim) {
      report(FP8_DEV_TIMEOUT);
      return false;
    }
  }
}
__device__ __forceinline__ void set_flag_release(int* flag, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(v) : "memory");
}

// ============================================================== prefill, CTA pair
// Dense GEMM on 256 x 256 output tiles computed by a cluster of two CTAs on
// two SMs with tcgen05.mma.cta_group::2: each CTA stages 128 rows of A (its
// half of the tile's rows) and 128 rows of B (its half of the tile's
// columns), so every SM moves 32 KB per 128-deep k-block for a 256 x 256 x
// 128 product - two thirds of the operand traffic of a 128 x 256 single-SM
// tile per unit of work. The even CTA's MMA thread issues the pair MMAs; both
// CTAs' TMA loads complete on the even CTA's full barrier; each MMA commit is
// multicast to the stage's empty barrier (or the accumulator's full barrier)
// in both CTAs; each CTA drains its own 128 TMEM lanes (its 128 rows), and the
// even CTA's accumulator-empty barrier counts the epilogue warps of both.
template <int STAGES, int STG_BUFS = 1>
struct PairCfg {
  static constexpr int kHalf = 128;                  // rows of A and of B per CTA
  static constexpr int kBN = 256;                    // tile columns
  static constexpr int kABytes = kHalf * kBK;
  static constexpr int kBBytes = kHalf * kBK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 512;              // two 256-column accumulators
  static constexpr int kBarBytes = 8 * (2 * STAGES + 4) + 16;
  // epilogue staging: STG_BUFS 2 KB chunks and 128 column scales per epilogue
  // warp
  static constexpr int kStgBytes = kEpiWarps * (STG_BUFS * kStageChunkBytes + 128 * 4);
  static constexpr size_t kSmem =
      1024 + static_cast<size_t>(STAGES) * kStageBytes + kStgBytes + kBarBytes;
};

//
// GROUPED: the per-expert GEMM on the same pairs. Expert e's rows are cut
// into 256-row pair tiles (the last one masked at the expert's end); the
// tiles are decoded on the GPU from the row offsets as in the single-SM
// grouped kernel.
//
// GEGLU (grouped only): B holds each expert's gate and up rows interleaved
// in blocks of 128 (tile tn = gate rows of features 128 tn .. 128 tn + 127,
// then up rows of the same features), so a tile's accumulator has gate and
// up of 128 features side by side; the epilogue rounds both to bf16 as the
// plain GEMM would store them and writes h = bf16(gelu_tanh(gate) * up)
// [M_total, n_out] instead. A last feature tile with at most 64 features
// is half width: each CTA loads 64 B rows (through tmBh, a map with 64-row
// boxes) and the MMAs run with N = 128, so the leader's gate rows fill
// accumulator columns 0..63 and the peer's up rows columns 64..127.
// Grouped launches (short K per expert tile, so the epilogue sets the pace)
// give each epilogue warp two staging buffers.
template <bool GROUPED>
__host__ __device__ constexpr int pair_stg_bufs() { return GROUPED ? 2 : 1; }

template <int STAGES, bool GROUPED = false, bool GEGLU = false, int KD = kKindE4M3, bool SPLIT = false>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmBh, const __grid_constant__ CUtensorMap tmY,
                     const GemmArgs g) {
  constexpr int kStgBufs = pair_stg_bufs<GROUPED>();
  using C = PairCfg<STAGES, kStgBufs>;
  static_assert(GROUPED || !GEGLU, "the GeGLU epilogue is for the grouped GEMM");
  static_assert(!GEGLU || KD == kKindE4M3, "the GeGLU epilogue is for E4M3 operands");
  static_assert(!SPLIT || !GROUPED, "the k-block split is for the dense GEMM");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::kABytes;
  uint8_t* stg_all = sB + STAGES * C::kBBytes;  // epilogue staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg_all + C::kStgBytes);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  // grouped: 2 * (E + 1) ints after the barriers (the launch adds grouped_smem_bytes(E))
  int* mt_off = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(bars) + C::kBarBytes);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * STAGES);
  const uint32_t tempty0 = smem_u32(bars + 2 * STAGES + 2);

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();        // 0 = leader (issues the MMAs)
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const KBlocking kblk = k_blocking(g.K);
  const int num_kb = kblk.num_kb;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 2 * kEpiWarps);
    }
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (GEGLU) tma_prefetch_desc(&tmBh);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), C::kTmemCols);
    tmem_relinquish_pair();
  }
  if constexpr (GROUPED) {
    if (warp == 2) grouped_prefix(g, mt_off, 256, lane);  // pair m-tiles of 256 rows
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrive or load
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // tiles of 256 x 256; the fields of a Tile here are the pair's (row 0 of
  // the tile, column 0), each CTA adding rank * 128 to its A and B rows
  const int num_tiles = GROUPED ? mt_off[g.num_experts] * g.tiles_n : g.tiles_m * g.tiles_n;
  // GeGLU: the last feature tile holds at most 64 features (tiles are
  // numbered m-tile major, so tile % tiles_n is the feature tile)
  auto half_width = [&](int t) { return GEGLU && g.n_out - 128 * (t % g.tiles_n) <= 64; };
  int e_seen = 0;  // this thread's expert cursor (tiles are decoded in increasing order)
  auto tile_of = [&](int t) {
    if constexpr (GROUPED) {
      return grouped_tile(g, mt_off, t, C::kBN, 256, e_seen);
    } else {
      int tm, tn;
      tile_coords(t, g.tiles_m, g.tiles_n, g.group_m, tm, tn);
      Tile T;
      T.a_row = tm * 256;
      T.row_end = g.M;
      T.b_row = tn * C::kBN;
      T.col0 = tn * C::kBN;
      T.sb_off = 0;
      return T;
    }
  };

  if (warp == 0) {
    if (lane == 0) {
      pdl_wait();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      PairItems items;
      items.init(pair, npairs, num_tiles, SPLIT ? g.sk_tiles : 0, num_kb);
      WorkItem w;
      while (ok && items.next(w)) {
        const int tile = w.tile;
        const Tile T = tile_of(tile);
        const int a_row = T.a_row + rank * C::kHalf;
        const int b_row = T.b_row + rank * C::kHalf;
        const bool half = half_width(tile);  // 64 B rows per CTA
        const CUtensorMap* mapB = half ? &tmBh : &tmB;
        const uint32_t stage_tx = 2 * (C::kABytes + (half ? C::kBBytes / 2 : C::kBBytes));
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1)) { ok = false; break; }
          const uint32_t fb_local = full0 + 8 * stage;
          const uint32_t fb_leader = mapa_shared(fb_local, 0);
          // Both CTAs' bytes complete on the leader's full barrier.
          if (rank == 0) mbar_arrive_expect_tx(fb_local, stage_tx);
          tma_load_2d_pair(smem_u32(sA + stage * C::kABytes), &tmA, fb_leader, kblk.x(kb), a_row);
          tma_load_2d_pair(smem_u32(sB + stage * C::kBBytes), mapB, fb_leader, kblk.x(kb), b_row);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t kIdescFull = idesc_kind<KD>(256, C::kBN);
      constexpr uint32_t kIdescHalf = idesc_kind<KD>(256, C::kBN / 2);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      PairItems items;
      items.init(pair, npairs, num_tiles, SPLIT ? g.sk_tiles : 0, num_kb);
      WorkItem w;
      while (ok && items.next(w)) {
        const int tile = w.tile;
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * C::kBN;
        const uint32_t idesc = half_width(tile) ? kIdescHalf : kIdescFull;
        // one k-block's MMAs from k-step k0 on (k0 > 0 only for a shifted
        // last block); the item's first MMA overwrites the accumulator
        auto kblock = [&](int kb, int k0) {
          if (!mbar_wait(full0 + 8 * stage, phase)) return false;
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::kABytes);
          const uint32_t b0 = smem_u32(sB + stage * C::kBBytes);
#pragma unroll
          for (int k = k0; k < kBK / 32; ++k) {
            umma_kind_pair<KD>(d_tmem, sw128_kmajor_desc(a0 + 32 * k), sw128_kmajor_desc(b0 + 32 * k),
                               idesc, kb != w.kb0 || k != k0);
          }
          umma_commit_pair(empty0 + 8 * stage, 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
          return true;
        };
        // the hot loop keeps constant k-steps; a shifted last block is peeled off
        const int kb_full = (w.kb1 == num_kb && kblk.last_k0 != 0) ? num_kb - 1 : w.kb1;
        for (int kb = w.kb0; ok && kb < kb_full; ++kb) ok = kblock(kb, 0);
        if (ok && kb_full < w.kb1) ok = kblock(num_kb - 1, kblk.last_k0);
        umma_commit_pair(tfull0 + 8 * acc, 0x3);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else {
    // Epilogue warps 2..9 of each CTA drain that CTA's 128 TMEM lanes: warp
    // (quad, half) takes TMEM lane quadrant quad (32 rows) and half of the
    // tile's columns. Each warp stages its own 128 column scales (GeGLU: its
    // 64 gate and 64 up columns), so the warps of a tile never wait for one
    // another: a tile is a TMEM-full wait, the warp's chunks and an arrive.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    // this warp's staging chunk(s), used in turn
    StgRing stg = {stg_all + (warp - 2) * kStgBufs * kStageChunkBytes, kStgBufs, 0, -1};
    float* sbw =
        reinterpret_cast<float*>(stg_all + kEpiWarps * kStgBufs * kStageChunkBytes) + (warp - 2) * 128;
    const int N = g.N;
    // 16-byte stores of y rows and 16-byte loads of the column scales
    const bool vec_ok = (N % 8) == 0 && (reinterpret_cast<uintptr_t>(g.s_b) & 15) == 0;
    const uint32_t tempty_leader0 = mapa_shared(tempty0, 0);
    // this lane's 4 of the warp's 128 column scales (tile-relative column)
    const int scol = GEGLU ? (lane < 16 ? half * 64 + 4 * lane : 128 + half * 64 + 4 * (lane - 16))
                           : half * 128 + 4 * lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    // Tiles are drained in the order the MMAs produce them, with their
    // coordinates and scales fetched ahead: the tile after next is decoded
    // and the next tile's s_a and s_b are loaded while the current tile
    // drains, so no global-load latency sits between tiles (with short K the
    // epilogue paces the kernel).
    pdl_wait();  // s_a and the expert offsets may come from the preceding grid
    auto fetch_scales = [&](const Tile& Tt, float4& sbv, float& sav) {
      const int col = Tt.col0 + scol;
      const float* src = g.s_b + Tt.sb_off + col;
      if (!g.s_b) {  // unscaled columns
        sbv.x = col < N ? 1.0f : 0.0f;
        sbv.y = col + 1 < N ? 1.0f : 0.0f;
        sbv.z = col + 2 < N ? 1.0f : 0.0f;
        sbv.w = col + 3 < N ? 1.0f : 0.0f;
      } else if (vec_ok) {  // N % 8 == 0: the lane's 4 columns are all inside N or all past it
        sbv = col < N ? __ldg(reinterpret_cast<const float4*>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        sbv.x = col < N ? __ldg(src) : 0.0f;
        sbv.y = col + 1 < N ? __ldg(src + 1) : 0.0f;
        sbv.z = col + 2 < N ? __ldg(src + 2) : 0.0f;
        sbv.w = col + 3 < N ? __ldg(src + 3) : 0.0f;
      }
      const int rr = Tt.a_row + rank * C::kHalf + quad * 32 + lane;
      sav = rr < Tt.row_end ? (g.s_a ? __ldg(g.s_a + rr) : 1.0f) : 0.0f;
    };
    PairItems ahead;  // this pair's items, decoded two ahead of the one drained
    ahead.init(pair, npairs, num_tiles, SPLIT ? g.sk_tiles : 0, num_kb);
    WorkItem w = {}, w1 = {}, w2 = {};
    bool has = ahead.next(w);
    bool has1 = has && ahead.next(w1);
    Tile T = {}, T1 = {};
    float4 sb_v = make_float4(0.f, 0.f, 0.f, 0.f);
    float sa = 0.0f;
    if (has) {
      T = tile_of(w.tile);
      fetch_scales(T, sb_v, sa);
    }
    if (has1) T1 = tile_of(w1.tile);
    while (has) {
      const int tile = w.tile;
      float4 sb_v1 = make_float4(0.f, 0.f, 0.f, 0.f);
      float sa1 = 0.0f;
      if (has1) fetch_scales(T1, sb_v1, sa1);
      const bool has2 = has1 && ahead.next(w2);
      const Tile T2 = has2 ? tile_of(w2.tile) : T1;
      // this tile's column scales into the warp's buffer (its lanes finished
      // reading the previous tile's before the last __syncwarp)
      *reinterpret_cast<float4*>(sbw + 4 * lane) = sb_v;
      const bool got = mbar_wait(tfull0 + 8 * acc, acc_phase);
      __syncwarp();  // the scales are visible to the whole warp
      if (!__all_sync(0xFFFFFFFFu, got)) break;
      tc_fence_after();
      const int row = T.a_row + rank * C::kHalf + quad * 32 + lane;
      // whole 32-row chunk inside the tile's rows: one TMA store per chunk
      const bool tma_rows = g.use_tma_store && (row - lane) + 32 <= T.row_end;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * C::kBN;
      if constexpr (GEGLU) {
        // accumulator columns 0..127: gate of the tile's 128 features,
        // 128..255: their up (a half-width tile: 0..63 and 64..127); this
        // warp takes 64 features in two chunks
        const int f_base = T.col0 >> 1;
        const int up_col = half_width(tile) ? 64 : 128;
#pragma unroll 1
        for (int fc = half * 2; fc < half * 2 + 2; ++fc) {
          const int f0 = f_base + fc * 32;
          if (f0 >= g.n_out) continue;  // warp-uniform
          uint32_t rg[32], ru[32];
          tmem_ld32(t_row + fc * 32, rg);
          tmem_ld32(t_row + up_col + fc * 32, ru);
          tmem_ld_wait();
          const float* sbg = sbw + (fc - half * 2) * 32;
          const float* sbu = sbg + 64;
          uint4 pk[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float gv[8], uv[8], hv[8];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
              const int j = 8 * q + i;
              // gate and up exactly as the plain GEMM stores them in bf16
              fmul2_rn(gv[i], gv[i + 1], __uint_as_float(rg[j]), __uint_as_float(rg[j + 1]), sa, sa);
              fmul2_rn(gv[i], gv[i + 1], gv[i], gv[i + 1], sbg[j], sbg[j + 1]);
              fmul2_rn(uv[i], uv[i + 1], __uint_as_float(ru[j]), __uint_as_float(ru[j + 1]), sa, sa);
              fmul2_rn(uv[i], uv[i + 1], uv[i], uv[i + 1], sbu[j], sbu[j + 1]);
            }
            float gb[8], ub[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              gb[i] = __uint_as_float(static_cast<uint32_t>(f32_to_bf16_rn(gv[i])) << 16);
              ub[i] = __uint_as_float(static_cast<uint32_t>(f32_to_bf16_rn(uv[i])) << 16);
            }
            geglu8_f32(gb, ub, hv);
            pk[q] = make_uint4(pack_bf16x2(hv[0], hv[1]), pack_bf16x2(hv[2], hv[3]),
                               pack_bf16x2(hv[4], hv[5]), pack_bf16x2(hv[6], hv[7]));
          }
          epi_store_chunk(pk, stg, g.y, row, T.row_end, g.n_out, f0, lane, &tmY, tma_rows);
        }
      } else {
        constexpr int kCh = 4;  // 32-column chunks per warp
        // split items: this warp's flag and its rows of a pair's part
        const int wslot = (warp - 2);
        // a warp's part: its 4 chunks x 8 16-byte vectors x 32 lanes, the
        // lanes of one vector contiguous (each warp access is 512 bytes)
        auto part_at = [&](int q, int c) {
          return reinterpret_cast<uint4*>(g.ws_part) +
                 (((static_cast<size_t>(q) * 2 + rank) * 8 + wslot) * kCh + (c - half * kCh)) * 8 * 32 + lane;
        };
        auto flag_at = [&](int q) { return g.ws_flag + (q * 2 + static_cast<int>(rank)) * 8 + wslot; };
        // an owned piece's parts: pairs pair+1 .. q_end-1 (the later k-blocks, in order)
        int q_end = pair + 1;
        const bool is_part = SPLIT && w.role == kPart;
        if constexpr (SPLIT) {
          if (w.role == kOwned) {
            const int tile_end_u = (tile - ahead.T_dp + 1) * ahead.nkb;
            while (q_end < npairs && ahead.u_lo(q_end) < tile_end_u) ++q_end;
            if (lane == 0)
              for (int q = pair + 1; q < q_end; ++q) wait_flag_set(flag_at(q));
            __syncwarp();
          }
        }
#pragma unroll 1
        for (int c = half * kCh; c < (half + 1) * kCh; ++c) {
          if (SPLIT && T.col0 + c * 32 >= N) continue;  // warp-uniform; no part either
          // owned: the next pair's part of this chunk is requested before the
          // TMEM load, so that the two latencies overlap (usually one part)
          uint4 pv0[8];
          if constexpr (SPLIT) {
            if (w.role == kOwned && q_end > pair + 1) {
              const uint4* src = part_at(pair + 1, c);
#pragma unroll
              for (int v = 0; v < 8; ++v) pv0[v] = __ldcg(src + 32 * v);
            }
          }
          uint32_t r[32];
          tmem_ld32(t_row + c * 32, r);
          tmem_ld_wait();
          if constexpr (SPLIT) {
            if (is_part) {  // raw accumulator words to the workspace
              uint4* dst = part_at(pair, c);
#pragma unroll
              for (int v = 0; v < 8; ++v)
                __stcg(dst + 32 * v, make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]));
              continue;
            }
            // owned: add the later k-blocks' parts in pair order (int32
            // sums for kind::i8, exact; fp32 otherwise)
            for (int q = pair + 1; q < q_end; ++q) {
              uint4 pvs[8];
              if (q == pair + 1) {
#pragma unroll
                for (int v = 0; v < 8; ++v) pvs[v] = pv0[v];
              } else {
                const uint4* src = part_at(q, c);
#pragma unroll
                for (int v = 0; v < 8; ++v) pvs[v] = __ldcg(src + 32 * v);
              }
#pragma unroll
              for (int v = 0; v < 8; ++v) {
                const uint4 pv = pvs[v];
                const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  uint32_t& x = r[4 * v + j];
                  if constexpr (KD == kKindS8)
                    x = static_cast<uint32_t>(static_cast<int>(x) + static_cast<int>(pw[j]));
                  else
                    x = __float_as_uint(__fadd_rn(__uint_as_float(x), __uint_as_float(pw[j])));
                }
              }
            }
          }
          acc_to_f32<KD>(r);
          epi_chunk(r, sbw + (c - half * kCh) * 32, sa, vec_ok, stg, g.y, row, T.row_end, N,
                    T.col0 + c * 32, lane, &tmY, tma_rows);
        }
        if constexpr (SPLIT) {
          if (w.role == kPart) {  // this warp's rows of the part are written
            __threadfence();
            __syncwarp();
            if (lane == 0) set_flag_release(flag_at(pair), 1);
          } else if (w.role == kOwned) {  // parts read: their flags back to 0 for the next call
            __syncwarp();
            if (lane == 0)
              for (int q = pair + 1; q < q_end; ++q) *flag_at(q) = 0;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8 * acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      T = T1;
      sb_v = sb_v1;
      sa = sa1;
      T1 = T2;
      w = w1;
      w1 = w2;
      has = has1;
      has1 = has2;
    }
    if (lane == 0) bulk_wait_group_all();  // this warp's TMA stores of y are complete
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair's MMAs have read both CTAs' shared memory; remote arrives are done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

// ============================================================== decode
// KBS 128-byte k-blocks per pipeline stage (one TMA box each per operand).
template <int BNT, int STAGES, int KBS>
struct DecodeCfg {
  static constexpr int kWBytes = kBM * kBK;   // one weight box: 128 channels x 128 K bytes
  static constexpr int kXBytes = BNT * kBK;   // one token box
  static constexpr int kStageBytes = KBS * (kWBytes + kXBytes);
  static constexpr int kTmemCols = tmem_cols_for(BNT);
  static constexpr int kPipeBytes = STAGES * kStageBytes;
  static constexpr int kYBytes = BNT * kBM * 2;    // bf16 output tile, reuses the pipeline
  static constexpr int kBarBytes = 8 * (2 * STAGES + 1) + 16;
  static constexpr int kScaleBytes = (kBM + BNT) * 4;  // s_ch of the tile, s_tok
  static constexpr int kRedBytes = BNT * kBM * 4;  // fp32 partials [rank][token][row in slice]
  static constexpr int kFixed = kPipeBytes + kBarBytes + kScaleBytes;
  // Shared memory without (single) and with (split) the reduction buffer.
  static constexpr size_t kSmemSingle = 1024 + static_cast<size_t>(kFixed);
  static constexpr size_t kSmemSplit = kSmemSingle + kRedBytes;
  static_assert(BNT % 16 == 0 && BNT >= 16 && BNT <= 256, "BNT");
  static_assert(kXBytes % 1024 == 0, "token tile must keep 1024-byte alignment");
  static_assert(kYBytes <= kPipeBytes, "output tile must fit in the pipeline buffers");
};

// y is written either by one TMA store per output tile (tmY valid, N % 8 == 0;
// its box is {rows written per CTA, BNT}) or element by element.
template <int BNT, int STAGES, int KBS, int KD = kKindE4M3>
__global__ void __launch_bounds__(192)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmY, const float* __restrict__ s_tok,
                       const float* __restrict__ s_ch, uint16_t* __restrict__ y, int M, int N,
                       int K, int splits, int kb_per_split, int use_tma_store) {
  using C = DecodeCfg<BNT, STAGES, KBS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sW = smem;                                   // STAGES x KBS weight boxes
  uint8_t* sX = smem + STAGES * KBS * C::kWBytes;       // STAGES x KBS token boxes
  uint16_t* ytile = reinterpret_cast<uint16_t*>(smem);  // after the MMAs: bf16 [token][row]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kPipeBytes);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);
  float* sch_s = reinterpret_cast<float*>(smem + C::kPipeBytes + C::kBarBytes);
  float* stok_s = sch_s + kBM;
  float* red = reinterpret_cast<float*>(smem + C::kFixed);  // split only
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + STAGES);
  const uint32_t tfull = smem_u32(bars + 2 * STAGES);
  // Abort word shared by the producer and MMA roles (mbar_wait_ab): the
  // first whose wait runs out makes the other leave at once.
  const uint32_t abort_w = smem_u32(tmem_holder + 1);

  const int warp = warp_id(), lane = lane_id();
  const int tile_n = blockIdx.x / splits;
  const int rank = blockIdx.x % splits;  // == %cluster_ctarank for cluster dims (splits,1,1)
  const int num_kb = (K + kBK - 1) / kBK;
  const int num_steps = (num_kb + KBS - 1) / KBS;       // pipeline steps over all of K
  const int st0 = rank * kb_per_split;                  // kb_per_split counts steps
  const int st1 = min(num_steps, st0 + kb_per_split);
  const bool split = splits > 1;
  const int rows = kBM / splits;                        // output rows each rank writes
  bool have_acc = st1 > st0;
  const int pre = have_acc ? min(STAGES, st1 - st0) : 0;

  if (split) cluster_arrive_relaxed();  // this CTA has started (waited on before any DSMEM store)
  // Test hook: CTA 0 skips one pipeline step's stage (no arrive, no loads).
  const int drop = blockIdx.x == 0 ? *const_cast<volatile int*>(&g_fault_drop_step) : -1;
  // The stages the producer armed and the phase parity each last arm fills.
  uint32_t armed = 0u, armed_par = 0u;
  if (warp == 0 && lane == 0) {
    st_shared_volatile_u32(abort_w, 0u);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(tfull, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    // The weight stream depends neither on the TMEM allocation nor on a
    // preceding quantizer grid: start the first ring of weight boxes now.
    const uint64_t pol_w = l2_policy_evict_first();
    for (int i = 0; i < pre; ++i) {
      if (i == drop) continue;
      const uint32_t fb = full0 + 8 * i;
      mbar_arrive_expect_tx(fb, C::kStageBytes);
      armed |= 1u << i;
#pragma unroll
      for (int j = 0; j < KBS; ++j)
        tma_load_2d(smem_u32(sW + (i * KBS + j) * C::kWBytes), &tmW, fb,
                    ((st0 + i) * KBS + j) * kBK, tile_n * kBM, pol_w);
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
  // Let the next grid on the stream launch now: in a chain of decode linears
  // its CTAs take the idle SMs and start their own weight streams while this
  // one finishes. Signalled only once this CTA holds its TMEM, so a waiting
  // dependent can never take the columns this CTA still has to allocate. The
  // dependent touches nothing this grid writes before griddepcontrol.wait.
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0 && have_acc) {
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      pdl_wait();  // activations come from a preceding quantizer grid
      for (int i = 0; i < pre; ++i) {
        if (i == drop) continue;
#pragma unroll
        for (int j = 0; j < KBS; ++j)
          tma_load_2d(smem_u32(sX + (i * KBS + j) * C::kXBytes), &tmX, full0 + 8 * i,
                      ((st0 + i) * KBS + j) * kBK, 0, pol_x);
      }
      int stage = pre % STAGES;
      uint32_t phase = pre == STAGES ? 1u : 0u;
      for (int st = st0 + pre; st < st1; ++st) {
        if (!mbar_wait_ab(empty0 + 8 * stage, phase ^ 1, abort_w)) break;
        if (st - st0 != drop) {
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, C::kStageBytes);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
#pragma unroll
          for (int j = 0; j < KBS; ++j) {
            tma_load_2d(smem_u32(sW + (stage * KBS + j) * C::kWBytes), &tmW, fb, (st * KBS + j) * kBK,
                        tile_n * kBM, pol_w);
            tma_load_2d(smem_u32(sX + (stage * KBS + j) * C::kXBytes), &tmX, fb, (st * KBS + j) * kBK,
                        0, pol_x);
          }
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      // Let every copy this thread started land (each wait bounded) before
      // the CTA can leave, also after an abort: a stage's last arm fills the
      // phase with the recorded parity, which completes once its bytes have
      // arrived (at once if the MMA already consumed it).
      for (int s2 = 0; s2 < STAGES; ++s2)
        if ((armed >> s2) & 1u) mbar_wait(full0 + 8 * s2, (armed_par >> s2) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0 && have_acc) {
      constexpr uint32_t idesc = idesc_kind<KD>(kBM, BNT);
      int stage = 0;
      uint32_t phase = 0;
      for (int st = st0; st < st1; ++st) {
        if (!mbar_wait_ab(full0 + 8 * stage, phase, abort_w)) break;
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < KBS; ++j) {
          const uint32_t a0 = smem_u32(sW + (stage * KBS + j) * C::kWBytes);
          const uint32_t b0 = smem_u32(sX + (stage * KBS + j) * C::kXBytes);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) {
            umma_kind<KD>(tmem_base, sw128_kmajor_desc(a0 + 32 * k), sw128_kmajor_desc(b0 + 32 * k),
                          idesc, (st != st0) || (j != 0) || (k != 0));
          }
        }
        umma_commit(empty0 + 8 * stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      umma_commit(tfull);
      // the issued MMAs have finished before this thread can reach the TMEM
      // release (also when the loop above was left by an abort)
      mbar_wait(tfull, 0);
    }
  } else {
    const int et = threadIdx.x - 64;                 // 0..127
    const int quad = warp & 3;
    const int ch = quad * 32 + lane;                 // channel within the tile (TMEM lane)
    // Stage both scale vectors while the main loop runs.
    {
      const int n = tile_n * kBM + et;
      sch_s[et] = n < N ? (s_ch ? __ldg(s_ch + n) : 1.0f) : 0.0f;
      pdl_wait();  // per-token scales come from a preceding quantizer grid
      if (et < BNT) stok_s[et] = et < M ? (s_tok ? s_tok[et] : 1.0f) : 0.0f;
      named_bar_sync(1, 128);
    }
    if (have_acc && !mbar_wait(tfull, 0)) have_acc = false;
    __syncwarp();
    tc_fence_after();
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    uint32_t dst = 0;
    if (split) {
      cluster_wait_acquire();  // every CTA of the cluster has started
      dst = mapa_shared(smem_u32(red) + static_cast<uint32_t>((rank * BNT * rows + ch % rows) * 4),
                        ch / rows);
    }
    const float sc = sch_s[ch];
#pragma unroll 1
    for (int c = 0; c < BNT / 16; ++c) {
      uint32_t r[16];
      tmem_ld16(t_row + c * 16, r);
      tmem_ld_wait();
      // split partials travel as raw accumulator words (int32 for kind::i8,
      // summed exactly by the owner); a single CTA converts them here
      if (!split) acc_to_f32<KD>(r);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int tok = c * 16 + j;
        const uint32_t word = have_acc ? r[j] : 0u;  // 0u is both 0.0f and int 0
        if (!split) {
          ytile[tok * kBM + ch] =
              f32_to_bf16_rn(__fmul_rn(__fmul_rn(__uint_as_float(word), stok_s[tok]), sc));
        } else if (tok < M) {
          // owner's buffer [rank][token][row in slice]: lanes write consecutive words
          st_shared_cluster_f32(dst + static_cast<uint32_t>(tok * rows * 4), __uint_as_float(word));
        }
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
    if (warp < 2) cluster_wait_acquire();  // the first barrier phase, for the non-epilogue warps
    cluster_arrive_release();              // this CTA's partials are in their owners' buffers
    cluster_wait_acquire();
    if (warp >= 2) {
      const int et = threadIdx.x - 64;
      for (int e = et; e < rows * BNT; e += 128) {
        const int tok = e / rows;
        const int rl = e % rows;
        float sum;
        if constexpr (KD == kKindS8) {  // exact int32 sum, one rounding to fp32
          int isum = __float_as_int(red[tok * rows + rl]);
          for (int j = 1; j < splits; ++j) isum += __float_as_int(red[(j * BNT + tok) * rows + rl]);
          sum = __int2float_rn(isum);
        } else {
          sum = red[tok * rows + rl];
          for (int j = 1; j < splits; ++j) sum = __fadd_rn(sum, red[(j * BNT + tok) * rows + rl]);
        }
        ytile[tok * rows + rl] =
            f32_to_bf16_rn(__fmul_rn(__fmul_rn(sum, stok_s[tok]), sch_s[rank * rows + rl]));
      }
    }
  }
  // Write the tile (or this rank's slice of it): [BNT tokens][rows_out channels].
  const int rows_out = split ? rows : kBM;
  const int n0 = tile_n * kBM + (split ? rank * rows : 0);
  if (use_tma_store) {
    if (warp >= 2) {
      fence_proxy_async_shared();  // generic writes of the tile -> visible to the TMA store
      named_bar_sync(1, 128);
      if (threadIdx.x == 64) {
        tma_store_2d(&tmY, smem_u32(ytile), n0, 0);
        bulk_commit_group();
        bulk_wait_group_all();
      }
    }
  } else if (warp >= 2) {
    named_bar_sync(1, 128);
    const int et = threadIdx.x - 64;
    for (int e = et; e < rows_out * BNT; e += 128) {
      const int tok = e / rows_out, rl = e % rows_out;
      if (tok < M && n0 + rl < N) y[static_cast<int64_t>(tok) * N + n0 + rl] = ytile[tok * rows_out + rl];
    }
  }
}

}  // namespace fp8k
