// fp8w8a8.cu - the C ABI (include/fp8w8a8.h): argument checks, TMA tensor
// maps, kernel selection and launches. Every kernel of the library lives in
// this translation unit (quant.cuh, gemm.cuh), so the device status word is
// a single __device__ variable per device.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fp8w8a8.h"
#include "gemm.cuh"
#include "moe.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "w4a16.cuh"

namespace {

constexpr int kMaxDevices = 64;

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

struct DeviceInfo {
  int sm_count = 0;
  int smem_optin = 0;     // largest dynamic shared memory a block may opt into
  int pair_clusters = 0;  // co-resident 2-CTA clusters of the pair GEMM
  bool supported = false;
  bool attrs_set = false;
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Current device's info; sets the kernels' shared-memory attributes once.
fp8_status device_info(DeviceInfo** out);

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major uint8 matrix [rows, cols] (pitch = cols bytes), 128-byte-wide
// boxes of box_rows rows, 128B swizzle, out-of-bounds elements read as 0.
bool make_tmap_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  std::memset(m, 0, sizeof(*m));
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major bf16 matrix [rows, cols] (pitch = cols elements), boxes of
// box_cols x box_rows, no swizzle; out-of-range parts of a stored box are
// not written. Requires cols % 8 == 0 (16-byte pitch).
bool make_tmap_bf16_store(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                          uint32_t box_cols, uint32_t box_rows,
                          CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  std::memset(m, 0, sizeof(*m));
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major 2-D array [rows, cols] of `dtype` elements (row pitch
// `pitch_bytes`, a multiple of 16), boxes of box_cols x box_rows, no
// swizzle, out-of-range elements read as zero.
bool make_tmap_plain(CUtensorMap* m, CUtensorMapDataType dtype, const void* base, uint64_t rows,
                     uint64_t cols, uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  std::memset(m, 0, sizeof(*m));
  return fn(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Store map of the prefill epilogues: y [rows, cols] bf16 in 32 x 32 boxes
// whose 64-byte rows use the 64-byte swizzle of the staging buffers. Sets
// g.use_tma_store when y can be stored that way (cols % 8 == 0).
void make_epilogue_store_map(CUtensorMap* m, fp8k::GemmArgs& g, const uint16_t* y, uint64_t rows,
                             uint64_t cols) {
  std::memset(m, 0, sizeof(*m));
  g.use_tma_store = (cols % 8 == 0) && (reinterpret_cast<uintptr_t>(y) & 15) == 0 &&
                    make_tmap_bf16_store(m, y, rows, cols, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

fp8_status last_launch() {
  return cudaGetLastError() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

// ----------------------------------------------------------------- GEMM plans
using namespace fp8k;

template <int BN, int STAGES, bool GROUPED, int KD = kKindE4M3>
fp8_status set_prefill_attr() {
  const size_t smem = PrefillCfg<BN, STAGES>::kSmem + (GROUPED ? grouped_smem_bytes(kMaxExperts) : 0);
  return cudaFuncSetAttribute(gemm_prefill_kernel<BN, STAGES, GROUPED, KD>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(smem)) == cudaSuccess
             ? FP8_OK
             : FP8_ERR_CUDA;
}

// Deep-ring variants whose split-K layout would not fit are set up (and
// launched) without a K split only.
template <int BNT, int STAGES, int KBS, int KD = kKindE4M3>
fp8_status set_decode_attr(int smem_optin) {
  using C = DecodeCfg<BNT, STAGES, KBS>;
  const size_t smem = C::kSmemSplit <= static_cast<size_t>(smem_optin) ? C::kSmemSplit : C::kSmemSingle;
  return cudaFuncSetAttribute(gemm_decode_kernel<BNT, STAGES, KBS, KD>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) ==
                 cudaSuccess
             ? FP8_OK
             : FP8_ERR_CUDA;
}

// Shared memory of a grouped pair launch with E experts.
template <int STAGES>
size_t grouped_pair_smem(int E) {
  return PairCfg<STAGES, pair_stg_bufs<true>()>::kSmem + grouped_smem_bytes(E);
}

template <int STAGES, int GSTAGES>
fp8_status set_pair_attr() {
  return cudaFuncSetAttribute(gemm_pair_kernel<STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(PairCfg<STAGES>::kSmem)) == cudaSuccess &&
                 cudaFuncSetAttribute(gemm_pair_kernel<STAGES, false, false, kKindE4M3, true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(PairCfg<STAGES>::kSmem)) == cudaSuccess &&
                 cudaFuncSetAttribute(gemm_pair_kernel<STAGES, false, false, kKindS8, true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(PairCfg<STAGES>::kSmem)) == cudaSuccess &&
                 cudaFuncSetAttribute(gemm_pair_kernel<STAGES, false, false, kKindS8>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(PairCfg<STAGES>::kSmem)) == cudaSuccess &&
                 cudaFuncSetAttribute(gemm_pair_kernel<STAGES, false, false, kKindBF16>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(PairCfg<STAGES>::kSmem)) == cudaSuccess &&
                 cudaFuncSetAttribute(gemm_pair_kernel<GSTAGES, true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(grouped_pair_smem<GSTAGES>(kMaxExperts))) ==
                     cudaSuccess &&
                 cudaFuncSetAttribute(gemm_pair_kernel<GSTAGES, true, true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(grouped_pair_smem<GSTAGES>(kMaxExperts))) ==
                     cudaSuccess
             ? FP8_OK
             : FP8_ERR_CUDA;
}

// Every decode variant launch_linear can pick, for one operand kind.
template <int KD>
fp8_status set_decode_attrs(int so) {
  fp8_status st = FP8_OK;
  st = st != FP8_OK ? st : set_decode_attr<16, 2, 2, KD>(so);
  st = st != FP8_OK ? st : set_decode_attr<16, 3, 2, KD>(so);
  st = st != FP8_OK ? st : set_decode_attr<16, 6, 2, KD>(so);
  st = st != FP8_OK ? st : set_decode_attr<32, 4, 1, KD>(so);
  st = st != FP8_OK ? st : set_decode_attr<32, 3, 2, KD>(so);
  st = st != FP8_OK ? st : set_decode_attr<64, 4, 1, KD>(so);
  st = st != FP8_OK ? st : set_decode_attr<64, 4, 2, KD>(so);
  st = st != FP8_OK ? st : set_decode_attr<128, 3, 1, KD>(so);
  st = st != FP8_OK ? st : set_decode_attr<128, 4, 1, KD>(so);
  st = st != FP8_OK ? st : set_decode_attr<128, 3, 2, KD>(so);
  return st;
}

template <int BNT, int RS, int AS>
fp8_status set_w4_attr(int smem_optin) {
  using C = W4DecodeCfg<BNT, RS, AS>;
  const size_t smem = C::kSmemSplit <= static_cast<size_t>(smem_optin) ? C::kSmemSplit : C::kSmemSingle;
  return cudaFuncSetAttribute(gemm_w4_decode_kernel<BNT, RS, AS>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) ==
                 cudaSuccess
             ? FP8_OK
             : FP8_ERR_CUDA;
}

constexpr int kPairStages = 6;
// Grouped pair launches: five stages, which leaves room for the epilogue's
// second staging buffer per warp.
constexpr int kGroupedPairStages = 5;
constexpr int kPrefillBN = 256;
// Shared memory the staged quantizer may use per block (one block per SM).
constexpr int kStagedSmemBudget = 200 * 1024;
constexpr int kPrefillStages = 4;

fp8_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.attrs_set) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return FP8_ERR_CUDA;
    d.sm_count = prop.multiProcessorCount;
    d.smem_optin = static_cast<int>(prop.sharedMemPerBlockOptin);
    d.supported = prop.major == 10 && prop.minor == 0;
    if (!d.supported) return FP8_ERR_UNSUPPORTED;
    fp8_status st = FP8_OK;
    st = st != FP8_OK ? st : set_prefill_attr<kPrefillBN, kPrefillStages, false>();
    st = st != FP8_OK ? st : set_prefill_attr<kPrefillBN, kPrefillStages, false, kKindS8>();
    st = st != FP8_OK ? st : set_prefill_attr<kPrefillBN, kPrefillStages, false, kKindBF16>();
    st = st != FP8_OK ? st : set_prefill_attr<256, kPrefillStages, true>();
    st = st != FP8_OK ? st : set_pair_attr<kPairStages, kGroupedPairStages>();
    if (st == FP8_OK) {
      // A persistent grid must fit at once: count the 2-CTA clusters that can
      // be resident together (an SM left over in a GPC cannot host a pair).
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (d.sm_count / 2));
      cfg.blockDim = dim3(kPrefillThreads);
      cfg.dynamicSmemBytes = PairCfg<kPairStages>::kSmem;
      cudaLaunchAttribute a;
      a.id = cudaLaunchAttributeClusterDimension;
      a.val.clusterDim.x = 2;
      a.val.clusterDim.y = 1;
      a.val.clusterDim.z = 1;
      cfg.attrs = &a;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<kPairStages>, &cfg) != cudaSuccess)
        st = FP8_ERR_CUDA;
      d.pair_clusters = n;
    }
    const int so = d.smem_optin;
    st = st != FP8_OK ? st : set_decode_attrs<kKindE4M3>(so);
    st = st != FP8_OK ? st : set_decode_attrs<kKindS8>(so);
    st = st != FP8_OK ? st : set_decode_attrs<kKindBF16>(so);
    st = st != FP8_OK ? st : set_w4_attr<16, 6, 4>(so);
    st = st != FP8_OK ? st : set_w4_attr<16, 3, 2>(so);
    st = st != FP8_OK ? st : set_w4_attr<32, 6, 3>(so);
    st = st != FP8_OK ? st : set_w4_attr<32, 3, 2>(so);
    st = st != FP8_OK ? st : set_w4_attr<64, 4, 3>(so);
    st = st != FP8_OK ? st : set_w4_attr<64, 2, 2>(so);
    st = st != FP8_OK ? st : set_w4_attr<128, 4, 2>(so);
    if (st == FP8_OK &&
        (cudaFuncSetAttribute(quant_act_staged_kernel<false>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kStagedSmemBudget + 1024) != cudaSuccess ||
         cudaFuncSetAttribute(quant_act_staged_kernel<true>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kStagedSmemBudget + 1024) != cudaSuccess ||
         cudaFuncSetAttribute(quant_act_staged_kernel<false, kEncI8>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kStagedSmemBudget + 1024) != cudaSuccess ||
         cudaFuncSetAttribute(quant_act_staged_kernel<true, kEncI8>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kStagedSmemBudget + 1024) != cudaSuccess ||
         cudaFuncSetAttribute(quant_act_staged_kernel<true, kEncE4M3, 2>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kStagedSmemBudget + 1024) != cudaSuccess ||
         cudaFuncSetAttribute(quant_act_staged_kernel<true, kEncI8, 2>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kStagedSmemBudget + 1024) != cudaSuccess))
      st = FP8_ERR_CUDA;
    if (st == FP8_OK &&
        cudaFuncSetAttribute(convert_fnuz_staged_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kStagedSmemBudget + 1024) != cudaSuccess)
      st = FP8_ERR_CUDA;
    if (st == FP8_OK &&
        (cudaFuncSetAttribute(repack_qat_staged_kernel<kEncE4M3>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, 110 * 1024) != cudaSuccess ||
         cudaFuncSetAttribute(repack_qat_staged_kernel<kEncI8>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, 110 * 1024) != cudaSuccess))
      st = FP8_ERR_CUDA;
    if (st != FP8_OK) return st;
    d.attrs_set = true;
  }
  if (!d.supported) return FP8_ERR_UNSUPPORTED;
  *out = &d;
  return FP8_OK;
}

void set_pdl(cudaLaunchAttribute* a, int& n, bool pdl) {
  if (!pdl) return;
  a[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
}

// Operands are row-major [rows, K] arrays of 1-byte (E4M3, int8) or 2-byte
// (bf16) elements; K here counts BYTES per row. A null scale means 1.
template <int KD = kKindE4M3>
fp8_status launch_prefill(const DeviceInfo& dev, const uint8_t* x8, const float* s_tok,
                          const uint8_t* w8, const float* s_ch, int M, int N, int K, uint16_t* y,
                          cudaStream_t stream, bool pdl) {
  constexpr int BN = kPrefillBN, ST = kPrefillStages;
  CUtensorMap tmA, tmB;
  if (!make_tmap_u8(&tmA, x8, M, K, kBM) || !make_tmap_u8(&tmB, w8, N, K, BN)) return FP8_ERR_CUDA;
  const int tiles_m = (M + kBM - 1) / kBM;
  const int tiles_n = (N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int group_m = std::min(tiles_m, 16);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(std::min(num_tiles, dev.sm_count));
  cfg.blockDim = dim3(kPrefillThreads);
  cfg.dynamicSmemBytes = PrefillCfg<BN, ST>::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[1];
  int na = 0;
  set_pdl(attrs, na, pdl);
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  GemmArgs g = {};
  g.s_a = s_tok;
  g.s_b = s_ch;
  g.y = y;
  g.M = M;
  g.N = N;
  g.K = K;
  g.tiles_m = tiles_m;
  g.tiles_n = tiles_n;
  g.group_m = group_m;
  CUtensorMap tmY;
  make_epilogue_store_map(&tmY, g, y, M, N);
  if (cudaLaunchKernelEx(&cfg, gemm_prefill_kernel<BN, ST, false, KD>, tmA, tmB, tmY, g) != cudaSuccess)
    return FP8_ERR_CUDA;
  return FP8_OK;
}

// Dense GEMM on 256 x 256 tiles per CTA pair (clusters of 2, persistent).
template <int KD = kKindE4M3>
fp8_status launch_pair(const DeviceInfo& dev, const uint8_t* x8, const float* s_tok,
                       const uint8_t* w8, const float* s_ch, int M, int N, int K, uint16_t* y,
                       cudaStream_t stream, bool pdl, void* ws = nullptr, size_t ws_bytes = 0) {
  CUtensorMap tmA, tmB;
  if (!make_tmap_u8(&tmA, x8, M, K, 128) || !make_tmap_u8(&tmB, w8, N, K, 128)) return FP8_ERR_CUDA;
  const int tiles_m = (M + 255) / 256;
  const int tiles_n = (N + 255) / 256;
  const int num_tiles = tiles_m * tiles_n;
  const int pairs = std::min(num_tiles, dev.pair_clusters);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kPrefillThreads);
  cfg.dynamicSmemBytes = PairCfg<kPairStages>::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  attrs[na].id = cudaLaunchAttributeClusterDimension;
  attrs[na].val.clusterDim.x = 2;
  attrs[na].val.clusterDim.y = 1;
  attrs[na].val.clusterDim.z = 1;
  ++na;
  set_pdl(attrs, na, pdl);
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  GemmArgs g = {};
  g.s_a = s_tok;
  g.s_b = s_ch;
  g.y = y;
  g.M = M;
  g.N = N;
  g.K = K;
  g.tiles_m = tiles_m;
  g.tiles_n = tiles_n;
  // Rasters of 16 row-tile pairs: each group re-reads the weights once, and
  // 16 pairs' activation rows (e.g. 4096 x 5376 bytes) still sit in L2
  // (measured on B200 at M = 65536, K = 5376, N = 21504: 8 -> 16 pairs,
  // 6.4 -> 5.7 ms per GEMM under the power cap; 32 pairs: 5.8 ms).
  g.group_m = std::min(tiles_m, 16);
  CUtensorMap tmY;
  make_epilogue_store_map(&tmY, g, y, M, N);
  // A partial last wave of tiles (fewer than 8 waves, so that it costs a
  // noticeable share) is evened out by the k-block split when the caller
  // gave a workspace: the last full wave and the partial one are shared
  // out by k-blocks over all pairs.
  if constexpr (KD == kKindE4M3 || KD == kKindS8) {
    if (ws && ws_bytes >= split_ws_bytes(pairs) && num_tiles > pairs && num_tiles % pairs != 0 &&
        num_tiles < 8 * pairs) {
      g.sk_tiles = pairs + num_tiles % pairs;
      g.ws_flag = static_cast<int*>(ws);
      g.ws_part = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + split_flag_bytes(pairs));
      if (cudaLaunchKernelEx(&cfg, gemm_pair_kernel<kPairStages, false, false, KD, true>, tmA, tmB, tmB,
                             tmY, g) != cudaSuccess)
        return FP8_ERR_CUDA;
      return FP8_OK;
    }
  }
  if (cudaLaunchKernelEx(&cfg, gemm_pair_kernel<kPairStages, false, false, KD>, tmA, tmB, tmB, tmY,
                         g) != cudaSuccess)
    return FP8_ERR_CUDA;
  return FP8_OK;
}

// Per-expert GEMM: persistent grid, tiles decoded on the GPU from offsets.
template <int BN, int ST>
fp8_status launch_grouped(const DeviceInfo& dev, const uint8_t* x8, const float* s_rows,
                          const int32_t* offsets, int E, int M_total, const uint8_t* w8,
                          const float* s_ch, int N, int K, uint16_t* y, cudaStream_t stream) {
  CUtensorMap tmA, tmB;
  if (!make_tmap_u8(&tmA, x8, M_total, K, kBM) ||
      !make_tmap_u8(&tmB, w8, static_cast<uint64_t>(E) * N, K, BN))
    return FP8_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(dev.sm_count);
  cfg.blockDim = dim3(kPrefillThreads);
  cfg.dynamicSmemBytes = PrefillCfg<BN, ST>::kSmem + grouped_smem_bytes(E);
  cfg.stream = stream;
  cudaLaunchAttribute attrs[1];
  int na = 0;
  set_pdl(attrs, na, true);
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  GemmArgs g = {};
  g.s_a = s_rows;
  g.s_b = s_ch;
  g.y = y;
  g.M = M_total;
  g.N = N;
  g.K = K;
  g.tiles_n = (N + BN - 1) / BN;
  g.offsets = offsets;
  g.num_experts = E;
  CUtensorMap tmY;
  make_epilogue_store_map(&tmY, g, y, M_total, N);
  if (cudaLaunchKernelEx(&cfg, gemm_prefill_kernel<BN, ST, true>, tmA, tmB, tmY, g) != cudaSuccess)
    return FP8_ERR_CUDA;
  return FP8_OK;
}

// Per-expert GEMM on CTA pairs (256-row pair tiles per expert): persistent
// grid of the co-resident pairs, tiles decoded on the GPU from offsets.
// With n_out > 0 the GeGLU epilogue writes h [M_total, n_out] (w8 / s_ch in
// the interleaved gate/up layout, N = 256 * ceil(n_out / 128) rows per expert).
fp8_status launch_grouped_pair(const DeviceInfo& dev, const uint8_t* x8, const float* s_rows,
                               const int32_t* offsets, int E, int M_total, const uint8_t* w8,
                               const float* s_ch, int N, int K, uint16_t* y, cudaStream_t stream,
                               int n_out = 0) {
  CUtensorMap tmA, tmB;
  if (!make_tmap_u8(&tmA, x8, M_total, K, 128) ||
      !make_tmap_u8(&tmB, w8, static_cast<uint64_t>(E) * N, K, 128))
    return FP8_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * dev.pair_clusters);
  cfg.blockDim = dim3(kPrefillThreads);
  cfg.dynamicSmemBytes = grouped_pair_smem<kGroupedPairStages>(E);
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  attrs[na].id = cudaLaunchAttributeClusterDimension;
  attrs[na].val.clusterDim.x = 2;
  attrs[na].val.clusterDim.y = 1;
  attrs[na].val.clusterDim.z = 1;
  ++na;
  set_pdl(attrs, na, true);
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  GemmArgs g = {};
  g.s_a = s_rows;
  g.s_b = s_ch;
  g.y = y;
  g.M = M_total;
  g.N = N;
  g.K = K;
  g.tiles_n = (N + 255) / 256;
  g.offsets = offsets;
  g.num_experts = E;
  g.n_out = n_out;
  CUtensorMap tmY;
  make_epilogue_store_map(&tmY, g, y, M_total, n_out > 0 ? n_out : N);
  // GeGLU: half-width last feature tiles load 64 B rows per CTA through tmBh
  CUtensorMap tmBh = tmB;
  if (n_out > 0 && !make_tmap_u8(&tmBh, w8, static_cast<uint64_t>(E) * N, K, 64)) return FP8_ERR_CUDA;
  const auto kernel = n_out > 0 ? gemm_pair_kernel<kGroupedPairStages, true, true>
                                : gemm_pair_kernel<kGroupedPairStages, true, false>;
  if (cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, tmBh, tmY, g) != cudaSuccess) return FP8_ERR_CUDA;
  return FP8_OK;
}

// Launch of a plain kernel as a programmatic dependent of the previous work
// in the stream (its prologue may overlap that work; the kernel itself calls
// griddepcontrol.wait before reading what the previous grid wrote).
template <typename... KArgs, typename... Args>
fp8_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, cudaStream_t stream,
                      Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[1];
  int na = 0;
  set_pdl(attrs, na, true);
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

// As launch_pdl, with dynamic shared memory.
template <typename... KArgs, typename... Args>
fp8_status launch_pdl_smem(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                           cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[1];
  int na = 0;
  set_pdl(attrs, na, true);
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

// Number of K splits the decode GEMM uses for N output channels.
int decode_splits(const DeviceInfo& dev, int N, int K, int kbs) {
  const int tiles = (N + kBM - 1) / kBM;
  const int num_steps = (K + kBK * kbs - 1) / (kBK * kbs);
  // K is split over a cluster only when there are too few 128-channel tiles to
  // keep the SMs streaming (measured on B200: with >= SMs/4 tiles the cluster
  // reduction costs more than the extra streams bring). Splits divide 128 and
  // keep at least two pipeline steps each.
  int splits = 1;
  if (4 * tiles < dev.sm_count)
    while (splits < 8 && tiles * splits * 2 <= dev.sm_count && splits * 4 <= num_steps) splits *= 2;
  return splits;
}

template <int BNT, int ST, int KBS, int KD = kKindE4M3>
fp8_status launch_decode_t(const DeviceInfo& dev, const uint8_t* x8, const float* s_tok,
                           const uint8_t* w8, const float* s_ch, int M, int N, int K, uint16_t* y,
                           cudaStream_t stream, bool pdl, int force_splits = 0) {
  using C = DecodeCfg<BNT, ST, KBS>;
  CUtensorMap tmW, tmX;
  if (!make_tmap_u8(&tmW, w8, N, K, kBM) || !make_tmap_u8(&tmX, x8, M, K, BNT))
    return FP8_ERR_CUDA;
  const int tiles = (N + kBM - 1) / kBM;
  const int num_steps = (K + kBK * KBS - 1) / (kBK * KBS);
  int splits = decode_splits(dev, N, K, KBS);
  if (force_splits > 0) splits = force_splits;
  if (splits > 1 && C::kSmemSplit > static_cast<size_t>(dev.smem_optin)) return FP8_ERR_UNSUPPORTED;
  const int steps_per_split = (num_steps + splits - 1) / splits;
  CUtensorMap tmY;
  std::memset(&tmY, 0, sizeof(tmY));
  const int use_tma_store =
      (N % 8 == 0) && make_tmap_bf16_store(&tmY, y, M, N, kBM / splits, BNT) ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles * splits);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = splits > 1 ? C::kSmemSplit : C::kSmemSingle;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  attrs[na].id = cudaLaunchAttributeClusterDimension;
  attrs[na].val.clusterDim.x = splits;
  attrs[na].val.clusterDim.y = 1;
  attrs[na].val.clusterDim.z = 1;
  ++na;
  set_pdl(attrs, na, pdl);
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  if (cudaLaunchKernelEx(&cfg, gemm_decode_kernel<BNT, ST, KBS, KD>, tmW, tmX, tmY, s_tok, s_ch, y, M,
                         N, K, splits, steps_per_split, use_tma_store) != cudaSuccess)
    return FP8_ERR_CUDA;
  return FP8_OK;
}

// y = (a . b^T) * s_a * s_b for one operand kind; K counts bytes per row.
template <int KD = kKindE4M3>
fp8_status launch_linear(const DeviceInfo& dev, const uint8_t* x8, const float* s_tok,
                         const uint8_t* w8, const float* s_ch, int M, int N, int K, uint16_t* y,
                         cudaStream_t stream, bool pdl, void* ws = nullptr, size_t ws_bytes = 0) {
  // Decode-sized M: swap-AB kernel. Pipeline depth is chosen so that every
  // CTA is resident at once: with more 128-channel tiles than SMs, two CTAs
  // share an SM (<= ~110 KB of stages each), otherwise one CTA gets ~200 KB.
  // The deepest rings (most of a CTA's weights requested before it waits for
  // the preceding grid) are used when there is no K split.
  const int tiles = (N + kBM - 1) / kBM;
  const bool one_per_sm = tiles <= dev.sm_count;
  const bool no_split = 4 * tiles >= dev.sm_count;  // decode_splits() gives 1
  if (M <= 16) {
    // Up to 16 tokens: many short weight streams beat few long ones (measured
    // on B200 in chains of linears, e.g. 2048 x 4096: 6.3 vs 10.0 us). Split K
    // over a cluster while at most two CTAs per SM result and each CTA keeps
    // at least 4 k-blocks, and take that split when it reaches 4.
    const int num_kb = (K + kBK - 1) / kBK;
    int s = 1;
    while (s < 8 && tiles * s * 2 <= 2 * dev.sm_count && s * 2 * 4 <= num_kb) s *= 2;
    if (s >= 4) return launch_decode_t<16, 2, 2, KD>(dev, x8, s_tok, w8, s_ch, M, N, K, y, stream, pdl, s);
    return one_per_sm && no_split
               ? launch_decode_t<16, 6, 2, KD>(dev, x8, s_tok, w8, s_ch, M, N, K, y, stream, pdl)
               : launch_decode_t<16, 3, 2, KD>(dev, x8, s_tok, w8, s_ch, M, N, K, y, stream, pdl);
  }
  if (M <= 32)
    return one_per_sm ? launch_decode_t<32, 3, 2, KD>(dev, x8, s_tok, w8, s_ch, M, N, K, y, stream, pdl)
                      : launch_decode_t<32, 4, 1, KD>(dev, x8, s_tok, w8, s_ch, M, N, K, y, stream, pdl);
  if (M <= 64)
    return one_per_sm ? launch_decode_t<64, 4, 2, KD>(dev, x8, s_tok, w8, s_ch, M, N, K, y, stream, pdl)
                      : launch_decode_t<64, 4, 1, KD>(dev, x8, s_tok, w8, s_ch, M, N, K, y, stream, pdl);
  if (M <= 128) {
    // One CTA per SM with no split: two 128-byte k-blocks per stage, so each
    // weight row is read 256 contiguous bytes at a time (measured on B200 at
    // 14336 x 4096, M = 128: 19.8 -> 19.3 us per linear against one k-block
    // per stage in a ring of the same size).
    if (!one_per_sm)
      return launch_decode_t<128, 3, 1, KD>(dev, x8, s_tok, w8, s_ch, M, N, K, y, stream, pdl);
    return no_split ? launch_decode_t<128, 3, 2, KD>(dev, x8, s_tok, w8, s_ch, M, N, K, y, stream, pdl)
                    : launch_decode_t<128, 4, 1, KD>(dev, x8, s_tok, w8, s_ch, M, N, K, y, stream, pdl);
  }
  // Prefill: 256 x 256 tiles on CTA pairs or 128 x 256 tiles on single SMs
  // (the same work per SM per tile). Pairs move a third less operand traffic
  // per tile, so they win whenever they need no more waves of tiles than the
  // single-SM grid - on equal waves only when K is long enough to amortize
  // their heavier start (measured on B200 for M = 160..512: 14336 x 4096 and
  // 21504 x 5376 favour pairs except where pairs need 3 waves against 2;
  // 8192 x 2048 favours single SMs).
  if (dev.pair_clusters > 0) {
    const int64_t tiles_n = (N + 255) / 256;
    const int64_t pair_waves = ((M + 255) / 256 * tiles_n + dev.pair_clusters - 1) / dev.pair_clusters;
    const int64_t sm_waves = ((M + kBM - 1) / kBM * tiles_n + dev.sm_count - 1) / dev.sm_count;
    if (pair_waves < sm_waves || (pair_waves == sm_waves && K >= 4096))
      return launch_pair<KD>(dev, x8, s_tok, w8, s_ch, M, N, K, y, stream, pdl, ws, ws_bytes);
  }
  return launch_prefill<KD>(dev, x8, s_tok, w8, s_ch, M, N, K, y, stream, pdl);
}

// W4A16 decode, weights unpacked on chip (M <= 128, K % 128 == 0). K is split
// over a cluster (powers of two up to 8) while the CTAs still fit one per SM
// and each keeps four or more 128-value steps; the deep-ring variant (one CTA
// per SM) when the grid fits the SMs, else a shallow one (two per SM). Up to
// 128 tokens: one CTA per SM and no split (the token tiles take the room).
template <int BNT, int RS, int AS>
fp8_status launch_w4_decode_t(const DeviceInfo& dev, const uint16_t* x, const uint8_t* q4,
                              const float* d, int M, int N, int K, uint16_t* y, int splits,
                              cudaStream_t stream, bool pdl) {
  using C = W4DecodeCfg<BNT, RS, AS>;
  CUtensorMap tmQ, tmD, tmX;
  if (!make_tmap_plain(&tmQ, CU_TENSOR_MAP_DATA_TYPE_UINT8, q4, N, K / 2, K / 2, 64, kBM) ||
      !make_tmap_plain(&tmD, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, d, N, K / 32, static_cast<uint64_t>(K / 32) * 4,
                       4, kBM) ||
      !make_tmap_u8(&tmX, x, M, static_cast<uint64_t>(2) * K, BNT))
    return FP8_ERR_CUDA;
  if (splits > 1 && C::kSmemSplit > static_cast<size_t>(dev.smem_optin)) return FP8_ERR_UNSUPPORTED;
  const int tiles = (N + kBM - 1) / kBM;
  const int num_st = (K + 127) / 128;
  const int st_per_split = (num_st + splits - 1) / splits;
  CUtensorMap tmY;
  std::memset(&tmY, 0, sizeof(tmY));
  const int use_tma_store =
      (N % 8 == 0) && make_tmap_bf16_store(&tmY, y, M, N, kBM / splits, BNT) ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles * splits);
  cfg.blockDim = dim3(w4_threads(RS));
  cfg.dynamicSmemBytes = splits > 1 ? C::kSmemSplit : C::kSmemSingle;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  attrs[na].id = cudaLaunchAttributeClusterDimension;
  attrs[na].val.clusterDim.x = splits;
  attrs[na].val.clusterDim.y = 1;
  attrs[na].val.clusterDim.z = 1;
  ++na;
  set_pdl(attrs, na, pdl);
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, gemm_w4_decode_kernel<BNT, RS, AS>, tmQ, tmD, tmX, tmY, y, M, N, K,
                            splits, st_per_split, use_tma_store) == cudaSuccess
             ? FP8_OK
             : FP8_ERR_CUDA;
}

fp8_status launch_w4_decode(const DeviceInfo& dev, const uint16_t* x, const uint8_t* q4,
                            const float* d, int M, int N, int K, uint16_t* y, cudaStream_t stream) {
  const int tiles = (N + kBM - 1) / kBM;
  const int num_st = (K + 127) / 128;
  int splits = 1;
  while (splits < 8 && tiles * splits * 2 <= dev.sm_count && splits * 4 <= num_st) splits *= 2;
  const bool deep = tiles * splits <= dev.sm_count;
  if (M <= 16)
    return deep ? launch_w4_decode_t<16, 6, 4>(dev, x, q4, d, M, N, K, y, splits, stream, true)
                : launch_w4_decode_t<16, 3, 2>(dev, x, q4, d, M, N, K, y, splits, stream, true);
  if (M <= 32)
    return deep ? launch_w4_decode_t<32, 6, 3>(dev, x, q4, d, M, N, K, y, splits, stream, true)
                : launch_w4_decode_t<32, 3, 2>(dev, x, q4, d, M, N, K, y, splits, stream, true);
  if (M <= 64)
    return deep ? launch_w4_decode_t<64, 4, 3>(dev, x, q4, d, M, N, K, y, splits, stream, true)
                : launch_w4_decode_t<64, 2, 2>(dev, x, q4, d, M, N, K, y, splits, stream, true);
  return launch_w4_decode_t<128, 4, 2>(dev, x, q4, d, M, N, K, y, 1, stream, true);
}

// Blocks of a row-staged streaming kernel that fit on one SM at once (its
// registers and `smem` bytes of row buffers), so that the grid is resident
// at once; at least 1.
template <typename Kernel>
int64_t staged_blocks_per_sm(Kernel kernel, int threads, size_t smem) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess)
    n = 1;
  return std::max(1, n);
}

// ----------------------------------------------------------------- quant plans
// Every quantizer kernel waits for the preceding grid before it reads x and
// writes nothing before that, so it is always launched as a programmatic
// dependent: in a chain of linears it starts while the previous GEMM ends.
template <int ENC = kEncE4M3>
fp8_status launch_quant_act(const DeviceInfo& dev, const uint16_t* x, int64_t M, int64_t K,
                            int64_t ldx, uint8_t* x8, float* s_tok, cudaStream_t stream) {
  const int64_t nvec = K / 8;
  const uint32_t row_pad = static_cast<uint32_t>((2 * K + 127) / 128 * 128);
  const int64_t staged_warps = std::min<int64_t>(8, kStagedSmemBudget / (2 * int64_t(row_pad) + 16));
  if (M > 1024 && staged_warps >= 2) {
    // Large M: warp-per-row pipeline through shared memory; as many blocks per
    // SM as registers and row buffers allow (the occupancy query), so that
    // short rows still keep enough rows in flight.
    const int warps = static_cast<int>(staged_warps);
    const size_t smem = static_cast<size_t>(warps) * 2 * row_pad + 16 * warps;
    const int64_t per_sm = staged_blocks_per_sm(quant_act_staged_kernel<false, ENC>, 32 * warps, smem);
    // Long rows that leave fewer than 16 warps per SM: a warp pair per row,
    // each warp staging half of it, where that gives 24 or more warps per SM
    // (measured on B200: 8192 x 4096 20.4 -> 17.7 us with 24 warps per SM;
    // 65536 x 5376, where pairs give 16, 169 -> 177 us, so not there).
    const uint32_t half_pad = static_cast<uint32_t>((K + 127) / 128 * 128);
    const int64_t pair_warps = std::min<int64_t>(8, kStagedSmemBudget / (2 * int64_t(half_pad) + 24)) & ~int64_t(1);
    const int pw = static_cast<int>(pair_warps);
    const size_t psmem = static_cast<size_t>(pw) * 2 * half_pad + 24 * pw;
    const int64_t pper_sm =
        pw >= 2 ? staged_blocks_per_sm(quant_act_staged_kernel<true, ENC, 2>, 32 * pw, psmem) : 0;
    if (per_sm * warps < 16 && pper_sm * pw >= 24) {  // many warps per SM: packed divisions
      const int64_t pblocks = std::min<int64_t>(pper_sm * dev.sm_count, (M + pw / 2 - 1) / (pw / 2));
      return launch_pdl_smem(quant_act_staged_kernel<true, ENC, 2>, dim3(static_cast<unsigned>(pblocks)),
                             dim3(32 * pw), psmem, stream, x, M, K, ldx, x8, s_tok, half_pad);
    }
    const int64_t blocks = std::min<int64_t>(per_sm * dev.sm_count, (M + warps - 1) / warps);
    // Short rows (16 or more warps per SM) are issue-bound: packed divisions.
    const auto kernel = per_sm * warps >= 16 ? quant_act_staged_kernel<true, ENC>
                                             : quant_act_staged_kernel<false, ENC>;
    return launch_pdl_smem(kernel, dim3(static_cast<unsigned>(blocks)), dim3(32 * warps), smem,
                           stream, x, M, K, ldx, x8, s_tok, row_pad);
  }
  if (M <= 1024) {
    // Few tokens: a whole block per token row, sized so that the row sits in
    // registers (one memory round trip for the amax, none for the quantize).
    const dim3 grid(static_cast<unsigned>(M));
    if (nvec <= 4 * 256)
      return launch_pdl(quant_act_kernel<256, 4, 256, ENC>, grid, dim3(256), stream, x, M, K, ldx, x8, s_tok);
    return launch_pdl(quant_act_kernel<1024, 8, 1024, ENC>, grid, dim3(1024), stream, x, M, K, ldx, x8,
                      s_tok);
  }
  const dim3 grid(static_cast<unsigned>((M + 7) / 8));
  if (nvec <= 24 * 32)
    return launch_pdl(quant_act_kernel<32, 24, 256, ENC>, grid, dim3(256), stream, x, M, K, ldx, x8, s_tok);
  return launch_pdl(quant_act_kernel<32, 0, 256, ENC>, grid, dim3(256), stream, x, M, K, ldx, x8, s_tok);
}

bool dims_ok(int64_t v, int64_t lim) { return v >= 0 && v <= lim; }

constexpr int64_t kMaxRows = (int64_t(1) << 31) - 1;

// QAT q4_0 -> per-channel codes of one encoder (E4M3 or int8): checks, then
// rows staged through shared memory (two blocks of 8 warps per SM) when K %
// 128 == 0 and there are enough rows, else the register-cached kernel.
template <int ENC>
fp8_status repack_qat_checked(const uint8_t* q4, const float* d, int64_t N, int64_t K, uint8_t* w8,
                              float* s_ch, cudaStream_t stream) {
  if (!dims_ok(N, kMaxRows) || !dims_ok(K, int64_t(1) << 24)) return FP8_ERR_INVALID_ARG;
  if (K % 32 != 0) return FP8_ERR_SHAPE;
  if (N == 0) return FP8_OK;
  if (!q4 || !d || !w8 || !s_ch) return FP8_ERR_INVALID_ARG;
  if (!aligned16(q4) || !aligned16(w8) || !aligned4(d) || !aligned4(s_ch)) return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  const uint32_t rbuf = static_cast<uint32_t>((K / 2 + K / 8 + 127) / 128 * 128);
  const size_t rsmem = size_t(8) * kRepackBufs * rbuf + 8 * 8 * kRepackBufs;
  if (K % 128 == 0 && N >= 4 * dev->sm_count && rsmem <= 110 * 1024) {
    const int64_t blocks = std::min<int64_t>(2 * dev->sm_count, (N + 7) / 8);
    repack_qat_staged_kernel<ENC><<<static_cast<unsigned>(blocks), 256, rsmem, stream>>>(
        q4, d, N, K, w8, s_ch, rbuf);
    return last_launch();
  }
  const dim3 grid(static_cast<unsigned>((N + 7) / 8));
  if (K / 32 <= 6 * 32)
    repack_qat_kernel<32, 6, ENC><<<grid, 256, 0, stream>>>(q4, d, N, K, w8, s_ch);
  else
    repack_qat_kernel<32, 0, ENC><<<grid, 256, 0, stream>>>(q4, d, N, K, w8, s_ch);
  return last_launch();
}

}  // namespace

// =================================================================== C ABI
extern "C" {

int fp8_version(void) { return 100; }

const char* fp8_status_string(fp8_status s) {
  switch (s) {
    case FP8_OK: return "FP8_OK";
    case FP8_ERR_INVALID_ARG: return "FP8_ERR_INVALID_ARG";
    case FP8_ERR_ALIGNMENT: return "FP8_ERR_ALIGNMENT";
    case FP8_ERR_SHAPE: return "FP8_ERR_SHAPE";
    case FP8_ERR_CUDA: return "FP8_ERR_CUDA";
    case FP8_ERR_UNSUPPORTED: return "FP8_ERR_UNSUPPORTED";
    case FP8_ERR_SCRATCH_LIMIT: return "FP8_ERR_SCRATCH_LIMIT";
  }
  return "FP8_ERR_UNKNOWN";
}

int fp8_device_supported(int device) {
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return 0;
  return prop.major == 10 && prop.minor == 0;
}

fp8_status fp8_test_set_fault(int64_t wait_cycles, int32_t drop_step) {
  if (wait_cycles < 0 || drop_step < -1) return FP8_ERR_INVALID_ARG;
  const long long lim = wait_cycles == 0 ? fp8k::kWaitCycles : static_cast<long long>(wait_cycles);
  const int drop = drop_step;
  if (cudaDeviceSynchronize() != cudaSuccess) return FP8_ERR_CUDA;
  if (cudaMemcpyToSymbol(fp8k::g_wait_limit, &lim, sizeof(lim)) != cudaSuccess ||
      cudaMemcpyToSymbol(fp8k::g_fault_drop_step, &drop, sizeof(drop)) != cudaSuccess)
    return FP8_ERR_CUDA;
  return cudaDeviceSynchronize() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

fp8_status fp8_get_device_status(unsigned int* out) {
  if (!out) return FP8_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return FP8_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, fp8k::g_dev_status, sizeof(v)) != cudaSuccess) return FP8_ERR_CUDA;
  if (cudaMemcpyToSymbol(fp8k::g_dev_status, &zero, sizeof(zero)) != cudaSuccess) return FP8_ERR_CUDA;
  *out = v;
  return FP8_OK;
}

fp8_status fp8_repack_qat(const uint8_t* q4, const float* d, int64_t N, int64_t K, uint8_t* w8,
                          float* s_ch, void* stream) {
  return repack_qat_checked<kEncE4M3>(q4, d, N, K, w8, s_ch, as_stream(stream));
}

fp8_status fp8_convert_fnuz(const uint8_t* w8_fnuz, const float* s_fnuz, int64_t N, int64_t K,
                            uint8_t* w8, float* s_ch, void* stream) {
  if (!dims_ok(N, kMaxRows) || !dims_ok(K, int64_t(1) << 24)) return FP8_ERR_INVALID_ARG;
  if (K % 16 != 0) return FP8_ERR_SHAPE;
  if (N == 0) return FP8_OK;
  if (!w8_fnuz || !s_fnuz || !w8 || !s_ch) return FP8_ERR_INVALID_ARG;
  if (!aligned16(w8_fnuz) || !aligned16(w8) || !aligned4(s_fnuz) || !aligned4(s_ch))
    return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  const uint32_t row_pad = static_cast<uint32_t>((K + 127) / 128 * 128);
  const int64_t warps = std::min<int64_t>(8, kStagedSmemBudget / (2 * int64_t(row_pad) + 16));
  if (N >= 4 * dev->sm_count && K >= 128 && warps >= 2) {
    // Rows staged through shared memory, as many 8-warp blocks per SM as fit.
    const size_t smem = static_cast<size_t>(warps) * 2 * row_pad + 16 * warps;
    const int64_t per_sm =
        staged_blocks_per_sm(convert_fnuz_staged_kernel, static_cast<int>(32 * warps), smem);
    const int64_t blocks = std::min<int64_t>(per_sm * dev->sm_count, (N + warps - 1) / warps);
    convert_fnuz_staged_kernel<<<static_cast<unsigned>(blocks), static_cast<unsigned>(32 * warps),
                                 smem, as_stream(stream)>>>(w8_fnuz, s_fnuz, N, K, w8, s_ch, row_pad);
    return last_launch();
  }
  const dim3 grid(static_cast<unsigned>((N + 7) / 8));
  convert_fnuz_kernel<32><<<grid, 256, 0, as_stream(stream)>>>(w8_fnuz, s_fnuz, N, K, w8, s_ch);
  return last_launch();
}

fp8_status fp8_quant_act(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, uint8_t* x8,
                         float* s_tok, void* stream) {
  if (!dims_ok(M, kMaxRows) || !dims_ok(K, int64_t(1) << 24) || ldx < K) return FP8_ERR_INVALID_ARG;
  if (K % 16 != 0 || ldx % 8 != 0) return FP8_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8_OK;
  if (!x || !x8 || !s_tok) return FP8_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x8) || !aligned4(s_tok)) return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  return launch_quant_act(*dev, x, M, K, ldx, x8, s_tok, as_stream(stream));
}

static fp8_status check_linear(const void* x, const float* s_tok, const uint8_t* w8,
                               const float* s_ch, int64_t M, int64_t N, int64_t K,
                               const uint16_t* y) {
  if (!dims_ok(M, kMaxRows) || !dims_ok(N, kMaxRows) || !dims_ok(K, 65536))
    return FP8_ERR_INVALID_ARG;
  if (K % 16 != 0) return FP8_ERR_SHAPE;
  if (M == 0 || N == 0) return FP8_OK;
  if (!x || !s_tok || !w8 || !s_ch || !y) return FP8_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w8) || !aligned16(y) || !aligned4(s_tok) || !aligned4(s_ch))
    return FP8_ERR_ALIGNMENT;
  return FP8_OK;
}

fp8_status fp8_rowwise_linear(const uint8_t* x8, const float* s_tok, const uint8_t* w8,
                              const float* s_ch, int64_t M, int64_t N, int64_t K, uint16_t* y,
                              void* stream) {
  if (fp8_status st = check_linear(x8, s_tok, w8, s_ch, M, N, K, y)) return st;
  if (M == 0 || N == 0) return FP8_OK;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  if (K == 0) {
    if (cudaMemsetAsync(y, 0, static_cast<size_t>(M) * N * 2, as_stream(stream)) != cudaSuccess)
      return FP8_ERR_CUDA;
    return FP8_OK;
  }
  return launch_linear(*dev, x8, s_tok, w8, s_ch, static_cast<int>(M), static_cast<int>(N),
                       static_cast<int>(K), y, as_stream(stream), true);
}

size_t fp8_linear_workspace_bytes(void) {
  DeviceInfo* dev;
  if (device_info(&dev) != FP8_OK || dev->pair_clusters <= 0) return 0;
  return split_ws_bytes(dev->pair_clusters);
}

fp8_status fp8_rowwise_linear_ws(const uint8_t* x8, const float* s_tok, const uint8_t* w8,
                                 const float* s_ch, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                 void* ws, size_t ws_bytes, void* stream) {
  if (fp8_status st = check_linear(x8, s_tok, w8, s_ch, M, N, K, y)) return st;
  if (ws && !aligned16(ws)) return FP8_ERR_ALIGNMENT;
  if (M == 0 || N == 0) return FP8_OK;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  if (K == 0) {
    if (cudaMemsetAsync(y, 0, static_cast<size_t>(M) * N * 2, as_stream(stream)) != cudaSuccess)
      return FP8_ERR_CUDA;
    return FP8_OK;
  }
  return launch_linear(*dev, x8, s_tok, w8, s_ch, static_cast<int>(M), static_cast<int>(N),
                       static_cast<int>(K), y, as_stream(stream), true, ws, ws_bytes);
}

fp8_status fp8_linear_bf16(const uint16_t* x, const uint8_t* w8, const float* s_ch, int64_t M,
                           int64_t N, int64_t K, uint8_t* x8, float* s_tok, uint16_t* y,
                           void* stream) {
  if (fp8_status st = check_linear(x, s_tok, w8, s_ch, M, N, K, y)) return st;
  if (M == 0 || N == 0) return FP8_OK;
  if (!x8) return FP8_ERR_INVALID_ARG;
  if (!aligned16(x8)) return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  if (K == 0) {
    if (cudaMemsetAsync(y, 0, static_cast<size_t>(M) * N * 2, as_stream(stream)) != cudaSuccess)
      return FP8_ERR_CUDA;
    return FP8_OK;
  }
  // Two launches: the GEMM is a programmatic dependent of the quantizer, so
  // its weight stream starts while the quantizer runs. (Quantizing inside the
  // decode GEMM was measured slower on B200: every CTA must quantize the whole
  // token block, and staging it costs the second CTA per SM.)
  if (fp8_status st = launch_quant_act(*dev, x, M, K, K, x8, s_tok, as_stream(stream))) return st;
  return launch_linear(*dev, x8, s_tok, w8, s_ch, static_cast<int>(M), static_cast<int>(N),
                       static_cast<int>(K), y, as_stream(stream), true);
}

fp8_status fp8_linear_bf16_siblings(const uint16_t* x, int64_t M, int64_t K, int32_t count,
                                    const uint8_t* const* w8, const float* const* s_ch,
                                    const int64_t* N, uint8_t* x8, float* s_tok,
                                    uint16_t* const* y, void* stream) {
  if (count < 1 || count > 16 || !w8 || !s_ch || !N || !y) return FP8_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i)
    if (fp8_status st = check_linear(x, s_tok, w8[i], s_ch[i], M, N[i], K, y[i])) return st;
  if (M == 0) return FP8_OK;
  if (!x8) return FP8_ERR_INVALID_ARG;
  if (!aligned16(x8)) return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  const cudaStream_t stream_ = as_stream(stream);
  if (K == 0) {
    for (int i = 0; i < count; ++i)
      if (N[i] > 0 && cudaMemsetAsync(y[i], 0, static_cast<size_t>(M) * N[i] * 2, stream_) != cudaSuccess)
        return FP8_ERR_CUDA;
    return FP8_OK;
  }
  // One quantization of x, then every GEMM as a programmatic dependent of the
  // one before (each reads only w8 / s_ch before its grid-dependency wait).
  if (fp8_status st = launch_quant_act(*dev, x, M, K, K, x8, s_tok, stream_)) return st;
  for (int i = 0; i < count; ++i) {
    if (N[i] == 0) continue;
    if (fp8_status st = launch_linear(*dev, x8, s_tok, w8[i], s_ch[i], static_cast<int>(M),
                                      static_cast<int>(N[i]), static_cast<int>(K), y[i], stream_, true))
      return st;
  }
  return FP8_OK;
}

fp8_status fp8_cast_e4m3(const float* x, int64_t n, uint8_t* out, void* stream) {
  if (n < 0 || n > (int64_t(1) << 40)) return FP8_ERR_INVALID_ARG;
  if (n == 0) return FP8_OK;
  if (!x || !out) return FP8_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  const int64_t threads = (n + 3) / 4;
  const dim3 grid(static_cast<unsigned>((threads + 255) / 256));
  cast_e4m3_kernel<<<grid, 256, 0, as_stream(stream)>>>(x, n, out);
  return last_launch();
}

fp8_status fp8_moe_route(const int32_t* topk_ids, int64_t tokens, int32_t top_k,
                         int32_t num_experts, int32_t* perm, int32_t* inv, int32_t* offsets,
                         void* stream) {
  if (tokens < 0 || top_k < 1 || num_experts < 1 || num_experts > kMaxExperts)
    return FP8_ERR_INVALID_ARG;
  const int64_t n = tokens * top_k;
  if (n >= (int64_t(1) << 31)) return FP8_ERR_SHAPE;
  if (!offsets || (n > 0 && (!topk_ids || !perm || !inv))) return FP8_ERR_INVALID_ARG;
  if (!aligned4(topk_ids) || !aligned4(perm) || !aligned4(inv) || !aligned4(offsets))
    return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  return launch_pdl(moe_route_kernel, dim3(num_experts), dim3(kRouteThreads), as_stream(stream),
                    topk_ids, n, static_cast<int>(num_experts), perm, inv, offsets);
}

fp8_status fp8_moe_gather(const uint8_t* x8, const float* s_tok, const int32_t* perm,
                          int64_t rows, int64_t K, int32_t top_k, uint8_t* x8_rows,
                          float* s_rows, void* stream) {
  if (rows < 0 || K < 0 || top_k < 1) return FP8_ERR_INVALID_ARG;
  if (K % 16 != 0) return FP8_ERR_SHAPE;
  if (rows == 0 || K == 0) return FP8_OK;
  if (!x8 || !s_tok || !perm || !x8_rows || !s_rows) return FP8_ERR_INVALID_ARG;
  if (!aligned16(x8) || !aligned16(x8_rows) || !aligned4(s_tok) || !aligned4(perm) ||
      !aligned4(s_rows))
    return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  return launch_pdl(moe_gather_kernel, dim3(static_cast<unsigned>((rows + 7) / 8)), dim3(256),
                    as_stream(stream), x8, s_tok, perm, rows, K, static_cast<int>(top_k), x8_rows,
                    s_rows);
}

fp8_status fp8_grouped_linear(const uint8_t* x8_rows, const float* s_rows, const int32_t* offsets,
                              int32_t num_experts, int64_t M_total, const uint8_t* w8,
                              const float* s_ch, int64_t N, int64_t K, uint16_t* y, void* stream) {
  if (num_experts < 1 || num_experts > kMaxExperts) return FP8_ERR_INVALID_ARG;
  if (fp8_status st = check_linear(x8_rows, s_rows, w8, s_ch, M_total, N, K, y)) return st;
  if (M_total == 0 || N == 0) return FP8_OK;
  if (!offsets) return FP8_ERR_INVALID_ARG;
  if (!aligned4(offsets)) return FP8_ERR_ALIGNMENT;
  if (static_cast<int64_t>(num_experts) * N >= (int64_t(1) << 31)) return FP8_ERR_SHAPE;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  if (K == 0) {
    if (cudaMemsetAsync(y, 0, static_cast<size_t>(M_total) * N * 2, as_stream(stream)) != cudaSuccess)
      return FP8_ERR_CUDA;
    return FP8_OK;
  }
  // 256-column tiles even when N is not a multiple of 256: measured on B200,
  // the wider tile's halved operand traffic per MMA outweighs a partly empty
  // last tile (N = 1408: 245 us vs 265 us with 128-column tiles).
  if (dev->pair_clusters > 0)
    return launch_grouped_pair(*dev, x8_rows, s_rows, offsets, num_experts,
                               static_cast<int>(M_total), w8, s_ch, static_cast<int>(N),
                               static_cast<int>(K), y, as_stream(stream));
  return launch_grouped<256, kPrefillStages>(*dev, x8_rows, s_rows, offsets, num_experts,
                                             static_cast<int>(M_total), w8, s_ch,
                                             static_cast<int>(N), static_cast<int>(K), y,
                                             as_stream(stream));
}

fp8_status fp8_moe_interleave_gate_up(const uint8_t* w8, const float* s_ch, int32_t num_experts,
                                      int64_t inter, int64_t K, uint8_t* w8_il, float* s_il,
                                      void* stream) {
  if (num_experts < 1 || num_experts > kMaxExperts || inter < 1 || !dims_ok(K, 65536))
    return FP8_ERR_INVALID_ARG;
  if (K % 16 != 0 || inter % 16 != 0) return FP8_ERR_SHAPE;
  const int64_t tiles = (inter + 127) / 128;
  const int64_t rows_out = static_cast<int64_t>(num_experts) * 256 * tiles;
  if (rows_out >= (int64_t(1) << 31) || static_cast<int64_t>(num_experts) * 2 * inter >= (int64_t(1) << 31))
    return FP8_ERR_SHAPE;
  if (!w8 || !s_ch || !w8_il || !s_il) return FP8_ERR_INVALID_ARG;
  if (!aligned16(w8) || !aligned16(w8_il) || !aligned4(s_ch) || !aligned4(s_il))
    return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  moe_interleave_gate_up_kernel<<<static_cast<unsigned>((rows_out + 7) / 8), 256, 0,
                                  as_stream(stream)>>>(w8, s_ch, num_experts, inter, K, tiles, w8_il,
                                                       s_il);
  return last_launch();
}

fp8_status fp8_grouped_linear_geglu(const uint8_t* x8_rows, const float* s_rows,
                                    const int32_t* offsets, int32_t num_experts, int64_t M_total,
                                    const uint8_t* w8_il, const float* s_il, int64_t inter,
                                    int64_t K, uint16_t* h, void* stream) {
  if (num_experts < 1 || num_experts > kMaxExperts || inter < 1) return FP8_ERR_INVALID_ARG;
  if (inter % 16 != 0) return FP8_ERR_SHAPE;
  const int64_t n_il = 256 * ((inter + 127) / 128);  // interleaved rows per expert
  if (fp8_status st = check_linear(x8_rows, s_rows, w8_il, s_il, M_total, n_il, K, h)) return st;
  if (M_total == 0) return FP8_OK;
  if (!offsets) return FP8_ERR_INVALID_ARG;
  if (!aligned4(offsets) || !aligned16(s_il)) return FP8_ERR_ALIGNMENT;
  if (static_cast<int64_t>(num_experts) * n_il >= (int64_t(1) << 31)) return FP8_ERR_SHAPE;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  if (dev->pair_clusters <= 0) return FP8_ERR_UNSUPPORTED;
  if (K == 0) {  // gate = up = 0, so h = 0
    if (cudaMemsetAsync(h, 0, static_cast<size_t>(M_total) * inter * 2, as_stream(stream)) !=
        cudaSuccess)
      return FP8_ERR_CUDA;
    return FP8_OK;
  }
  return launch_grouped_pair(*dev, x8_rows, s_rows, offsets, num_experts, static_cast<int>(M_total),
                             w8_il, s_il, static_cast<int>(n_il), static_cast<int>(K), h,
                             as_stream(stream), static_cast<int>(inter));
}

fp8_status fp8_moe_geglu_quant(const uint16_t* gate_up, int64_t M, int64_t inter, uint8_t* h8,
                               float* s_h, uint16_t* h_out, void* stream) {
  if (M < 0 || inter < 0) return FP8_ERR_INVALID_ARG;
  if (inter % 16 != 0) return FP8_ERR_SHAPE;
  if (M == 0 || inter == 0) return FP8_OK;
  if (!gate_up || !h8 || !s_h) return FP8_ERR_INVALID_ARG;
  if (!aligned16(gate_up) || !aligned16(h8) || !aligned4(s_h) || (h_out && !aligned16(h_out)))
    return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  return launch_pdl(moe_geglu_quant_kernel, dim3(static_cast<unsigned>((M + 7) / 8)), dim3(256),
                    as_stream(stream), gate_up, M, inter, h8, s_h, h_out);
}

fp8_status fp8_moe_combine(const uint16_t* rows, const int32_t* inv, int64_t tokens,
                           int32_t top_k, int64_t H, const float* weights, uint16_t* out,
                           void* stream) {
  if (tokens < 0 || top_k < 1 || top_k > kCombineMaxK || H < 0) return FP8_ERR_INVALID_ARG;
  if (H % 8 != 0) return FP8_ERR_SHAPE;
  if (tokens == 0 || H == 0) return FP8_OK;
  if (!rows || !inv || !out) return FP8_ERR_INVALID_ARG;
  if (!aligned16(rows) || !aligned16(out) || !aligned4(inv) || (weights && !aligned4(weights)))
    return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  const dim3 grid(static_cast<unsigned>((tokens + 7) / 8));
  if (top_k <= 8)
    return launch_pdl(moe_combine_kernel<8>, grid, dim3(256), as_stream(stream), rows, inv, tokens,
                      static_cast<int>(top_k), H, weights, out);
  return launch_pdl(moe_combine_kernel<kCombineMaxK>, grid, dim3(256), as_stream(stream), rows, inv,
                    tokens, static_cast<int>(top_k), H, weights, out);
}

// ------------------------------------------------------------ bf16 GEMM, router
fp8_status bf16_linear(const uint16_t* x, const uint16_t* w, int64_t M, int64_t N, int64_t K,
                       uint16_t* y, void* stream) {
  if (!dims_ok(M, kMaxRows) || !dims_ok(N, kMaxRows) || !dims_ok(K, 32768)) return FP8_ERR_INVALID_ARG;
  if (K % 8 != 0) return FP8_ERR_SHAPE;
  if (M == 0 || N == 0) return FP8_OK;
  if (!x || !w || !y) return FP8_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  if (K == 0) {
    if (cudaMemsetAsync(y, 0, static_cast<size_t>(M) * N * 2, as_stream(stream)) != cudaSuccess)
      return FP8_ERR_CUDA;
    return FP8_OK;
  }
  // bf16 rows are 2K bytes; no scales (y = bf16(acc)).
  return launch_linear<kKindBF16>(*dev, reinterpret_cast<const uint8_t*>(x), nullptr,
                                  reinterpret_cast<const uint8_t*>(w), nullptr, static_cast<int>(M),
                                  static_cast<int>(N), static_cast<int>(2 * K), y, as_stream(stream),
                                  true);
}

fp8_status fp8_moe_topk(const uint16_t* logits, int64_t tokens, int32_t num_experts, int32_t top_k,
                        int32_t* ids, float* weights, void* stream) {
  if (tokens < 0 || num_experts < 1 || num_experts > kTopkMaxE || top_k < 1 || top_k > kTopkMaxK ||
      top_k > num_experts)
    return FP8_ERR_INVALID_ARG;
  if (tokens == 0) return FP8_OK;
  if (!logits || !ids || !weights) return FP8_ERR_INVALID_ARG;
  if (!aligned4(ids) || !aligned4(weights) || (reinterpret_cast<uintptr_t>(logits) & 1))
    return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  const dim3 grid(static_cast<unsigned>((tokens + 7) / 8));
  const cudaStream_t st = as_stream(stream);
  if (num_experts <= 128)
    return launch_pdl(moe_topk_kernel<4>, grid, dim3(256), st, logits, tokens, num_experts, top_k, ids, weights);
  if (num_experts <= 256)
    return launch_pdl(moe_topk_kernel<8>, grid, dim3(256), st, logits, tokens, num_experts, top_k, ids, weights);
  return launch_pdl(moe_topk_kernel<32>, grid, dim3(256), st, logits, tokens, num_experts, top_k, ids, weights);
}

// ------------------------------------------------------------ W4A16 build
static fp8_status w4a16_check(const uint8_t* q4, const float* d, int64_t N, int64_t K) {
  if (!dims_ok(N, kMaxRows) || !dims_ok(K, 32768)) return FP8_ERR_INVALID_ARG;
  if (K % 32 != 0) return FP8_ERR_SHAPE;
  if (N > 0 && K > 0 && (!q4 || !d)) return FP8_ERR_INVALID_ARG;
  if (!aligned16(q4) || !aligned4(d)) return FP8_ERR_ALIGNMENT;
  return FP8_OK;
}

fp8_status w4a16_dequant(const uint8_t* q4, const float* d, int64_t N, int64_t K, uint16_t* w,
                         void* stream) {
  if (fp8_status st = w4a16_check(q4, d, N, K)) return st;
  if (N == 0 || K == 0) return FP8_OK;
  if (!w) return FP8_ERR_INVALID_ARG;
  if (!aligned16(w)) return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  const int64_t groups = N * (K / 32);
  const int64_t blocks = std::min<int64_t>((groups + 255) / 256, int64_t(dev->sm_count) * 8);
  return launch_pdl(w4a16_dequant_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256),
                    as_stream(stream), q4, d, groups, w);
}

size_t w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  if (M <= 128 && K % 128 == 0) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(K) * 2;
}

fp8_status w4a16_linear(const uint16_t* x, const uint8_t* q4, const float* d, int64_t M, int64_t N,
                        int64_t K, uint16_t* y, uint16_t* w_ws, size_t ws_bytes, void* stream) {
  if (fp8_status st = w4a16_check(q4, d, N, K)) return st;
  if (!dims_ok(M, kMaxRows)) return FP8_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return FP8_OK;
  if (!x || !y) return FP8_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  if (K == 0) {
    if (cudaMemsetAsync(y, 0, static_cast<size_t>(M) * N * 2, as_stream(stream)) != cudaSuccess)
      return FP8_ERR_CUDA;
    return FP8_OK;
  }
  const size_t need = w4a16_workspace_bytes(M, N, K);
  if (need == 0)
    return launch_w4_decode(*dev, x, q4, d, static_cast<int>(M), static_cast<int>(N),
                            static_cast<int>(K), y, as_stream(stream));
  if (!w_ws || ws_bytes < need) return FP8_ERR_INVALID_ARG;
  if (!aligned16(w_ws)) return FP8_ERR_ALIGNMENT;
  if (fp8_status st = w4a16_dequant(q4, d, N, K, w_ws, stream)) return st;
  return launch_linear<kKindBF16>(*dev, reinterpret_cast<const uint8_t*>(x), nullptr,
                                  reinterpret_cast<const uint8_t*>(w_ws), nullptr, static_cast<int>(M),
                                  static_cast<int>(N), static_cast<int>(2 * K), y, as_stream(stream),
                                  true);
}

// ------------------------------------------------------------ int8 W8A8 build
fp8_status int8_repack_qat(const uint8_t* q4, const float* d, int64_t N, int64_t K, int8_t* w8,
                           float* s_ch, void* stream) {
  return repack_qat_checked<kEncI8>(q4, d, N, K, reinterpret_cast<uint8_t*>(w8), s_ch,
                                    as_stream(stream));
}

fp8_status int8_quant_act(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int8_t* x8,
                          float* s_tok, void* stream) {
  if (!dims_ok(M, kMaxRows) || !dims_ok(K, int64_t(1) << 24) || ldx < K) return FP8_ERR_INVALID_ARG;
  if (K % 16 != 0 || ldx % 8 != 0) return FP8_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8_OK;
  if (!x || !x8 || !s_tok) return FP8_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x8) || !aligned4(s_tok)) return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  return launch_quant_act<kEncI8>(*dev, x, M, K, ldx, reinterpret_cast<uint8_t*>(x8), s_tok,
                                  as_stream(stream));
}

fp8_status int8_rowwise_linear(const int8_t* x8, const float* s_tok, const int8_t* w8,
                               const float* s_ch, int64_t M, int64_t N, int64_t K, uint16_t* y,
                               void* stream) {
  if (fp8_status st = check_linear(x8, s_tok, reinterpret_cast<const uint8_t*>(w8), s_ch, M, N, K, y))
    return st;
  if (M == 0 || N == 0) return FP8_OK;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  if (K == 0) {
    if (cudaMemsetAsync(y, 0, static_cast<size_t>(M) * N * 2, as_stream(stream)) != cudaSuccess)
      return FP8_ERR_CUDA;
    return FP8_OK;
  }
  return launch_linear<kKindS8>(*dev, reinterpret_cast<const uint8_t*>(x8), s_tok,
                                reinterpret_cast<const uint8_t*>(w8), s_ch, static_cast<int>(M),
                                static_cast<int>(N), static_cast<int>(K), y, as_stream(stream), true);
}

fp8_status int8_rowwise_linear_ws(const int8_t* x8, const float* s_tok, const int8_t* w8,
                                  const float* s_ch, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                  void* ws, size_t ws_bytes, void* stream) {
  if (fp8_status st = check_linear(x8, s_tok, reinterpret_cast<const uint8_t*>(w8), s_ch, M, N, K, y))
    return st;
  if (ws && !aligned16(ws)) return FP8_ERR_ALIGNMENT;
  if (M == 0 || N == 0) return FP8_OK;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  if (K == 0) {
    if (cudaMemsetAsync(y, 0, static_cast<size_t>(M) * N * 2, as_stream(stream)) != cudaSuccess)
      return FP8_ERR_CUDA;
    return FP8_OK;
  }
  return launch_linear<kKindS8>(*dev, reinterpret_cast<const uint8_t*>(x8), s_tok,
                                reinterpret_cast<const uint8_t*>(w8), s_ch, static_cast<int>(M),
                                static_cast<int>(N), static_cast<int>(K), y, as_stream(stream), true, ws,
                                ws_bytes);
}

fp8_status int8_linear_bf16(const uint16_t* x, const int8_t* w8, const float* s_ch, int64_t M,
                            int64_t N, int64_t K, int8_t* x8, float* s_tok, uint16_t* y,
                            void* stream) {
  if (fp8_status st = check_linear(x, s_tok, reinterpret_cast<const uint8_t*>(w8), s_ch, M, N, K, y))
    return st;
  if (M == 0 || N == 0) return FP8_OK;
  if (!x8) return FP8_ERR_INVALID_ARG;
  if (!aligned16(x8)) return FP8_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  if (K == 0) {
    if (cudaMemsetAsync(y, 0, static_cast<size_t>(M) * N * 2, as_stream(stream)) != cudaSuccess)
      return FP8_ERR_CUDA;
    return FP8_OK;
  }
  uint8_t* xq = reinterpret_cast<uint8_t*>(x8);
  if (fp8_status st = launch_quant_act<kEncI8>(*dev, x, M, K, K, xq, s_tok, as_stream(stream))) return st;
  return launch_linear<kKindS8>(*dev, xq, s_tok, reinterpret_cast<const uint8_t*>(w8), s_ch,
                                static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), y,
                                as_stream(stream), true);
}

}  // extern "C"

// ============================================================ no-alloc linear
// Scratch for fp8_linear_bf16_noalloc: quantized activations, then scales.
// Host code must not use this symbol as a device address; it goes through
// the per-device address looked up below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FP8_NOALLOC_SCRATCH_BYTES];

namespace {
uint8_t* g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch array for the current device, looked up once
// per device (with that device current) and cached.
fp8_status noalloc_scratch(uint8_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FP8_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return FP8_OK;
}
}  // namespace

extern "C" fp8_status fp8_linear_bf16_noalloc(const uint16_t* x, const uint8_t* w8,
                                              const float* s_ch, int64_t M, int64_t N, int64_t K,
                                              uint16_t* y, void* stream) {
  // Any 16-byte-aligned stand-in passes the pointer checks for the scratch
  // operands; the real scratch addresses are substituted below.
  const float* scratch_probe = s_ch;
  if (fp8_status st = check_linear(x, scratch_probe, w8, s_ch, M, N, K, y)) return st;
  if (M == 0 || N == 0) return FP8_OK;
  const uint64_t x8_bytes = (static_cast<uint64_t>(M) * static_cast<uint64_t>(K) + 255u) & ~uint64_t(255);
  const uint64_t need = x8_bytes + 4u * static_cast<uint64_t>(M);
  if (need > FP8_NOALLOC_SCRATCH_BYTES) return FP8_ERR_SCRATCH_LIMIT;
  DeviceInfo* dev;
  if (fp8_status st = device_info(&dev)) return st;
  uint8_t* scratch = nullptr;
  if (fp8_status st = noalloc_scratch(&scratch)) return st;
  uint8_t* x8 = scratch;
  float* s_tok = reinterpret_cast<float*>(scratch + x8_bytes);
  if (K == 0) {
    if (cudaMemsetAsync(y, 0, static_cast<size_t>(M) * N * 2, as_stream(stream)) != cudaSuccess)
      return FP8_ERR_CUDA;
    return FP8_OK;
  }
  if (fp8_status st = launch_quant_act(*dev, x, M, K, K, x8, s_tok, as_stream(stream))) return st;
  return launch_linear(*dev, x8, s_tok, w8, s_ch, static_cast<int>(M), static_cast<int>(N),
                       static_cast<int>(K), y, as_stream(stream), true);
}
