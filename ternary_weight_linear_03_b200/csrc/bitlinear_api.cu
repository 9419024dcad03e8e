// C ABI of the BitLinear library (declared in include/bitlinear.h): argument checks,
// workspace layout, kernel selection and launches. One translation unit holds every
// kernel so that the device status word is a single object per device.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/bitlinear.h"
#include "act_quant.cuh"
#include "common.cuh"
#include "gemm_bf16.cuh"
#include "gemm_prefill.cuh"
#include "gemm_skinny.cuh"
#include "gemv.cuh"
#include "gemv3.cuh"
#include "per_device.h"
#include "rescale.cuh"
#include "weight_quant.cuh"

namespace {

using bl::WqWorkspace;

constexpr int kGemvMaxM = 4;            // M above this runs a tensor-core kernel
constexpr int kSkinnyMaxM = 256;        // M above this runs the prefill GEMM
static_assert(kSkinnyMaxM <= bl::sk::MAX_M, "the skinny kernel stages per-token factors for MAX_M tokens");
constexpr int kGemvMaxSmem = 200 * 1024;  // xq rows held in shared memory by the GEMV
constexpr unsigned long long kWaitLimitNs = 4000000000ull;  // 4 s per mbarrier wait
constexpr int kMinKbPerSplit = 8;  // skinny split-K: K blocks per split, at least

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool shape_ok(long long M, long long N, long long K) {
  if (M < 1 || N < 1 || K < 64 || (K % 64) != 0) return false;
  const long long lim = 1ll << 31;
  return M * K < lim && N * K < lim && M * N < lim;
}

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

// Multiprocessors of the current device (148 on B200 if the query fails).
int num_sms() {
  static bl::PerDevice cache;
  const int v = cache.get(current_device(), [](int dev) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return sms;
  });
  return v > 0 ? v : 148;
}

// Raises `kern`'s dynamic shared-memory limit to `bytes` on the current device, once per
// device (the attribute belongs to that device's context). False if the call failed.
template <class Kernel>
bool set_smem_limit_once(bl::PerDevice& cache, Kernel kern, int bytes) {
  return cache.get(current_device(), [&](int) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
                   cudaSuccess
               ? 1
               : 0;
  }) > 0;
}

// The CUDA-core GEMV for one or two tokens, and for up to kGemvMaxM tokens when the packed
// weights are small (at most 2 MB, where the tensor-core kernel's fixed latency dominates);
// measured on B200 against the skinny tensor-core kernel on the decode shapes.
bool use_gemv(int M, int N, int K) {
  if (static_cast<long long>(M) * K > kGemvMaxSmem) return false;
  return M <= 2 || (M <= kGemvMaxM && static_cast<long long>(N) * K / 4 <= (2ll << 20));
}

// Workspace layout of the forward / contract paths that run the GEMM:
//   [xq M*K int8][scale M fp32][rowsum M int32], each 256-byte aligned.
struct FwdWs {
  int8_t* xq;
  float* scale;
  int* rowsum;
  size_t bytes;
};
FwdWs fwd_ws_layout(void* base, int M, int K) {
  FwdWs w{};
  const size_t a = align_up(static_cast<size_t>(M) * K, 256);
  const size_t b = align_up(static_cast<size_t>(M) * 4, 256);
  char* p = static_cast<char*>(base);
  w.xq = reinterpret_cast<int8_t*>(p);
  w.scale = reinterpret_cast<float*>(p + a);
  w.rowsum = reinterpret_cast<int*>(p + a + b);
  w.bytes = a + 2 * b;
  return w;
}

// Split-K plan of the skinny tensor-core kernel for M tokens (4 < M <= 256).
struct SkinnyPlan {
  int bnt;     // token tile: M rounded up to a multiple of 16
  int tiles;   // 128-row weight tiles
  int splits;  // K ranges per tile
  int kbps;    // 128-wide K blocks per split
};
// sums_share: the int32 sums of one split may reach 1/sums_share of the packed weight bytes
// (4 for a single forward, whose quantization kernel clears the sums on every call; 1
// inside a layer chain, which clears them once per call and whose kernels leave them
// cleared).
SkinnyPlan skinny_plan_for(int M, int N, int K, int sms, int sums_share = 4) {
  SkinnyPlan p{};
  p.bnt = (M + 15) / 16 * 16;
  p.tiles = (N + bl::sk::BW - 1) / bl::sk::BW;
  const int KB = (K + bl::sk::BK - 1) / bl::sk::BK;
  // Split K only when the weight tiles alone leave CTA slots idle (two per SM for token
  // tiles up to 64, one above), and only as far as every CTA still has a slot: a CTA
  // runs at the pace of its handoffs, so a second wave would double the time. Keep at
  // least kMinKbPerSplit K blocks per split so that each CTA streams long enough to cover
  // its fixed costs, and keep the int32 sums the splits exchange (M x N x 4 bytes each)
  // within 1/sums_share of the packed weight bytes (measured on B200, single forwards:
  // beyond a quarter, clearing and reducing the sums costs more than the extra SMs bring;
  // in a chain, which clears them only once, up to the weight bytes paid: 3B sweep at 64
  // tokens 1.35 -> 1.32 ms).
  const long long slots = static_cast<long long>(p.bnt <= 64 ? 2 : 1) * sms;
  long long splits = 1;
  if (p.tiles < slots) splits = std::max<long long>(1, slots / p.tiles);
  const long long by_traffic = static_cast<long long>(
      (static_cast<double>(N) * K / 4.0) /
      (static_cast<double>(sums_share) * 4.0 * static_cast<double>(M) * N));
  splits = std::max<long long>(
      1, std::min<long long>({splits, std::max(1, KB / kMinKbPerSplit), by_traffic}));
  p.kbps = static_cast<int>((KB + splits - 1) / splits);
  p.kbps = (p.kbps + bl::sk::KPS - 1) / bl::sk::KPS * bl::sk::KPS;  // whole super-tiles
  p.splits = (KB + p.kbps - 1) / p.kbps;                          // no empty split
  return p;
}
SkinnyPlan skinny_plan(int M, int N, int K) { return skinny_plan_for(M, N, K, num_sms()); }
SkinnyPlan skinny_plan_chain(int M, int N, int K) {
  return skinny_plan_for(M, N, K, num_sms(), 1);
}

// Workspace of the skinny path: the FwdWs part, then (only when splits > 1) the int32
// sums [M][N] and one arrival counter per weight tile, contiguous so one memset clears
// both.
struct SkinnyWs {
  int* partial;
  unsigned int* counters;
  size_t bytes;  // total, including the FwdWs part
};
SkinnyWs skinny_ws_layout(void* base, int M, int N, int K, const SkinnyPlan& p) {
  SkinnyWs w{};
  const size_t head = fwd_ws_layout(nullptr, M, K).bytes;
  const size_t part = (p.splits > 1) ? align_up(static_cast<size_t>(M) * N * 4, 256) : 0;
  const size_t cnt = align_up(static_cast<size_t>(p.tiles) * 4, 256);
  char* c = static_cast<char*>(base);
  w.partial = reinterpret_cast<int*>(c + head);
  w.counters = reinterpret_cast<unsigned int*>(c + head + part);
  w.bytes = head + part + cnt;
  return w;
}

bl_status launch_status() {
  return (cudaGetLastError() == cudaSuccess) ? BL_OK : BL_ERR_CUDA;
}

// Options of a launch inside a layer chain (bitlinear_chain_forward); all off for the
// single-layer entry points.
struct ChainOpts {
  const float* amax_in = nullptr;  // absmax of the input rows, from the kernel that wrote them
  float* amax_out = nullptr;       // receives the absmax of this launch's output rows
  bool pdl = false;                // programmatic dependent launch on the kernel before
};

// Launches kern with or without programmatic stream serialization.
template <typename... KArgs, typename... Args>
bl_status launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                    bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess)
    return BL_ERR_CUDA;
  return launch_status();
}

// ------------------------------------------------------------------ TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
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

// 2-D uint8 tensor [rows][cols] with row pitch `pitch` bytes, box [box_rows][box_cols].
bool make_map_u8(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                 uint64_t pitch, uint32_t box_cols, uint32_t box_rows, bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 2-D tensor [rows][cols] (row pitch cols * 2 bytes), box [box_rows][64], 128-byte
// swizzle (64 bf16 = one swizzle row).
bool make_map_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                   uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ GEMV launch
// Lanes per weight row of the GEMV (log2). Small matrices need more lanes per row to give
// every SM work, at the price of idle lanes on short rows. Measured on B200 (3B and 700M
// shapes): for one token, the fewest lanes that keep the row's activations in registers
// (at most kGemvRegChunks chunks per lane) with blocks (16 warps x 32 / lanes rows each)
// for at least half the SMs; otherwise the fewest lanes whose blocks cover every SM for
// long rows (64 chunks or more), half of them for short rows.
int choose_lpr_log2(int cpr);
int gemv_lpr_log2(int cpr, int N, int M) {
  const int best = choose_lpr_log2(cpr);
  const long long half = (num_sms() + 1) / 2;
  auto blocks = [&](int l) {
    const long long rows_per_block = static_cast<long long>(bl::kGemvWarps) * (32 >> l);
    return (N + rows_per_block - 1) / rows_per_block;
  };
  if (M == 1)
    for (int l = best; l <= 5; ++l)
      if (((cpr + (1 << l) - 1) >> l) <= bl::kGemvRegChunks && blocks(l) >= half) return l;
  const long long want = (cpr >= 64) ? num_sms() : half;
  for (int l = best; l <= 5; ++l)
    if (blocks(l) >= want) return l;
  return 5;
}

int choose_lpr_log2(int cpr) {
  int best = 5;
  long long best_cost = (cpr + 31) / 32 * 32;
  for (int l = 4; l >= 2; --l) {
    const int L = 1 << l;
    const long long cost = static_cast<long long>(cpr + L - 1) / L * L;
    if (cost < best_cost) { best = l; best_cost = cost; }
  }
  return best;
}

template <int MT, int XM, int OM, bool XR, int R>
bl_status launch_gemv_t(const void* x, const uint8_t* packed, const float* gamma, void* y,
                        int N, int K, cudaStream_t s, const ChainOpts& o) {
  auto kern = bl::gemv_kernel<MT, XM, OM, XR, R>;
  const int smem = MT * K;
  static bl::PerDevice configured;
  if (!set_smem_limit_once(configured, kern, kGemvMaxSmem)) return BL_ERR_CUDA;
  int blocks_per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, kern, bl::kGemvThreads,
                                                    smem) != cudaSuccess ||
      blocks_per_sm < 1)
    blocks_per_sm = 1;
  const int lpr_log2 = gemv_lpr_log2(K / 64, N, MT);
  const long long rows_per_block = static_cast<long long>(bl::kGemvWarps) * (32 >> lpr_log2) * R;
  const long long need = (N + rows_per_block - 1) / rows_per_block;
  const long long slots = 1ll * blocks_per_sm * num_sms();
  const long long rpw = 32 >> lpr_log2;  // rows of one warp turn
  // The register path hands rows out block by block: just enough blocks. The shared-memory
  // path numbers warps across the grid, so it takes the same number of blocks on every SM
  // (every resident slot, or one per SM when fewer blocks would do) and the rows spread
  // evenly over them.
  const int grid = static_cast<int>(
      XR ? std::min(need, slots)
         : (need > num_sms() ? slots : std::min<long long>(num_sms(), (N + rpw - 1) / rpw)));
  const int chain = o.pdl ? 1 : 0;
  return launch_ex(kern, dim3(grid), dim3(bl::kGemvThreads), smem, s, o.pdl, x, packed, gamma,
                   y, N, K, lpr_log2, o.amax_in, o.amax_out, chain);
}

// Activations stay in registers for one token when a lane owns at most kGemvRegChunks
// chunks of a row (two tokens would spill).
bool gemv_x_in_registers(int M, int N, int K) {
  const int cpr = K / 64;
  const int lpr = 1 << gemv_lpr_log2(cpr, N, M);
  return M == 1 && (cpr + lpr - 1) / lpr <= bl::kGemvRegChunks;
}

// Rows summed at once per warp on the shared-memory path: two when one warp covers a
// whole row (large K) and there are rows enough for every warp of the GPU twice over.
bool gemv_two_rows(int M, int N, int K) {
  return gemv_lpr_log2(K / 64, N, M) == 5 && N >= 2 * bl::kGemvWarps * num_sms();
}

template <int MT, int XM, int OM>
bl_status launch_gemv_r(const void* x, const uint8_t* packed, const float* gamma, void* y,
                        int N, int K, cudaStream_t s, const ChainOpts& o) {
  return gemv_two_rows(MT, N, K)
             ? launch_gemv_t<MT, XM, OM, false, 2>(x, packed, gamma, y, N, K, s, o)
             : launch_gemv_t<MT, XM, OM, false, 1>(x, packed, gamma, y, N, K, s, o);
}

template <int XM, int OM>
bl_status launch_gemv_m(const void* x, const uint8_t* packed, const float* gamma, void* y,
                        int M, int N, int K, cudaStream_t s, const ChainOpts& o) {
  switch (M) {
    case 1:
      return gemv_x_in_registers(M, N, K)
                 ? launch_gemv_t<1, XM, OM, true, 1>(x, packed, gamma, y, N, K, s, o)
                 : launch_gemv_r<1, XM, OM>(x, packed, gamma, y, N, K, s, o);
    case 2: return launch_gemv_r<2, XM, OM>(x, packed, gamma, y, N, K, s, o);
    case 3: return launch_gemv_r<3, XM, OM>(x, packed, gamma, y, N, K, s, o);
    case 4: return launch_gemv_r<4, XM, OM>(x, packed, gamma, y, N, K, s, o);
    default: return BL_ERR_UNSUPPORTED_SHAPE;
  }
}

template <int XM>
bl_status launch_gemv_x(const void* x, const uint8_t* packed, const float* gamma, void* y,
                        int y_dtype, int M, int N, int K, cudaStream_t s,
                        const ChainOpts& o = {}) {
  switch (y_dtype) {
    case BL_F32: return launch_gemv_m<XM, bl::kOf32>(x, packed, gamma, y, M, N, K, s, o);
    case BL_BF16: return launch_gemv_m<XM, bl::kObf16>(x, packed, gamma, y, M, N, K, s, o);
    case BL_I32: return launch_gemv_m<XM, bl::kOi32>(x, packed, gamma, y, M, N, K, s, o);
    default: return BL_ERR_INVALID_ARG;
  }
}

// ------------------------------------------------------------------ base-3 GEMV launch
constexpr int kGemv3MaxM = 4;

template <int MT, int XM, int OM>
bl_status launch_gemv3_t(const void* x, const uint8_t* packed3, const float* gamma, void* y,
                         int N, int K, cudaStream_t s) {
  auto kern = bl::gemv3_kernel<MT, XM, OM>;
  const int CH = (K + 79) / 80;
  const int smem = MT * 80 * CH;
  static bl::PerDevice configured;
  if (!set_smem_limit_once(configured, kern, kGemvMaxSmem)) return BL_ERR_CUDA;
  int blocks_per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, kern, bl::kGemv3Threads,
                                                    smem) != cudaSuccess ||
      blocks_per_sm < 1)
    blocks_per_sm = 1;
  const int lpr_log2 = choose_lpr_log2(CH);
  const long long rows_per_block = static_cast<long long>(bl::kGemv3Warps) * (32 >> lpr_log2);
  const long long need = (N + rows_per_block - 1) / rows_per_block;
  // warps numbered across the grid: the same number of blocks on every SM (as the 2-bit
  // GEMV's shared-memory path)
  const int grid = static_cast<int>(
      need > num_sms() ? 1ll * blocks_per_sm * num_sms()
                       : std::min<long long>(num_sms(), (N + (32 >> lpr_log2) - 1) / (32 >> lpr_log2)));
  kern<<<grid, bl::kGemv3Threads, smem, s>>>(x, packed3, gamma, y, N, K, lpr_log2);
  return launch_status();
}

template <int XM, int OM>
bl_status launch_gemv3_m(const void* x, const uint8_t* packed3, const float* gamma, void* y,
                         int M, int N, int K, cudaStream_t s) {
  switch (M) {
    case 1: return launch_gemv3_t<1, XM, OM>(x, packed3, gamma, y, N, K, s);
    case 2: return launch_gemv3_t<2, XM, OM>(x, packed3, gamma, y, N, K, s);
    case 3: return launch_gemv3_t<3, XM, OM>(x, packed3, gamma, y, N, K, s);
    case 4: return launch_gemv3_t<4, XM, OM>(x, packed3, gamma, y, N, K, s);
    default: return BL_ERR_UNSUPPORTED_SHAPE;
  }
}

// ------------------------------------------------------------------ GEMM launch
// The prefill GEMM (M > 256 tokens): the weights as the TMEM A operand, the tokens by TMA.
template <int OM>
bl_status launch_gemm_t(const int8_t* xq, const uint8_t* packed, const int* rowsum,
                        const float* scale, const float* gamma, void* y, int M, int N, int K,
                        cudaStream_t s, const ChainOpts& o) {
  const int bnt = bl::pf::token_tile(M);
  CUtensorMap map_x, map_w;
  if (!make_map_u8(&map_x, xq, K, M, K, bl::pf::BK, bnt, true)) return BL_ERR_CUDA;
  if (!make_map_u8(&map_w, packed, K / 4, N, K / 4, bl::pf::BK / 4, bl::pf::BW, false))
    return BL_ERR_CUDA;
  auto kern = bl::gemm_prefill_kernel<OM>;
  static bl::PerDevice configured;
  if (!set_smem_limit_once(configured, kern, bl::pf::SMEM_BYTES)) return BL_ERR_CUDA;
  const long long tiles = static_cast<long long>((M + bnt - 1) / bnt) *
                          ((N + bl::pf::BW - 1) / bl::pf::BW);
  const int grid = static_cast<int>(std::min<long long>(tiles, num_sms()));
  return launch_ex(kern, dim3(grid), dim3(bl::pf::THREADS), bl::pf::SMEM_BYTES, s, o.pdl,
                   map_x, map_w, rowsum, scale, gamma, y, M, N, K, bnt, kWaitLimitNs,
                   o.amax_out);
}

bl_status launch_gemm(const int8_t* xq, const uint8_t* packed, const int* rowsum,
                      const float* scale, const float* gamma, void* y, int y_dtype, int M, int N,
                      int K, cudaStream_t s, const ChainOpts& o = {}) {
  switch (y_dtype) {
    case BL_F32: return launch_gemm_t<0>(xq, packed, rowsum, scale, gamma, y, M, N, K, s, o);
    case BL_BF16: return launch_gemm_t<1>(xq, packed, rowsum, scale, gamma, y, M, N, K, s, o);
    case BL_I32: return launch_gemm_t<2>(xq, packed, rowsum, scale, gamma, y, M, N, K, s, o);
    default: return BL_ERR_INVALID_ARG;
  }
}

template <int OM>
bl_status launch_skinny_t(const int8_t* xq, const uint8_t* packed, const int* rowsum,
                          const float* scale, const float* gamma, void* y, int M, int N, int K,
                          const SkinnyPlan& p, const SkinnyWs& w, cudaStream_t s,
                          float* amax_out) {
  CUtensorMap map_x, map_w;
  if (!make_map_u8(&map_x, xq, K, M, K, bl::sk::BK, p.bnt, true)) return BL_ERR_CUDA;
  if (!make_map_u8(&map_w, packed, K / 4, N, K / 4, bl::sk::BK * bl::sk::KPS / 4, bl::sk::BW,
                   true))
    return BL_ERR_CUDA;
  auto kern = bl::gemm_skinny_kernel<OM>;
  static bl::PerDevice configured;
  int most = 0;
  for (int b = 16; b <= bl::sk::BW * 2; b += 16) most = std::max(most, bl::sk::smem_bytes(b));
  if (!set_smem_limit_once(configured, kern, most)) return BL_ERR_CUDA;
  // Programmatic dependent launch: the kernel may start while the quantization kernel before
  // it (which also zeroed the split-K sums and counters) is still running; it loads W and
  // sets up TMEM meanwhile and waits for that grid before touching its outputs.
  return launch_ex(kern, dim3(static_cast<unsigned>(p.tiles * p.splits)),
                   dim3(bl::sk::THREADS), static_cast<size_t>(bl::sk::smem_bytes(p.bnt)), s,
                   true, map_x, map_w, rowsum, scale, gamma, y, w.partial, w.counters, M, N, K,
                   p.bnt, p.splits, p.kbps, kWaitLimitNs, amax_out);
}

// The part of the workspace the skinny kernel needs zeroed (split-K sums and counters; a
// multiple of 256 bytes), empty when K is not split. The kernel launched just before the
// skinny one clears it.
void skinny_zero_region(void* ws, int M, int N, int K, uint4** z, long long* n16) {
  const SkinnyPlan p = skinny_plan(M, N, K);
  const SkinnyWs w = skinny_ws_layout(ws, M, N, K, p);
  const size_t head = fwd_ws_layout(nullptr, M, K).bytes;
  *z = (p.splits > 1) ? reinterpret_cast<uint4*>(w.partial) : nullptr;
  *n16 = (p.splits > 1) ? static_cast<long long>((w.bytes - head) / 16) : 0;
}

bl_status launch_skinny_plan(const int8_t* xq, const uint8_t* packed, const int* rowsum,
                             const float* scale, const float* gamma, void* y, int y_dtype,
                             int M, int N, int K, const SkinnyPlan& p, const SkinnyWs& w,
                             cudaStream_t s, float* amax_out = nullptr) {
  switch (y_dtype) {
    case BL_F32:
      return launch_skinny_t<0>(xq, packed, rowsum, scale, gamma, y, M, N, K, p, w, s, amax_out);
    case BL_BF16:
      return launch_skinny_t<1>(xq, packed, rowsum, scale, gamma, y, M, N, K, p, w, s, amax_out);
    case BL_I32:
      return launch_skinny_t<2>(xq, packed, rowsum, scale, gamma, y, M, N, K, p, w, s, amax_out);
    default: return BL_ERR_INVALID_ARG;
  }
}

bl_status launch_skinny(const int8_t* xq, const uint8_t* packed, const int* rowsum,
                        const float* scale, const float* gamma, void* y, int y_dtype, int M,
                        int N, int K, void* ws, cudaStream_t s) {
  const SkinnyPlan p = skinny_plan(M, N, K);
  const SkinnyWs w = skinny_ws_layout(ws, M, N, K, p);
  return launch_skinny_plan(xq, packed, rowsum, scale, gamma, y, y_dtype, M, N, K, p, w, s);
}

// The skinny plan with K left unsplit: one CTA per weight tile, so the kernel needs no
// split-K sums or counters (only the staged activations).
SkinnyPlan skinny_plan_unsplit(int M, int N, int K) {
  SkinnyPlan p = skinny_plan(M, N, K);
  const int KB = (K + bl::sk::BK - 1) / bl::sk::BK;
  p.splits = 1;
  p.kbps = (KB + bl::sk::KPS - 1) / bl::sk::KPS * bl::sk::KPS;
  return p;
}

// Workspace bytes the forward / contract paths need for (M, N, K).
size_t fwd_ws_bytes(int M, int N, int K) {
  if (use_gemv(M, N, K)) return 0;
  if (M <= kSkinnyMaxM) return skinny_ws_layout(nullptr, M, N, K, skinny_plan(M, N, K)).bytes;
  return fwd_ws_layout(nullptr, M, K).bytes;
}

bl_status launch_act_quant(const void* x, int x_dtype, int M, int K, int8_t* xq, float* scale,
                           int* rowsum, cudaStream_t s, uint4* zero = nullptr,
                           long long zero_n16 = 0) {
  if (x_dtype == BL_BF16)
    bl::act_quant_kernel<true><<<M, bl::kAqThreads, 0, s>>>(x, K, xq, scale, rowsum, zero,
                                                            zero_n16);
  else
    bl::act_quant_kernel<false><<<M, bl::kAqThreads, 0, s>>>(x, K, xq, scale, rowsum, zero,
                                                             zero_n16);
  return launch_status();
}

// The activation quantization inside a chain: absmax given (from the kernel that wrote x)
// or not (the chain's input), launched with programmatic dependent launch.
bl_status launch_act_quant_chain(const void* x, int x_dtype, int M, int K, int8_t* xq,
                                 float* scale, int* rowsum, cudaStream_t s,
                                 const float* amax_in) {
  float* a = const_cast<float*>(amax_in);
  if (x_dtype == BL_BF16)
    return amax_in ? launch_ex(bl::act_quant_kernel<true, bl::kAqGiven>, dim3(M),
                               dim3(bl::kAqThreads), 0, s, true, x, K, xq, scale, rowsum,
                               static_cast<uint4*>(nullptr), 0ll, a)
                   : launch_ex(bl::act_quant_kernel<true, bl::kAqRow>, dim3(M),
                               dim3(bl::kAqThreads), 0, s, true, x, K, xq, scale, rowsum,
                               static_cast<uint4*>(nullptr), 0ll, a);
  return amax_in ? launch_ex(bl::act_quant_kernel<false, bl::kAqGiven>, dim3(M),
                             dim3(bl::kAqThreads), 0, s, true, x, K, xq, scale, rowsum,
                             static_cast<uint4*>(nullptr), 0ll, a)
                 : launch_ex(bl::act_quant_kernel<false, bl::kAqRow>, dim3(M),
                             dim3(bl::kAqThreads), 0, s, true, x, K, xq, scale, rowsum,
                             static_cast<uint4*>(nullptr), 0ll, a);
}

// ------------------------------------------------------------------ weight quantization
// Workspace of bitlinear_quantize_weights: the exact-sum columns and the barrier counters.
// Workspace of bitlinear_quantize_weights: the exact-sum columns and barrier counters, and
// for matrices of at least kWqSingleMin weights the band lists of the single-read mode.
constexpr long long kWqSingleMin = 4ll << 20;
size_t wq_ws_head() { return align_up(sizeof(WqWorkspace), 256); }
size_t wq_list_bytes() {
  return static_cast<size_t>(bl::kWqMaxBlocks) * bl::kWqListCap * sizeof(uint2);
}
size_t wq_ws_bytes(long long n) {
  return wq_ws_head() + (n >= kWqSingleMin ? wq_list_bytes() : 0);
}

template <bool kBf16, int MODE>
bl_status launch_weight_quant_t(const void* W, long long n, long long n_total, float eps,
                                void* ws, size_t ws_bytes, unsigned long long* sums,
                                float* gamma, uint32_t* packed, cudaStream_t s) {
  auto kern = bl::weight_quant_kernel<kBf16, MODE>;
  constexpr int kSmem = bl::kWqStages * bl::kWqStageBytes;
  // blocks of this kernel resident per SM, found once per device after raising its
  // shared-memory limit (a cooperative launch needs every block resident)
  static bl::PerDevice occupancy;
  const int blocks_per_sm = occupancy.get(current_device(), [&](int) {
    int b = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, bl::kWqThreads, kSmem) !=
            cudaSuccess)
      return 0;
    return b;
  });
  if (blocks_per_sm < 1) return BL_ERR_CUDA;
  // one block per 32 KB of weights at least, at most all resident blocks
  const long long want = (n * (kBf16 ? 2 : 4) + 32767) / 32768;
  const int grid = static_cast<int>(
      std::max<long long>(1, std::min<long long>(want, 1ll * blocks_per_sm * num_sms())));
  WqWorkspace* hdr = static_cast<WqWorkspace*>(ws);
  if (MODE != bl::kWqFinish &&
      cudaMemsetAsync(hdr, 0, sizeof(WqWorkspace), s) != cudaSuccess)
    return BL_ERR_CUDA;
  unsigned long long limit = kWaitLimitNs;
  // Single-read mode when a block's range does not fit its ring (the two-pass mode would
  // stream it twice) and the workspace holds the band lists.
  const long long words = n / 16;
  const long long range_bytes = (words + grid - 1) / grid * (kBf16 ? 32 : 64);
  uint2* list = nullptr;
  if (MODE == bl::kWqFull && range_bytes > 1ll * bl::kWqStages * bl::kWqStageBytes &&
      grid <= bl::kWqMaxBlocks && ws_bytes >= wq_ws_head() + wq_list_bytes())
    list = reinterpret_cast<uint2*>(static_cast<char*>(ws) + wq_ws_head());
  void* args[] = {const_cast<void**>(&W), &n, &n_total, &eps, &hdr, &sums, &gamma, &packed,
                  &limit, &list};
  if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid),
                                  dim3(bl::kWqThreads), args, kSmem, s) != cudaSuccess)
    return BL_ERR_CUDA;
  return launch_status();
}

template <int MODE>
bl_status launch_weight_quant(const void* W, bool bf16, long long n, long long n_total,
                              float eps, void* ws, size_t ws_bytes, unsigned long long* sums,
                              float* gamma, uint32_t* packed, cudaStream_t s) {
  return bf16 ? launch_weight_quant_t<true, MODE>(W, n, n_total, eps, ws, ws_bytes, sums, gamma,
                                                  packed, s)
              : launch_weight_quant_t<false, MODE>(W, n, n_total, eps, ws, ws_bytes, sums, gamma,
                                                   packed, s);
}

// ------------------------------------------------------------------ debug probe
__global__ void timeout_probe_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    bl::mbar_init(&bar, 1);
    bl::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) bl::mbar_wait(&bar, 0u, limit_ns);  // nothing ever arrives
}

}  // namespace

// ------------------------------------------------------------------ no-allocation forward
// Scratch for bitlinear_forward_noalloc: the int8 activations, per-token scales and
// row sums that the tensor-core path stages between its two kernels. It is a file-scope
// device array, so every GPU that loads this library holds these 16 MiB until the
// process exits, and every call of bitlinear_forward_noalloc on a device shares it.
static constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device. In host code the array's
// name is only a host-side stand-in, so the address is looked up once per device with
// cudaGetSymbolAddress (with that device current) and cached.
bl_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BL_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return BL_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return BL_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return BL_OK;
}

}  // namespace

extern "C" {

size_t bitlinear_workspace_size(int M, int N, int K) {
  if (!shape_ok(M, N, K)) return 0;
  const size_t need = std::max(wq_ws_bytes(static_cast<long long>(N) * K), fwd_ws_bytes(M, N, K));
  return align_up(need, 256);
}

bl_status bitlinear_quantize_weights(const void* W, int w_dtype, int N, int K, float eps,
                                     uint8_t* packed, float* gamma, void* ws, size_t ws_bytes,
                                     void* stream) {
  if (!W || !packed || !gamma || !ws) return BL_ERR_INVALID_ARG;
  if (w_dtype != BL_F32 && w_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return BL_ERR_INVALID_ARG;
  if (!shape_ok(1, N, K)) return BL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(gamma) || !aligned16(ws))
    return BL_ERR_MISALIGNED;
  if (ws_bytes < sizeof(WqWorkspace)) return BL_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long n = static_cast<long long>(N) * K;
  return launch_weight_quant<bl::kWqFull>(W, w_dtype == BL_BF16, n, n, eps, ws, ws_bytes, nullptr, gamma,
                                          reinterpret_cast<uint32_t*>(packed), s);
}

bl_status bitlinear_weight_abssum(const void* W, int w_dtype, int N, int K, uint64_t* sums,
                                  void* ws, size_t ws_bytes, void* stream) {
  if (!W || !sums || !ws) return BL_ERR_INVALID_ARG;
  if (w_dtype != BL_F32 && w_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (!shape_ok(1, N, K)) return BL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(W) || !aligned16(sums) || !aligned16(ws)) return BL_ERR_MISALIGNED;
  if (ws_bytes < sizeof(WqWorkspace)) return BL_ERR_WORKSPACE;
  const long long n = static_cast<long long>(N) * K;
  return launch_weight_quant<bl::kWqPartial>(
      W, w_dtype == BL_BF16, n, n, 0.0f, ws, ws_bytes, reinterpret_cast<unsigned long long*>(sums),
      nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

bl_status bitlinear_quantize_weights_from_abssum(const void* W, int w_dtype, int N, int K,
                                                 long long n_total, const uint64_t* sums,
                                                 float eps, uint8_t* packed, float* gamma,
                                                 void* stream) {
  if (!W || !sums || !packed || !gamma) return BL_ERR_INVALID_ARG;
  if (w_dtype != BL_F32 && w_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return BL_ERR_INVALID_ARG;
  if (!shape_ok(1, N, K)) return BL_ERR_UNSUPPORTED_SHAPE;
  if (n_total < static_cast<long long>(N) * K) return BL_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(sums) || !aligned16(packed) || !aligned16(gamma))
    return BL_ERR_MISALIGNED;
  return launch_weight_quant<bl::kWqFinish>(
      W, w_dtype == BL_BF16, static_cast<long long>(N) * K, n_total, eps, nullptr, 0,
      const_cast<unsigned long long*>(reinterpret_cast<const unsigned long long*>(sums)), gamma,
      reinterpret_cast<uint32_t*>(packed), static_cast<cudaStream_t>(stream));
}

bl_status bitlinear_quantize_acts(const void* x, int x_dtype, int M, int K, int8_t* xq,
                                  float* scale, void* stream) {
  if (!x || !xq || !scale) return BL_ERR_INVALID_ARG;
  if (x_dtype != BL_F32 && x_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (!shape_ok(M, 1, K)) return BL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || !aligned16(xq) || !aligned16(scale)) return BL_ERR_MISALIGNED;
  return launch_act_quant(x, x_dtype, M, K, xq, scale, nullptr, static_cast<cudaStream_t>(stream));
}

bl_status bitlinear_act_absmax(const void* x, int x_dtype, int M, int K, float* amax,
                               void* stream) {
  if (!x || !amax) return BL_ERR_INVALID_ARG;
  if (x_dtype != BL_F32 && x_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (!shape_ok(M, 1, K)) return BL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || !aligned16(amax)) return BL_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (x_dtype == BL_BF16)
    bl::act_quant_kernel<true, bl::kAqAbsmax><<<M, bl::kAqThreads, 0, s>>>(
        x, K, nullptr, nullptr, nullptr, nullptr, 0, amax);
  else
    bl::act_quant_kernel<false, bl::kAqAbsmax><<<M, bl::kAqThreads, 0, s>>>(
        x, K, nullptr, nullptr, nullptr, nullptr, 0, amax);
  return launch_status();
}

bl_status bitlinear_quantize_acts_absmax(const void* x, int x_dtype, int M, int K,
                                         const float* amax, int8_t* xq, float* scale,
                                         void* stream) {
  if (!x || !amax || !xq || !scale) return BL_ERR_INVALID_ARG;
  if (x_dtype != BL_F32 && x_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (!shape_ok(M, 1, K)) return BL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || !aligned16(amax) || !aligned16(xq) || !aligned16(scale))
    return BL_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* a = const_cast<float*>(amax);
  if (x_dtype == BL_BF16)
    bl::act_quant_kernel<true, bl::kAqGiven><<<M, bl::kAqThreads, 0, s>>>(
        x, K, xq, scale, nullptr, nullptr, 0, a);
  else
    bl::act_quant_kernel<false, bl::kAqGiven><<<M, bl::kAqThreads, 0, s>>>(
        x, K, xq, scale, nullptr, nullptr, 0, a);
  return launch_status();
}

bl_status bitlinear_rescale(const int32_t* acc, const float* scale, const float* gamma,
                            void* y, int y_dtype, int M, int N, void* stream) {
  if (!acc || !scale || !gamma || !y) return BL_ERR_INVALID_ARG;
  if (y_dtype != BL_F32 && y_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || static_cast<long long>(M) * N >= (1ll << 31))
    return BL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(acc) || !aligned16(scale) || !aligned16(gamma) || !aligned16(y))
    return BL_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long work = static_cast<long long>(M) * N / ((N % 4 == 0) ? 4 : 1);
  const int grid = static_cast<int>(std::max<long long>(
      1, std::min<long long>((work + bl::kRsThreads - 1) / bl::kRsThreads, 8ll * num_sms())));
  if (N % 4 == 0) {
    if (y_dtype == BL_F32) bl::rescale_kernel<0><<<grid, bl::kRsThreads, 0, s>>>(acc, scale, gamma, y, M, N);
    else bl::rescale_kernel<1><<<grid, bl::kRsThreads, 0, s>>>(acc, scale, gamma, y, M, N);
  } else {
    if (y_dtype == BL_F32)
      bl::rescale_scalar_kernel<0><<<grid, bl::kRsThreads, 0, s>>>(acc, scale, gamma, y, M, N);
    else
      bl::rescale_scalar_kernel<1><<<grid, bl::kRsThreads, 0, s>>>(acc, scale, gamma, y, M, N);
  }
  return launch_status();
}

bl_status bitlinear_forward(const void* x, int x_dtype, const uint8_t* packed,
                            const float* gamma, void* y, int y_dtype, int M, int N, int K,
                            void* ws, size_t ws_bytes, void* stream) {
  if (!x || !packed || !gamma || !y) return BL_ERR_INVALID_ARG;
  if (x_dtype != BL_F32 && x_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (y_dtype != BL_F32 && y_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (!shape_ok(M, N, K)) return BL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(gamma) || !aligned16(y))
    return BL_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_gemv(M, N, K)) {
    if (x_dtype == BL_BF16)
      return launch_gemv_x<bl::kXbf16>(x, packed, gamma, y, y_dtype, M, N, K, s);
    return launch_gemv_x<bl::kXf32>(x, packed, gamma, y, y_dtype, M, N, K, s);
  }
  if (!ws) return BL_ERR_WORKSPACE;
  if (!aligned16(ws)) return BL_ERR_MISALIGNED;
  if (ws_bytes < fwd_ws_bytes(M, N, K)) return BL_ERR_WORKSPACE;
  FwdWs w = fwd_ws_layout(ws, M, K);
  uint4* zero = nullptr;
  long long zero_n16 = 0;
  if (M <= kSkinnyMaxM) skinny_zero_region(ws, M, N, K, &zero, &zero_n16);
  bl_status st = launch_act_quant(x, x_dtype, M, K, w.xq, w.scale, w.rowsum, s, zero, zero_n16);
  if (st != BL_OK) return st;
  if (M <= kSkinnyMaxM)
    return launch_skinny(w.xq, packed, w.rowsum, w.scale, gamma, y, y_dtype, M, N, K, ws, s);
  return launch_gemm(w.xq, packed, w.rowsum, w.scale, gamma, y, y_dtype, M, N, K, s);
}

}  // extern "C"

namespace {

// ------------------------------------------------------------------ backward (STE)
// D[r][c] = alpha * sum_j A[r][j] B[c][j]; A bf16 [R][J]; B bf16 [C][J] or packed trits
// [C][J/4].
template <bool kPacked>
bl_status launch_gemm_bf16(const void* A, const void* B, const float* alpha, float* out, int R,
                           int C, int J, cudaStream_t s) {
  CUtensorMap map_a, map_b;
  if (!make_map_bf16(&map_a, A, J, R, bl::bf::BM)) return BL_ERR_CUDA;
  if (kPacked) {
    if (!make_map_u8(&map_b, B, J / 4, C, J / 4, bl::bf::BKE / 4, bl::bf::BN, false))
      return BL_ERR_CUDA;
  } else if (!make_map_bf16(&map_b, B, J, C, bl::bf::BN)) {
    return BL_ERR_CUDA;
  }
  auto kern = bl::gemm_bf16_kernel<kPacked>;
  constexpr int kSmem = bl::bf::smem_bytes<kPacked>();
  static bl::PerDevice configured;
  if (!set_smem_limit_once(configured, kern, kSmem)) return BL_ERR_CUDA;
  const long long tiles = static_cast<long long>((R + bl::bf::BM - 1) / bl::bf::BM) *
                          ((C + bl::bf::BN - 1) / bl::bf::BN);
  const int grid = static_cast<int>(std::min<long long>(tiles, num_sms()));
  return launch_ex(kern, dim3(grid), dim3(bl::bf::THREADS), kSmem, s, false, map_a, map_b,
                   alpha, out, R, C, J, kWaitLimitNs);
}

// Workspace of bitlinear_backward: [xq M*K][scale M][rowsum M][G^T N*Mp bf16][X~^T K*Mp bf16].
struct BwdWs {
  FwdWs f;
  __nv_bfloat16* gT;
  __nv_bfloat16* xT;
  int Mp;
  size_t bytes;
};
BwdWs bwd_ws_layout(void* base, int M, int N, int K) {
  BwdWs w{};
  w.f = fwd_ws_layout(base, M, K);
  w.Mp = (M + 7) / 8 * 8;
  char* p = static_cast<char*>(base) + w.f.bytes;
  const size_t g = align_up(static_cast<size_t>(N) * w.Mp * 2, 256);
  const size_t x = align_up(static_cast<size_t>(K) * w.Mp * 2, 256);
  w.gT = reinterpret_cast<__nv_bfloat16*>(p);
  w.xT = reinterpret_cast<__nv_bfloat16*>(p + g);
  w.bytes = w.f.bytes + g + x;
  return w;
}

int grid_for(long long work, int per_block) {
  return static_cast<int>(std::max<long long>(
      1, std::min<long long>((work + per_block - 1) / per_block, 16ll * num_sms())));
}

}  // namespace

extern "C" {

bl_status bitlinear_pack_transpose(const uint8_t* packed, int N, int K, uint8_t* packedT,
                                   void* stream) {
  if (!packed || !packedT) return BL_ERR_INVALID_ARG;
  if (!shape_ok(1, N, K) || N % 64 != 0) return BL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(packed) || !aligned16(packedT)) return BL_ERR_MISALIGNED;
  bl::pack_transpose_kernel<<<grid_for(static_cast<long long>(N / 64) * (K / 64), 1), 256, 0,
                              static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint32_t*>(packed), reinterpret_cast<uint32_t*>(packedT), N, K);
  return launch_status();
}

size_t bitlinear_backward_workspace_size(int M, int N, int K) {
  if (!shape_ok(M, N, K) || N % 64 != 0) return 0;
  return align_up(bwd_ws_layout(nullptr, M, N, K).bytes, 256);
}

bl_status bitlinear_backward(const void* x, int x_dtype, const void* grad_y,
                             const uint8_t* packedT, const float* gamma, float* grad_x,
                             float* grad_w, int M, int N, int K, void* ws, size_t ws_bytes,
                             void* stream) {
  if (!grad_y || (!grad_x && !grad_w)) return BL_ERR_INVALID_ARG;
  if (grad_x && (!packedT || !gamma)) return BL_ERR_INVALID_ARG;
  if (grad_w && (!x || !ws)) return BL_ERR_INVALID_ARG;
  if (x_dtype != BL_F32 && x_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (!shape_ok(M, N, K) || N % 64 != 0) return BL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(grad_y) || (x && !aligned16(x)) || (packedT && !aligned16(packedT)) ||
      (gamma && !aligned16(gamma)) || (grad_x && !aligned16(grad_x)) ||
      (grad_w && !aligned16(grad_w)) || (ws && !aligned16(ws)))
    return BL_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (grad_w) {
    const BwdWs w = bwd_ws_layout(ws, M, N, K);
    if (ws_bytes < w.bytes) return BL_ERR_WORKSPACE;
    bl_status st = launch_act_quant(x, x_dtype, M, K, w.f.xq, w.f.scale, nullptr, s);
    if (st != BL_OK) return st;
    const int tiles_g = ((w.Mp + 63) / 64) * (N / 64);
    bl::transpose_bf16_kernel<0><<<grid_for(tiles_g, 1), 256, 0, s>>>(grad_y, nullptr, w.gT, M,
                                                                       N, w.Mp);
    const int tiles_x = ((w.Mp + 63) / 64) * (K / 64);
    bl::transpose_bf16_kernel<1><<<grid_for(tiles_x, 1), 256, 0, s>>>(w.f.xq, w.f.scale, w.xT,
                                                                       M, K, w.Mp);
    if (launch_status() != BL_OK) return BL_ERR_CUDA;
    st = launch_gemm_bf16<false>(w.gT, w.xT, nullptr, grad_w, N, K, w.Mp, s);
    if (st != BL_OK) return st;
  }
  if (grad_x) return launch_gemm_bf16<true>(grad_y, packedT, gamma, grad_x, M, K, N, s);
  return BL_OK;
}

}  // extern "C"

namespace {

// Workspace plan of a layer chain (see bitlinear_chain_forward). Activation buffer j = 0 is
// the chain input x, j = l + 1 the output of layer l.
struct ChainPlan {
  int L = 0, M = 0, K0 = 0;
  size_t bytes = 0;
  // offsets into the workspace (bytes)
  size_t amax_off = 0;      // (L + 1) x M floats: absmax of every activation buffer
  size_t partial_off = 0;   // shared int32 split-K sums (self-cleaning), then counters
  size_t zero_bytes = 0;    // bytes from amax_off cleared once per call
  size_t counters_off = 0;
  std::vector<size_t> act_off;   // per layer: its output in the workspace (or SIZE_MAX)
  std::vector<size_t> xq_off;    // per buffer j: int8 codes + scale + rowsum (or SIZE_MAX)
  std::vector<char> consumed;    // per buffer j: read by a later layer
};

constexpr size_t kNone = static_cast<size_t>(-1);

bl_status chain_plan(int M, const bl_layer* layers, int L, ChainPlan* plan) {
  if (!layers || L < 1 || L > 4096 || M < 1) return BL_ERR_INVALID_ARG;
  ChainPlan p;
  p.L = L;
  p.M = M;
  p.consumed.assign(L + 1, 0);
  p.act_off.assign(L, kNone);
  p.xq_off.assign(L + 1, kNone);
  int K0 = -1;
  for (int l = 0; l < L; ++l) {
    const bl_layer& ly = layers[l];
    if (!ly.packed || !ly.gamma) return BL_ERR_INVALID_ARG;
    if (ly.src < -1 || ly.src >= l) return BL_ERR_INVALID_ARG;
    if (!shape_ok(M, ly.N, ly.K)) return BL_ERR_UNSUPPORTED_SHAPE;
    if (ly.src == -1) {
      if (K0 >= 0 && K0 != ly.K) return BL_ERR_UNSUPPORTED_SHAPE;
      K0 = ly.K;
    } else if (layers[ly.src].N != ly.K) {
      return BL_ERR_UNSUPPORTED_SHAPE;
    }
    if (!aligned16(ly.packed) || !aligned16(ly.gamma) || (ly.out && !aligned16(ly.out)))
      return BL_ERR_MISALIGNED;
    p.consumed[ly.src + 1] = 1;
  }
  if (K0 < 0) return BL_ERR_INVALID_ARG;  // nothing reads x
  p.K0 = K0;
  size_t off = 0;
  p.amax_off = off;
  off += align_up(static_cast<size_t>(L + 1) * M * 4, 256);
  size_t part = 0, tiles = 0;
  for (int l = 0; l < L; ++l) {
    const bl_layer& ly = layers[l];
    if (!use_gemv(M, ly.N, ly.K) && M <= kSkinnyMaxM) {
      const SkinnyPlan sp = skinny_plan_chain(M, ly.N, ly.K);
      if (sp.splits > 1) part = std::max(part, static_cast<size_t>(M) * ly.N * 4);
      tiles = std::max(tiles, static_cast<size_t>(sp.tiles));
    }
  }
  p.partial_off = off;
  off += align_up(part, 256);
  p.counters_off = off;
  off += align_up(tiles * 4, 256);
  p.zero_bytes = off - p.amax_off;
  for (int l = 0; l < L; ++l) {
    const bl_layer& ly = layers[l];
    const bool last = (l == L - 1);
    if (!last && ly.out == nullptr) {
      p.act_off[l] = off;
      off += align_up(static_cast<size_t>(M) * ly.N * 2, 256);
    }
    const int j = ly.src + 1;
    if (!use_gemv(M, ly.N, ly.K) && p.xq_off[j] == kNone) {
      p.xq_off[j] = off;
      off += fwd_ws_layout(nullptr, M, ly.K).bytes;
    }
  }
  p.bytes = align_up(std::max<size_t>(off, 256), 256);
  *plan = std::move(p);
  return BL_OK;
}

}  // namespace

extern "C" {

size_t bitlinear_chain_workspace_size(int M, const bl_layer* layers, int L) {
  ChainPlan p;
  if (chain_plan(M, layers, L, &p) != BL_OK) return 0;
  return p.bytes;
}

bl_status bitlinear_chain_forward(const void* x, int x_dtype, int M, const bl_layer* layers,
                                  int L, void* y, int y_dtype, void* ws, size_t ws_bytes,
                                  void* stream) {
  if (!x || !y || !ws) return BL_ERR_INVALID_ARG;
  if (x_dtype != BL_F32 && x_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (y_dtype != BL_F32 && y_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  ChainPlan p;
  bl_status st = chain_plan(M, layers, L, &p);
  if (st != BL_OK) return st;
  if (!aligned16(x) || !aligned16(y) || !aligned16(ws)) return BL_ERR_MISALIGNED;
  if (ws_bytes < p.bytes) return BL_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(ws);
  float* amax = reinterpret_cast<float*>(base + p.amax_off);
  if (cudaMemsetAsync(base + p.amax_off, 0, p.zero_bytes, s) != cudaSuccess) return BL_ERR_CUDA;
  std::vector<char> quantized(L + 1, 0);
  for (int l = 0; l < L; ++l) {
    const bl_layer& ly = layers[l];
    const int j = ly.src + 1;  // input buffer
    const void* in = (j == 0) ? x : (layers[ly.src].out ? layers[ly.src].out
                                                          : base + p.act_off[ly.src]);
    const int in_dtype = (j == 0) ? x_dtype : BL_BF16;
    const float* amax_in = (j == 0) ? nullptr : amax + static_cast<size_t>(j) * M;
    const bool last = (l == L - 1);
    void* out = last ? y : (ly.out ? ly.out : base + p.act_off[l]);
    const int out_dtype = last ? y_dtype : BL_BF16;
    float* amax_out = (!last && p.consumed[l + 1]) ? amax + static_cast<size_t>(l + 1) * M : nullptr;
    if (use_gemv(M, ly.N, ly.K)) {
      ChainOpts o;
      o.amax_in = amax_in;
      o.amax_out = amax_out;
      o.pdl = true;
      st = (in_dtype == BL_BF16)
               ? launch_gemv_x<bl::kXbf16>(in, ly.packed, ly.gamma, out, out_dtype, M, ly.N, ly.K, s, o)
               : launch_gemv_x<bl::kXf32>(in, ly.packed, ly.gamma, out, out_dtype, M, ly.N, ly.K, s, o);
      if (st != BL_OK) return st;
      continue;
    }
    FwdWs w = fwd_ws_layout(base + p.xq_off[j], M, ly.K);
    if (!quantized[j]) {  // once per input buffer, whatever number of layers read it
      st = launch_act_quant_chain(in, in_dtype, M, ly.K, w.xq, w.scale, w.rowsum, s, amax_in);
      if (st != BL_OK) return st;
      quantized[j] = 1;
    }
    if (M <= kSkinnyMaxM) {
      const SkinnyPlan sp = skinny_plan_chain(M, ly.N, ly.K);
      SkinnyWs sw{};
      sw.partial = reinterpret_cast<int*>(base + p.partial_off);
      sw.counters = reinterpret_cast<unsigned int*>(base + p.counters_off);
      st = launch_skinny_plan(w.xq, ly.packed, w.rowsum, w.scale, ly.gamma, out, out_dtype, M,
                              ly.N, ly.K, sp, sw, s, amax_out);
    } else {
      ChainOpts o;
      o.amax_out = amax_out;
      o.pdl = true;
      st = launch_gemm(w.xq, ly.packed, w.rowsum, w.scale, ly.gamma, out, out_dtype, M, ly.N,
                       ly.K, s, o);
    }
    if (st != BL_OK) return st;
  }
  return BL_OK;
}

bl_status bitlinear_contract_i32(const int8_t* xq, const uint8_t* packed, int32_t* acc, int M,
                                 int N, int K, void* ws, size_t ws_bytes, void* stream) {
  if (!xq || !packed || !acc) return BL_ERR_INVALID_ARG;
  if (!shape_ok(M, N, K)) return BL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(xq) || !aligned16(packed) || !aligned16(acc)) return BL_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_gemv(M, N, K)) return launch_gemv_x<bl::kXi8>(xq, packed, nullptr, acc, BL_I32, M, N, K, s);
  if (!ws) return BL_ERR_WORKSPACE;
  if (!aligned16(ws)) return BL_ERR_MISALIGNED;
  if (ws_bytes < fwd_ws_bytes(M, N, K)) return BL_ERR_WORKSPACE;
  FwdWs w = fwd_ws_layout(ws, M, K);
  uint4* zero = nullptr;
  long long zero_n16 = 0;
  if (M <= kSkinnyMaxM) skinny_zero_region(ws, M, N, K, &zero, &zero_n16);
  bl::rowsum_i8_kernel<<<M, bl::kAqThreads, 0, s>>>(xq, K, w.rowsum, zero, zero_n16);
  if (launch_status() != BL_OK) return BL_ERR_CUDA;
  if (M <= kSkinnyMaxM)
    return launch_skinny(xq, packed, w.rowsum, nullptr, nullptr, acc, BL_I32, M, N, K, ws, s);
  return launch_gemm(xq, packed, w.rowsum, nullptr, nullptr, acc, BL_I32, M, N, K, s);
}

size_t bitlinear_base3_row_bytes(int K) {
  if (K < 64 || K % 64 != 0) return 0;
  return static_cast<size_t>((K + 79) / 80) * 16;
}

bl_status bitlinear_pack_base3(const uint8_t* packed, int N, int K, uint8_t* packed3,
                               void* stream) {
  if (!packed || !packed3) return BL_ERR_INVALID_ARG;
  if (!shape_ok(1, N, K)) return BL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(packed) || !aligned16(packed3)) return BL_ERR_MISALIGNED;
  const long long chunks = static_cast<long long>(N) * ((K + 79) / 80);
  const int grid = static_cast<int>(
      std::max<long long>(1, std::min<long long>((chunks + 255) / 256, 16ll * num_sms())));
  bl::pack_base3_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint32_t*>(packed), reinterpret_cast<uint4*>(packed3), N, K);
  return launch_status();
}

bl_status bitlinear_forward_base3(const void* x, int x_dtype, const uint8_t* packed3,
                                  const float* gamma, void* y, int y_dtype, int M, int N, int K,
                                  void* stream) {
  if (!x || !packed3 || !gamma || !y) return BL_ERR_INVALID_ARG;
  if (x_dtype != BL_F32 && x_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (y_dtype != BL_F32 && y_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (!shape_ok(M, N, K) || M > kGemv3MaxM ||
      static_cast<long long>(M) * 80 * ((K + 79) / 80) > kGemvMaxSmem)
    return BL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || !aligned16(packed3) || !aligned16(gamma) || !aligned16(y))
    return BL_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (x_dtype == BL_BF16)
    return (y_dtype == BL_F32) ? launch_gemv3_m<bl::kXbf16, bl::kOf32>(x, packed3, gamma, y, M, N, K, s)
                               : launch_gemv3_m<bl::kXbf16, bl::kObf16>(x, packed3, gamma, y, M, N, K, s);
  return (y_dtype == BL_F32) ? launch_gemv3_m<bl::kXf32, bl::kOf32>(x, packed3, gamma, y, M, N, K, s)
                             : launch_gemv3_m<bl::kXf32, bl::kObf16>(x, packed3, gamma, y, M, N, K, s);
}

bl_status bitlinear_get_device_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return BL_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, bl::g_status, sizeof v) != cudaSuccess) return BL_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(bl::g_status, &zero, sizeof zero) != cudaSuccess) return BL_ERR_CUDA;
  if (v & bl::kStatusTimeout) return BL_ERR_TIMEOUT;
  if (v & bl::kStatusNonfinite) return BL_ERR_NONFINITE;
  return BL_OK;
}

// Same computation as bitlinear_forward, for callers that cannot allocate device memory:
// the staging buffers of the tensor-core paths live in g_noalloc_scratch instead of a
// caller-supplied workspace. Kernel choice: the GEMV where bitlinear_forward uses it, the
// skinny tensor-core kernel with K unsplit up to 256 tokens (bitlinear_forward may split K
// there, which needs int32 sums this scratch does not hold), the prefill GEMM above. Nothing in the scratch has to start at zero (each call
// writes every byte it later reads). No cudaMalloc, cudaFree or allocating library call
// is made. Calls that overlap on the GPU (other streams, other host threads) race on the
// shared scratch; callers serialize them.
bl_status bitlinear_forward_noalloc(const void* x, int x_dtype, const uint8_t* packed,
                                    const float* gamma, void* y, int y_dtype, int M, int N,
                                    int K, void* stream) {
  if (!x || !packed || !gamma || !y) return BL_ERR_INVALID_ARG;
  if (x_dtype != BL_F32 && x_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (y_dtype != BL_F32 && y_dtype != BL_BF16) return BL_ERR_INVALID_ARG;
  if (!shape_ok(M, N, K)) return BL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(gamma) || !aligned16(y))
    return BL_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_gemv(M, N, K)) {
    if (x_dtype == BL_BF16)
      return launch_gemv_x<bl::kXbf16>(x, packed, gamma, y, y_dtype, M, N, K, s);
    return launch_gemv_x<bl::kXf32>(x, packed, gamma, y, y_dtype, M, N, K, s);
  }
  if (fwd_ws_layout(nullptr, M, K).bytes > kNoAllocScratchBytes) return BL_ERR_WORKSPACE;
  void* scratch = nullptr;
  bl_status st = noalloc_scratch(&scratch);
  if (st != BL_OK) return st;
  FwdWs w = fwd_ws_layout(scratch, M, K);
  st = launch_act_quant(x, x_dtype, M, K, w.xq, w.scale, w.rowsum, s);
  if (st != BL_OK) return st;
  if (M <= kSkinnyMaxM) {
    SkinnyWs none{};
    return launch_skinny_plan(w.xq, packed, w.rowsum, w.scale, gamma, y, y_dtype, M, N, K,
                              skinny_plan_unsplit(M, N, K), none, s);
  }
  return launch_gemm(w.xq, packed, w.rowsum, w.scale, gamma, y, y_dtype, M, N, K, s);
}

bl_status bitlinear_debug_timeout_probe(uint64_t timeout_ns, void* stream) {
  if (timeout_ns < 1000ull || timeout_ns > 5000000000ull) return BL_ERR_INVALID_ARG;
  timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
  return launch_status();
}

bl_status bitlinear_debug_plan(int M, int N, int K, int sms, int* path, int* k_splits) {
  if (!path || !k_splits || sms < 1) return BL_ERR_INVALID_ARG;
  if (!shape_ok(M, N, K)) return BL_ERR_UNSUPPORTED_SHAPE;
  *k_splits = 1;
  if (use_gemv(M, N, K)) {
    *path = 0;
  } else if (M <= kSkinnyMaxM) {
    *path = 1;
    *k_splits = skinny_plan_for(M, N, K, sms).splits;
  } else {
    *path = 2;
  }
  return BL_OK;
}

const char* bitlinear_status_string(bl_status status) {
  switch (status) {
    case BL_OK: return "BL_OK";
    case BL_ERR_INVALID_ARG: return "BL_ERR_INVALID_ARG";
    case BL_ERR_UNSUPPORTED_SHAPE: return "BL_ERR_UNSUPPORTED_SHAPE";
    case BL_ERR_MISALIGNED: return "BL_ERR_MISALIGNED";
    case BL_ERR_CUDA: return "BL_ERR_CUDA";
    case BL_ERR_TIMEOUT: return "BL_ERR_TIMEOUT";
    case BL_ERR_NONFINITE: return "BL_ERR_NONFINITE";
    case BL_ERR_WORKSPACE: return "BL_ERR_WORKSPACE";
  }
  return "BL_ERR_UNKNOWN";
}

}  // extern "C"
