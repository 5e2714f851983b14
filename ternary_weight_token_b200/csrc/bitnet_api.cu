// bitnet_api.cu -- the C ABI (include/bitnet.h): host-side validation,
// dispatch and launch of the BitLinear kernels.  The only translation unit of
// the library: every kernel header is included here so the device error word
// is a single symbol.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <chrono>
#include <map>
#include <mutex>
#include <random>
#include <string>
#include <tuple>
#include <utility>
#include <unordered_map>

#include "../../include/bitnet.h"
#include "common.cuh"
#include "ffn_decode.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "gemv_tc.cuh"
#include "pack_weights.cuh"
#include "quant_act.cuh"

namespace bitnet {
namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

#define BN_CHECK_CUDA(expr)                                                              \
  do {                                                                                   \
    cudaError_t e_ = (expr);                                                             \
    if (e_ != cudaSuccess) return fail(BITNET_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align128(size_t x) { return (x + 127) & ~size_t(127); }

constexpr int kMaxK = 16384;

int check_k(int K) {
  if (K < 16 || K > kMaxK || K % 16 != 0)
    return fail(BITNET_ERR_INVALID_ARG, "K=%d must be a multiple of 16 in [16, %d]", K, kMaxK);
  return BITNET_OK;
}

struct DeviceInfo {
  int sms = 0;
  int max_smem_optin = 0;
  int smem_per_sm = 0;
};

int device_info(DeviceInfo& out) {
  static std::mutex mu;
  static std::unordered_map<int, DeviceInfo> cache;
  int dev = 0;
  BN_CHECK_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(dev);
  if (it == cache.end()) {
    DeviceInfo di;
    BN_CHECK_CUDA(cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev));
    BN_CHECK_CUDA(
        cudaDeviceGetAttribute(&di.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
    BN_CHECK_CUDA(
        cudaDeviceGetAttribute(&di.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev));
    it = cache.emplace(dev, di).first;
  }
  out = it->second;
  return BITNET_OK;
}

// Kernel attributes belong to each device's context: the dynamic
// shared-memory limit set for a kernel, and the occupancy found for a launch
// shape, are cached per device (so a call makes no driver query once warm)
// and cleared by bitnet_release_cache.
std::mutex g_attr_mu;
std::map<std::pair<int, const void*>, size_t> g_smem_set;
std::map<std::tuple<int, const void*, int, size_t>, int> g_occupancy;

int set_smem_attr(const void* fn, size_t bytes) {
  int dev = 0;
  BN_CHECK_CUDA(cudaGetDevice(&dev));
  {
    std::lock_guard<std::mutex> lock(g_attr_mu);
    auto it = g_smem_set.find({dev, fn});
    if (it != g_smem_set.end() && it->second >= bytes) return BITNET_OK;
  }
  BN_CHECK_CUDA(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
  std::lock_guard<std::mutex> lock(g_attr_mu);
  size_t& v = g_smem_set[{dev, fn}];
  if (bytes > v) v = bytes;
  return BITNET_OK;
}

int occupancy(int& per_sm, const void* fn, int threads, size_t smem) {
  int dev = 0;
  BN_CHECK_CUDA(cudaGetDevice(&dev));
  const auto key = std::make_tuple(dev, fn, threads, smem);
  {
    std::lock_guard<std::mutex> lock(g_attr_mu);
    auto it = g_occupancy.find(key);
    if (it != g_occupancy.end()) {
      per_sm = it->second;
      return BITNET_OK;
    }
  }
  BN_CHECK_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem));
  std::lock_guard<std::mutex> lock(g_attr_mu);
  g_occupancy[key] = per_sm;
  return BITNET_OK;
}

// ------------------------------------------------------------ TMA maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int get_encode_fn(EncodeTiledFn& fn) {
  static EncodeTiledFn cached = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess)
      cached = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (cached == nullptr)
    return fail(BITNET_ERR_CUDA, "cuTensorMapEncodeTiled unavailable: %s", cudaGetErrorString(err));
  fn = cached;
  return BITNET_OK;
}

struct MapKey {
  uintptr_t ptr;
  uint64_t d0, d1, stride;
  uint32_t b0, b1, swz, dtype;
  int dev;
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && d0 == o.d0 && d1 == o.d1 && stride == o.stride && b0 == o.b0 &&
           b1 == o.b1 && swz == o.swz && dtype == o.dtype && dev == o.dev;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    size_t h = std::hash<uint64_t>()(k.ptr);
    h = h * 1000003u ^ std::hash<uint64_t>()(k.d0);
    h = h * 1000003u ^ std::hash<uint64_t>()(k.d1);
    h = h * 1000003u ^ std::hash<uint64_t>()(k.stride);
    h = h * 1000003u ^ std::hash<uint64_t>()(((uint64_t)k.b0 << 32) | k.b1);
    h = h * 1000003u ^ std::hash<uint64_t>()(((uint64_t)k.swz << 40) | ((uint64_t)k.dtype << 32) |
                                             (uint32_t)k.dev);
    return h;
  }
};

constexpr size_t kMapCacheMax = 16384;   // descriptors (128 B each) kept at most
std::mutex g_map_mu;
std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_map_cache;

// 2-D tensor [d1 rows][d0 elements] of `dtype` with row stride `stride` bytes,
// box [b1 rows][b0 elements].
int tensor_map_2d(CUtensorMap& out, const void* ptr, CUtensorMapDataType dtype, uint64_t d0,
                  uint64_t d1, uint64_t stride, uint32_t b0, uint32_t b1,
                  CUtensorMapSwizzle swz) {
  int dev = 0;
  BN_CHECK_CUDA(cudaGetDevice(&dev));
  MapKey key{reinterpret_cast<uintptr_t>(ptr), d0, d1, stride, b0, b1, (uint32_t)swz,
             (uint32_t)dtype, dev};
  {
    std::lock_guard<std::mutex> lock(g_map_mu);
    auto it = g_map_cache.find(key);
    if (it != g_map_cache.end()) {
      out = it->second;
      return BITNET_OK;
    }
  }
  EncodeTiledFn enc = nullptr;
  if (int rc = get_encode_fn(enc)) return rc;
  cuuint64_t dims[2] = {d0, d1};
  cuuint64_t strides[1] = {stride};
  cuuint32_t box[2] = {b0, b1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&out, dtype, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BITNET_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  std::lock_guard<std::mutex> lock(g_map_mu);
  // bounded: a caller that keeps passing new buffers starts the cache over
  // instead of growing it without limit
  if (g_map_cache.size() >= kMapCacheMax) g_map_cache.clear();
  g_map_cache[key] = out;
  return BITNET_OK;
}

int tensor_map_2d_u8(CUtensorMap& out, const void* ptr, uint64_t d0, uint64_t d1, uint64_t stride,
                     uint32_t b0, uint32_t b1, CUtensorMapSwizzle swz) {
  return tensor_map_2d(out, ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, d0, d1, stride, b0, b1, swz);
}

// ------------------------------------------------------------- launchers

// Launch with programmatic dependent launch: the kernel may begin its on-chip
// setup while the preceding grid on the stream finishes; every kernel
// launched this way executes griddepcontrol.wait before touching global memory.
template <typename... KArgs, typename... Args>
int launch_pdl_if(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                  cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  BN_CHECK_CUDA(cudaLaunchKernelEx(&cfg, kern, args...));
  return BITNET_OK;
}

template <typename... KArgs, typename... Args>
int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
               Args... args) {
  return launch_pdl_if(true, kern, grid, block, smem, st, args...);
}
// Register-resident rows, NT threads x VPT 16-byte chunks, one CTA per row
// (grid-stride over at most sms * 64 CTAs).
template <int NT, int VPT>
int launch_quant_rows(const QuantParams& p, bool bf16, int prelude, cudaStream_t st) {
  DeviceInfo di;
  if (int rc = device_info(di)) return rc;
  void (*kern)(QuantParams) = nullptr;
  if (prelude == PRE_GLU_RMSNORM)
    kern = quant_act_reg_kernel<NT, VPT, PRE_GLU_RMSNORM, false>;
  else if (prelude == PRE_RMSNORM)
    kern = bf16 ? quant_act_reg_kernel<NT, VPT, PRE_RMSNORM, true>
                : quant_act_reg_kernel<NT, VPT, PRE_RMSNORM, false>;
  else
    kern = bf16 ? quant_act_reg_kernel<NT, VPT, PRE_NONE, true>
                : quant_act_reg_kernel<NT, VPT, PRE_NONE, false>;
  const int grid = p.M < di.sms * 64 ? p.M : di.sms * 64;
  return launch_pdl(kern, dim3(grid), dim3(NT), 0, st, p);
}

// X2: the up projection when prelude is PRE_GLU_RMSNORM (X is then the gate
// projection, both fp32), else null.
int launch_quant(const void* X, bool bf16, int M, int K, int prelude, const float* gain,
                 float eps, int8_t* Xq, float* scale, int32_t* rowsum, cudaStream_t st,
                 const float* X2 = nullptr) {
  DeviceInfo di;
  if (int rc = device_info(di)) return rc;
  QuantParams p;
  p.X = X; p.X2 = X2; p.M = M; p.K = K; p.gain = gain; p.eps = eps;
  p.fwht_c = (float)(1.0 / std::sqrt((double)K));
  p.Xq = Xq; p.scale = scale; p.rowsum = rowsum;
  if (!is_fwht(prelude)) {
    // NT threads x VPT 16-byte chunks must cover the row (K / 4 fp32 chunks,
    // K / 8 bf16 units of two chunks)
    const int k4 = K / 4;
    if (k4 <= 64 * 4) return launch_quant_rows<64, 4>(p, bf16, prelude, st);
    if (k4 <= 64 * 10) return launch_quant_rows<64, 10>(p, bf16, prelude, st);
    if (k4 <= 128 * 8) return launch_quant_rows<128, 8>(p, bf16, prelude, st);
    if (k4 <= 128 * 14) return launch_quant_rows<128, 14>(p, bf16, prelude, st);
    return launch_quant_rows<256, 16>(p, bf16, prelude, st);   // K <= 16384
  }
  // FWHT rows of 128 (fp32) / 256 (bf16) up to 2048 inputs: the row in
  // registers, one warp per row up to 256 inputs, two up to 1024, four at
  // 2048; other widths: the row staged in shared memory
  const bool silu = prelude == PRE_SILU_FWHT;
  if (K <= 2048 && K >= (bf16 ? 256 : 128) && !(silu && bf16)) {
    void (*kw)(QuantParams) = nullptr;
    if (silu) {                    // fp32 hidden rows of the H-BitLinear FFN
      switch (K) {
        case 128: kw = quant_fwht_warp_kernel<128, false, true, 1>; break;
        case 256: kw = quant_fwht_warp_kernel<256, false, true, 1>; break;
        case 512: kw = quant_fwht_warp_kernel<512, false, true, 2>; break;
        case 1024: kw = quant_fwht_warp_kernel<1024, false, true, 2>; break;
        default: kw = quant_fwht_warp_kernel<2048, false, true, 4>; break;
      }
    } else {
      switch (K) {
        case 128: kw = quant_fwht_warp_kernel<128, false, false, 1>; break;
        case 256:
          kw = bf16 ? quant_fwht_warp_kernel<256, true, false, 1> : quant_fwht_warp_kernel<256, false, false, 1>;
          break;
        case 512:
          kw = bf16 ? quant_fwht_warp_kernel<512, true, false, 2> : quant_fwht_warp_kernel<512, false, false, 2>;
          break;
        case 1024:
          kw = bf16 ? quant_fwht_warp_kernel<1024, true, false, 2> : quant_fwht_warp_kernel<1024, false, false, 2>;
          break;
        default:
          kw = bf16 ? quant_fwht_warp_kernel<2048, true, false, 4> : quant_fwht_warp_kernel<2048, false, false, 4>;
          break;
      }
    }
    const int wpr = K >= 2048 ? 4 : K >= 512 ? 2 : 1;
    const int rows_per_cta = 4 / wpr;
    const int need = (M + rows_per_cta - 1) / rows_per_cta;
    const int cap = di.sms * 16;
    return launch_pdl(kw, dim3(need < cap ? need : cap), dim3(128), 0, st, p);
  }
  const int threads = K >= 2048 ? 256 : 128;
  const size_t smem = (size_t)K * sizeof(float);
  const int grid = M < di.sms * 16 ? M : di.sms * 16;
  void (*kern)(QuantParams) =
      silu ? (bf16 ? quant_act_kernel<PRE_SILU_FWHT, true> : quant_act_kernel<PRE_SILU_FWHT, false>)
           : (bf16 ? quant_act_kernel<PRE_FWHT, true> : quant_act_kernel<PRE_FWHT, false>);
  if (int rc = set_smem_attr((const void*)kern, smem)) return rc;
  return launch_pdl(kern, dim3(grid), dim3(threads), smem, st, p);
}

int launch_gemv(const LinearParams& p, cudaStream_t st) {
  DeviceInfo di;
  if (int rc = device_info(di)) return rc;
  const int MT = p.M <= 1 ? 1 : p.M <= 2 ? 2 : p.M <= 4 ? 4 : p.M <= 8 ? 8 : 16;
  const size_t smem = (size_t)MT * (size_t)p.ldw * 4;
  if (smem > (size_t)di.max_smem_optin)
    return fail(BITNET_ERR_UNSUPPORTED, "decode activations (%d x %d) exceed shared memory", p.M,
                p.K);
  void (*kern)(LinearParams) = nullptr;
  switch (MT) {
    case 1: kern = gemv_kernel<1>; break;
    case 2: kern = gemv_kernel<2>; break;
    case 4: kern = gemv_kernel<4>; break;
    case 8: kern = gemv_kernel<8>; break;
    default: kern = gemv_kernel<16>; break;
  }
  if (int rc = set_smem_attr((const void*)kern, smem)) return rc;
  int per_sm = 0;
  if (int rc = occupancy(per_sm, (const void*)kern, kGemvThreads, smem)) return rc;
  if (per_sm < 1) per_sm = 1;
  const int rows_per_cta = (kGemvThreads / 32) * kGemvRows;
  const int need = (p.N + rows_per_cta - 1) / rows_per_cta;
  const int cap = di.sms * per_sm;
  const int grid = need < cap ? need : cap;
  kern<<<grid, kGemvThreads, smem, st>>>(p);
  BN_CHECK_CUDA(cudaGetLastError());
  return BITNET_OK;
}

template <class C>
int launch_tc_cfg(const LinearParams& lp, const uint8_t* W1, const float* gamma1,
                  cudaStream_t st) {
  DeviceInfo di;
  if (int rc = device_info(di)) return rc;
  CUtensorMap mx, mw0, mw1;
  if (int rc = tensor_map_2d_u8(mx, lp.Xq, (uint64_t)lp.K, (uint64_t)lp.M, (uint64_t)lp.K, 128,
                                C::BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return rc;
  // packed weight rows of BK/4 bytes, swizzled at that width (conflict-free
  // 16-byte loads in the converter)
  const CUtensorMapSwizzle wswz =
      C::BK / 4 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  static_assert(C::BK / 4 == 64 || C::BK / 4 == 32, "packed stage width");
  // GLU: 64 gate rows and 64 up rows per tile (two boxes), else 128 rows
  const uint32_t wrows = C::GLU ? C::BM / 2 : C::BM;
  if (int rc = tensor_map_2d_u8(mw0, lp.W, (uint64_t)lp.ldw, (uint64_t)lp.N, (uint64_t)lp.ldw,
                                C::BK / 4, wrows, wswz))
    return rc;
  mw1 = mw0;
  if (C::GLU) {
    if (int rc = tensor_map_2d_u8(mw1, W1, (uint64_t)lp.ldw, (uint64_t)lp.N, (uint64_t)lp.ldw,
                                  C::BK / 4, wrows, wswz))
      return rc;
  }
  // Output through TMA stores when its rows are whole 16-byte units.
  const int esz = lp.out_type == OUT_BF16 ? 2 : 4;
  const bool tma_out = ((size_t)lp.N * esz) % 16 == 0;
  CUtensorMap my = mx;
  if (tma_out) {
    const CUtensorMapDataType dt = lp.out_type == OUT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                   : lp.out_type == OUT_I32 ? CU_TENSOR_MAP_DATA_TYPE_INT32
                                                            : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    // the bf16 fragment epilogue (no GLU) stages 64-byte rows with the
    // 64-byte swizzle, so its transposing stores are bank-conflict free
    const bool frag = !C::GLU && lp.out_type == OUT_BF16;
    // GLU: each epilogue warp stores 16 features x 32 tokens (fp32 m)
    if (int rc = tensor_map_2d(my, lp.Y, dt, (uint64_t)lp.N, (uint64_t)lp.M,
                               (uint64_t)lp.N * esz, C::GLU ? 16 : 32, 32,
                               frag ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE))
      return rc;
  }
  // bf16 residual of the fragment epilogue through TMA (the same box and
  // swizzle as the output staging)
  CUtensorMap mr = my;
  const bool tma_res = tma_out && !C::GLU && lp.out_type == OUT_BF16 && lp.resid != nullptr &&
                       (lp.flags & EPI_RESIDUAL);
  if (tma_res) {
    if (int rc = tensor_map_2d(mr, lp.resid, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)lp.N,
                               (uint64_t)lp.M, (uint64_t)lp.N * 2, 32, 32,
                               CU_TENSOR_MAP_SWIZZLE_64B))
      return rc;
  }
  TcParams p;
  p.tma_out = tma_out ? 1 : 0;
  p.tma_res = tma_res ? 1 : 0;
  p.M = lp.M; p.N = lp.N; p.K = lp.K;
  p.num_kb = (lp.K + C::BK - 1) / C::BK;
  p.tiles_n = (lp.N + C::TILE_N - 1) / C::TILE_N;
  const int tiles_m = (lp.M + C::BN - 1) / C::BN;
  p.num_tiles = p.tiles_n * tiles_m;

  p.w_early = lp.w_early;
  p.xs = lp.xs; p.xrs = lp.xrs; p.gamma0 = lp.gamma; p.gamma1 = gamma1;
  p.Y = lp.Y; p.resid = lp.resid; p.out_type = lp.out_type; p.flags = lp.flags;
  // One CTA per SM: request enough shared memory that two never co-reside
  // (each holds all 512 tensor-memory columns).
  size_t smem = C::SMEM_ALLOC;
  const size_t one_per_sm = (size_t)di.max_smem_optin / 2 + 1024;
  if (smem < one_per_sm) smem = one_per_sm;
  if (smem > (size_t)di.max_smem_optin) smem = di.max_smem_optin;
  auto kern = gemm_tc_kernel<C>;
  if (int rc = set_smem_attr((const void*)kern, smem)) return rc;
  const int grid = p.num_tiles < di.sms ? p.num_tiles : di.sms;
  return launch_pdl(kern, dim3(grid), dim3(C::THREADS), smem, st, mx, mw0, mw1, my, mr, p);
}

// Devices whose context has the decode kernel's shared-memory attribute set
// (a bit per device ordinal); cleared by bitnet_release_cache so that a
// context created after cudaDeviceReset gets it again.
std::atomic<uint64_t> g_dec_attr_set{0};

using TcPlain = TcConfig<128, 256, 4, false>;
using TcPlain96 = TcConfig<96, 256, 4, false>;     // 96-token tiles (tile quantisation, below)
using TcPlain64 = TcConfig<64, 256, 4, false>;     // 64-token tiles (single-wave calls, below)
using TcSilu = TcConfig<128, 256, 4, false, true>;
using TcGlu = TcConfig<128, 256, 4, true>;

// The cluster size S of the tensor-core decode GEMV for a call of `tiles`
// 128-row weight tiles, or 0 when K does not split (K not a multiple of 64,
// or more than 8 slices of at most 14 64-input units needed).  Pure host
// logic, shared by the launch and bitnet_plan_linear.
int decode_cluster_size(int M, int K, int tiles, int flags, int sms) {
  const int units = K / 64;
  if (K % 64 != 0 || units < 1) return 0;
  const int s_min = (units + 13) / 14;                    // ceil(units / S) <= 14
  const int s_max = units < kDecMaxCluster ? units : kDecMaxCluster;
  if (s_min > s_max) return 0;
  // The cluster size S grows from the smallest split until the call has at
  // least half a CTA per SM, and for more than 8 tokens until a CTA's slice
  // is at most ten 64-input units while the call stays within two CTAs per
  // SM: more, shorter CTAs do not pay (2560 x 2560 with 80 CTAs of ten units
  // against 160 of five: 3-4 % faster at 3-8 tokens, 11 % at 16; 16 tokens on
  // 2560 x 6912 with 216 CTAs of ten units instead of 162 of fourteen: 4-5 %
  // faster, while up to 8 tokens run best on fourteen; on 2560 x 13824 the
  // 432 CTAs of ten units were no faster).  When the activation codes come
  // from the preceding kernel (a programmatic dependent launch without
  // LAUNCH_PDL_INPUTS), a CTA converts at most three weight chunks (its ring
  // of TMEM slots) before they arrive, and every further chunk costs a round
  // trip between the MMA and the converter warps after that; for up to 8
  // tokens, where the cross-CTA reduction is cheap, such a call takes a CTA
  // per SM and slices that fit the ring (three chunks, six units).
  const bool dependent = (flags & LAUNCH_PDL) && !(flags & LAUNCH_PDL_INPUTS);
  const bool few = M <= 8;
  const int units_fit = dependent && few ? 6 : 1 << 30;
  const int min_ctas = dependent && few ? sms : (sms + 1) / 2;
  int S = s_min;
  while (S < s_max) {
    const int slice = (units + S - 1) / S;
    const bool grow = tiles * S < min_ctas || slice > units_fit ||
                      (!few && slice > 10 && tiles * (S + 1) <= 2 * sms);
    if (!grow) break;
    ++S;
  }
  return S;
}

// Decode on the tensor cores: 128-row weight tiles, each split over K across a
// cluster of S CTAs (S <= 8, every slice at most 896 inputs).  Returns
// BITNET_ERR_UNSUPPORTED when K is too long for that split.
int launch_gemv_tc(const LinearParams& lp, cudaStream_t st) {
  DeviceInfo di;
  if (int rc = device_info(di)) return rc;
  if (decode_cluster_size(lp.M, lp.K, 1, lp.flags, di.sms) == 0) return BITNET_ERR_UNSUPPORTED;
  const int units = lp.K / 64;
  // every projection of the call: its 128-row tiles and packed-weight map
  DecParams p;
  DecMaps maps;
  int tiles = 0;
  p.nseg = lp.nseg;
  for (int i = 0; i < lp.nseg; ++i) {
    const int Ni = lp.seg_row0[i + 1] - lp.seg_row0[i];
    p.seg_tile0[i] = tiles;
    p.seg_N[i] = Ni;
    p.seg_gamma[i] = lp.seg_gamma[i];
    p.seg_Y[i] = lp.seg_Y[i];
    if (int rc = tensor_map_2d_u8(maps.w[i], lp.seg_W[i], (uint64_t)lp.ldw, (uint64_t)Ni,
                                  (uint64_t)lp.ldw, kDecChunkK / 4, 128,
                                  CU_TENSOR_MAP_SWIZZLE_NONE))
      return rc;
    tiles += (Ni + 127) / 128;
  }
  for (int i = lp.nseg; i <= kMaxSegments; ++i) p.seg_tile0[i] = tiles;
  for (int i = lp.nseg; i < kMaxSegments; ++i) maps.w[i] = maps.w[0];
  const int S = decode_cluster_size(lp.M, lp.K, tiles, lp.flags, di.sms);
  if (S == 0) return BITNET_ERR_UNSUPPORTED;
  CUtensorMap mx;
  if (int rc = tensor_map_2d_u8(mx, lp.Xq, (uint64_t)lp.K, (uint64_t)lp.M, (uint64_t)lp.K, 128,
                                kDecTokens, CU_TENSOR_MAP_SWIZZLE_128B))
    return rc;
  p.M = lp.M; p.K = lp.K; p.units = units;
  p.xs = lp.xs; p.xrs = lp.xrs;
  p.resid = lp.resid; p.out_type = lp.out_type;
  p.flags = lp.flags & ~LAUNCH_PDL;     // keeps LAUNCH_PDL_INPUTS for the kernel
  // The shared-memory attribute belongs to each device's context: set it once
  // per device (a bit per device ordinal; ordinals past 63 set it every call).
  std::atomic<uint64_t>& attr_set = g_dec_attr_set;
  int dev = 0;
  BN_CHECK_CUDA(cudaGetDevice(&dev));
  const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t)1 << dev : 0;
  if (bit == 0 || (attr_set.load(std::memory_order_acquire) & bit) == 0) {
    BN_CHECK_CUDA(cudaFuncSetAttribute(gemv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       DecSmem::ALLOC));
    attr_set.fetch_or(bit, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(tiles * S), 1, 1);
  cfg.blockDim = dim3(kDecThreads, 1, 1);
  cfg.dynamicSmemBytes = DecSmem::ALLOC;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = (unsigned)S;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = (lp.flags & LAUNCH_PDL) ? 1 : 0;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  BN_CHECK_CUDA(cudaLaunchKernelEx(&cfg, gemv_tc_kernel, mx, maps, p));
  return BITNET_OK;
}

// Decode for 1..2 tokens with K a multiple of 64: the dp4a streaming kernel
// (a warp per R rows, all of a lane's weight loads in flight at once).
constexpr int kStreamChunks = 8;               // packed chunks per lane, at most

template <int MT>
int launch_stream_mt(const LinearParams& p, int L, int warps, int grid, cudaStream_t st) {
  void (*kern)(LinearParams, int) = gemv_stream_kernel<MT, kStreamChunks>;
  const size_t smem = (size_t)MT * (size_t)p.K;  // activation codes
  if (int rc = set_smem_attr((const void*)kern, smem)) return rc;
  LinearParams q = p;
  q.flags &= ~LAUNCH_PDL;
  return launch_pdl_if((p.flags & LAUNCH_PDL) != 0, kern, dim3(grid), dim3(32 * warps), smem, st,
                       q, L);
}

constexpr int kFlatThreads = 256;

template <int MT>
int launch_flat_mt(const LinearParams& p, int R, bool bulk, cudaStream_t st) {
  void (*kern)(LinearParams) = nullptr;
#define BN_FLAT_CASE(RR)                                                                  \
  case RR:                                                                                \
    kern = bulk ? gemv_flat_kernel<MT, RR, kStreamChunks, kFlatThreads, true>             \
                : gemv_flat_kernel<MT, RR, kStreamChunks, kFlatThreads, false>;           \
    break;
  switch (R) {
    BN_FLAT_CASE(1)
    BN_FLAT_CASE(2)
    BN_FLAT_CASE(3)
    BN_FLAT_CASE(4)
    BN_FLAT_CASE(5)
    BN_FLAT_CASE(6)
    BN_FLAT_CASE(7)
    default:
      kern = bulk ? gemv_flat_kernel<MT, 8, kStreamChunks, kFlatThreads, true>
                  : gemv_flat_kernel<MT, 8, kStreamChunks, kFlatThreads, false>;
      break;
  }
#undef BN_FLAT_CASE
  const int warps = kFlatThreads / 32;
  const int grid = (p.N + warps * R - 1) / (warps * R);
  // (bulk) the CTA's weight rows, then the activation codes
  const size_t smem = (bulk ? (size_t)warps * R * p.ldw : 0) + (size_t)MT * (size_t)p.K;
  if (int rc = set_smem_attr((const void*)kern, smem)) return rc;
  LinearParams q = p;
  q.flags &= ~LAUNCH_PDL;
  return launch_pdl_if((p.flags & LAUNCH_PDL) != 0, kern, dim3(grid), dim3(kFlatThreads), smem,
                       st, q);
}

// Launch shape of the streaming decode kernels for a call (pure host logic,
// shared by the launch and bitnet_plan_linear): the flat kernel (`flat`,
// token tile mt, R rows per warp, bulk-copied rows) or the row groups (L
// lanes per row, `warps` warps per CTA); `grid` CTAs.
struct StreamShape {
  bool flat = false, bulk = false;
  int mt = 1, R = 1, L = 1, warps = 1, grid = 0;
};

StreamShape stream_shape(int M, int N, int K, int ldw, int flags, int sms) {
  StreamShape sh;
  const int C = ldw / 16;                      // 16-byte chunks per row (K / 64), <= 256
  const int mt = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
  // Independent calls (LAUNCH_PDL_INPUTS) and 3-8 tokens take the flat
  // kernel; independent calls on 4 MB of weights or more bulk-copy their
  // weight rows into shared memory there, so that more calls' CTAs share an
  // SM (1.6 MB single and 2.5 MB q/k/v calls measured slower with the bulk
  // copies, 4.4 MB ones faster).  Dependent calls take the row groups.
  const bool independent = (flags & LAUNCH_PDL_INPUTS) != 0;
  if (independent || mt == 8 || (mt == 4 && (long long)N * K <= (1ll << 20))) {
    // R rows per warp: about one CTA per two SMs per call (fewer, fuller CTAs
    // let more back-to-back calls overlap: independent 1-2 token calls on
    // 2560 x 2560 0.88 -> 0.81 / 1.49 -> 1.31 us and the q/k/v step 1.15 ->
    // 1.08 us against a CTA per SM), at most 8 chunks a lane
    const int warps = kFlatThreads / 32;
    const int half = (sms + 1) / 2;
    int R = (N + half * warps - 1) / (half * warps);
    if (R > 8) R = 8;
    while (R > 1 && R * C > 32 * kStreamChunks) --R;
    sh.mt = mt == 4 ? 8 : mt;                  // the flat kernel's token tiles: 1, 2, 8
    if (sh.mt == 8 && R > 4) R = 4;            // lane r * MT + m holds (row, token): R MT <= 32
    sh.flat = true;
    sh.R = R;
    sh.warps = warps;
    sh.bulk = independent && (long long)N * ldw >= (1ll << 22);
    sh.grid = (N + warps * R - 1) / (warps * R);
    return sh;
  }
  // L lanes per row (a power of two): each lane at most kStreamChunks chunks,
  // and on small matrices more lanes per row, so that the call still has
  // about 256 lanes per SM, 128 for 3-4 tokens, whose longer per-lane sums
  // pay off there (2560 x 2560, dependent: 5.05 -> 4.69 us at 4 tokens; 1-2
  // tokens were 3-6 % slower with 128) (a row has C chunks: no more than C
  // lanes)
  const long long lanes_per_sm = mt == 4 ? 128 : 256;
  int L = 1;
  while (L * kStreamChunks < C) L *= 2;
  while (L < 32 && L < C && (long long)N * L < (long long)sms * lanes_per_sm) L *= 2;
  const int G = 32 / L;                        // rows per warp
  // warps per CTA: about one CTA per SM per call (so several back-to-back
  // calls can be resident at once), at most 8
  int warps = N / (sms * G);
  if (warps > 8) warps = 8;
  if (warps < 1) warps = 1;
  const int rows = warps * G;
  sh.mt = mt;
  sh.L = L;
  sh.warps = warps;
  sh.grid = (N + rows - 1) / rows;
  return sh;
}

int launch_gemv_stream(const LinearParams& p, cudaStream_t st) {
  DeviceInfo di;
  if (int rc = device_info(di)) return rc;
  const StreamShape sh = stream_shape(p.M, p.N, p.K, p.ldw, p.flags, di.sms);
  if (sh.flat) {
    if (sh.mt == 1) return launch_flat_mt<1>(p, sh.R, sh.bulk, st);
    if (sh.mt == 2) return launch_flat_mt<2>(p, sh.R, sh.bulk, st);
    return launch_flat_mt<8>(p, sh.R, sh.bulk, st);
  }
  if (sh.mt == 1) return launch_stream_mt<1>(p, sh.L, sh.warps, sh.grid, st);
  if (sh.mt == 2) return launch_stream_mt<2>(p, sh.L, sh.warps, sh.grid, st);
  return launch_stream_mt<4>(p, sh.L, sh.warps, sh.grid, st);
}

// Projection i of a call as a call of its own.
LinearParams segment_params(const LinearParams& p, int i) {
  LinearParams q = p;
  q.W = p.seg_W[i];
  q.gamma = p.seg_gamma[i];
  q.Y = p.seg_Y[i];
  q.N = p.seg_row0[i + 1] - p.seg_row0[i];
  single_segment(q);
  return q;
}

// The persistent GEMM runs ceil(tiles / SMs) waves of tiles.  A tile's time is
// a fixed part (converting its 128 weight rows, the epilogue's setup) plus a
// part proportional to its tokens; timing 6912 -> 2560 at 4096 tokens with
// 128- and 96-token tiles (5 and 6 waves: 61.8 and 68.5 us) puts the fixed
// part at ~270 tokens' worth.  The token tile (128, 96 or 64 tokens) is the
// one with the smallest waves x (tokens + 270), 128 unless another is clearly
// (3 %) smaller.  96 takes a last wave of 128-token tiles that would leave
// most SMs idle, e.g. 2048 tokens x 2560 rows (320 tiles, 3 waves; 440 tiles
// of 96, still 3 waves); 64 wins on single-wave GEMMs with few row tiles,
// e.g. 1024 tokens x 512 rows (64 tiles of 64 against 44 of 96: each CTA
// multiplies and dequantises fewer tokens for the same weight stages; H-FFN
// 25.5 -> 24.4 us).
int token_tile(int M, int N, int sms) {
  if (sms <= 0) return 128;
  auto cost = [&](int bn) {
    const long long tiles = (long long)((M + bn - 1) / bn) * ((N + 127) / 128);
    return ((tiles + sms - 1) / sms) * (bn + 270);
  };
  int best = 128;
  long long best_cost = cost(128) * 97;
  for (int bn : {96, 64}) {
    if (cost(bn) * 100 < best_cost) {
      best = bn;
      best_cost = cost(bn) * 100;
    }
  }
  return best;
}

// Whether a call takes the streaming decode kernels (pure host logic).
// 1-2 tokens: the dp4a streaming kernels (measured faster than the cluster
// tensor-core path there).  Up to 8 tokens on small weight matrices (<= 2^20
// weights, e.g. 256 x 512): the streaming kernels too, whose short CTAs beat
// the cluster path's TMEM set-up and reduction there (6.2 -> 4.4 us per
// quantise + project pair).  3-4 tokens of a dependent call on rows of up to
// 4096 inputs: the row-group streaming kernel (dependent 3-4 token calls on
// 2560-input rows 4-9 % faster than the cluster tensor-core kernel; on
// 6912-input rows its lanes' chains are long and it was 7-11 % slower).
bool takes_stream(int M, int N, int K, int ldw, int flags) {
  const bool stream_ok = K % 64 == 0 && ldw / 16 <= 32 * 8;
  const bool dependent4 = M <= 4 && (flags & LAUNCH_PDL_INPUTS) == 0 && K <= 4096;
  return stream_ok && (M <= 2 || dependent4 || (M <= 8 && (long long)N * K <= (1ll << 20)));
}

int launch_linear(const LinearParams& p, cudaStream_t st) {
  // Every decode kernel runs all projections of the call in one launch.
  if (takes_stream(p.M, p.N, p.K, p.ldw, p.flags)) return launch_gemv_stream(p, st);
  if (p.M <= 16) {
    const int rc = launch_gemv_tc(p, st);
    if (rc != BITNET_ERR_UNSUPPORTED) return rc;
  }
  // one launch per projection: the prefill GEMM, or decode inputs too long
  // for the cluster split (the plain dp4a kernel)
  DeviceInfo di;
  if (int rc = device_info(di)) return rc;
  for (int i = 0; i < p.nseg; ++i) {
    LinearParams q = segment_params(p, i);
    int rc;
    if (q.M <= 16) {
      q.flags &= ~(LAUNCH_PDL | LAUNCH_PDL_INPUTS);
      rc = launch_gemv(q, st);
    } else if (q.flags & EPI_SILU) {
      rc = launch_tc_cfg<TcSilu>(q, nullptr, nullptr, st);
    } else if (const int bn = token_tile(q.M, q.N, di.sms); bn != 128) {
      rc = bn == 96 ? launch_tc_cfg<TcPlain96>(q, nullptr, nullptr, st)
                    : launch_tc_cfg<TcPlain64>(q, nullptr, nullptr, st);
    } else {
      rc = launch_tc_cfg<TcPlain>(q, nullptr, nullptr, st);
    }
    if (rc) return rc;
  }
  return BITNET_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Epochs of the grid-wide exchanges (persistent decode FFN, one-launch pack): a per-process
// 64-bit counter started at a random value, so no launch reuses an epoch and
// a workspace's initial contents match one with negligible probability.
uint64_t next_epoch() {
  static std::atomic<uint64_t> counter{[] {
    std::random_device rd;
    uint64_t v = ((uint64_t)rd() << 32) ^ (uint64_t)rd() ^
                 (uint64_t)std::chrono::steady_clock::now().time_since_epoch().count();
    return v | 1u;
  }()};
  uint64_t e = counter.fetch_add(1, std::memory_order_relaxed);
  return e == 0 ? counter.fetch_add(1, std::memory_order_relaxed) : e;
}

// The decode FFN in one cooperative launch (ffn_decode.cuh).  Returns
// BITNET_ERR_UNSUPPORTED (nothing launched) when the shape does not fit it:
// widths not multiples of 128, more than 64 features per CTA, or staged
// weights and codes beyond the shared memory of an SM.
int launch_ffn_decode(FfnDecodeParams p, cudaStream_t st, bool tail = false) {
  DeviceInfo di;
  if (int rc = device_info(di)) return rc;
  if (p.M < 1 || p.M > 16 || p.H % 128 != 0 || p.I % 128 != 0) return BITNET_ERR_UNSUPPORTED;
  int G = std::min(std::min(di.sms, kFdMaxGrid), (p.I + 7) / 8);
  p.nf_per = (p.I + G - 1) / G;
  p.slots = (p.nf_per + 7) / 8;
  if (p.slots > kFdMaxSlots) return BITNET_ERR_UNSUPPORTED;
  p.nr_per = (p.H + G - 1) / G;
  if (p.nr_per > 32) return BITNET_ERR_UNSUPPORTED;
  p.mpad = p.M <= 8 ? 8 : 16;
  p.sx_h = p.H + kFdRowPad;
  p.sx_i = p.I + kFdRowPad;
  // gate and up sub-blocks, then down (TAIL: o_proj rows first, in the same
  // place), then the staged codes
  const size_t gu = align128((size_t)sb_bytes(p.nf_per, p.ldwH));
  p.off_u = (int)gu;
  p.off_d = (int)(2 * gu);
  const size_t dn = std::max((size_t)sb_bytes(p.nr_per, p.ldwI),
                             tail ? (size_t)sb_bytes(p.nr_per, p.ldwH) : (size_t)0);
  p.off_act = (int)align128((size_t)p.off_d + dn);
  const size_t smem =
      (size_t)p.off_act + (size_t)p.mpad * (size_t)std::max(p.sx_h, p.sx_i) + 128;
  if (smem + sizeof(FfnDecodeShared) + 1024 > (size_t)di.max_smem_optin) return BITNET_ERR_UNSUPPORTED;
  void (*kern)(FfnDecodeParams) = tail ? ffn_decode_kernel<true> : ffn_decode_kernel<false>;
  if (int rc = set_smem_attr((const void*)kern, smem)) return rc;
  int per_sm = 0;
  if (int rc = occupancy(per_sm, (const void*)kern, kFdThreads, smem)) return rc;
  if (per_sm < 1) return BITNET_ERR_UNSUPPORTED;
  p.epoch = next_epoch();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)G);
  cfg.blockDim = dim3(kFdThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;     // every CTA resident: the exchange waits on all
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  BN_CHECK_CUDA(cudaLaunchKernelEx(&cfg, kern, p));
  return BITNET_OK;
}

int validate_linear(const int8_t* Xq, const float* xs, const int32_t* xrs, const uint8_t* W,
                    const float* gamma, int M, int N, int K, const void* Y, int epilogue,
                    const void* resid) {
  if (M < 0 || N < 0) return fail(BITNET_ERR_INVALID_ARG, "M=%d, N=%d must be >= 0", M, N);
  if (int rc = check_k(K)) return rc;
  const int ot = epilogue & BITNET_EPI_TYPE_MASK;
  const int flags = epilogue & ~BITNET_EPI_TYPE_MASK;
  if (ot != BITNET_F32 && ot != BITNET_BF16 && ot != BITNET_I32)
    return fail(BITNET_ERR_INVALID_ARG, "bad output type %d", ot);
  if (flags & ~(BITNET_EPI_RESIDUAL | BITNET_EPI_SILU | BITNET_LAUNCH_PDL | BITNET_LAUNCH_PDL_INPUTS))
    return fail(BITNET_ERR_INVALID_ARG, "unknown epilogue flags 0x%x", flags);
  if (ot == BITNET_I32 && (flags & (BITNET_EPI_RESIDUAL | BITNET_EPI_SILU)))
    return fail(BITNET_ERR_UNSUPPORTED, "the int32 output takes no residual or SiLU");
  if ((flags & BITNET_EPI_RESIDUAL) && resid == nullptr)
    return fail(BITNET_ERR_INVALID_ARG, "residual flag set but residual is NULL");
  if (!(flags & BITNET_EPI_RESIDUAL) && resid != nullptr)
    return fail(BITNET_ERR_INVALID_ARG, "residual given without BITNET_EPI_RESIDUAL");
  if (M == 0 || N == 0) return BITNET_OK;
  if (!Xq || !xs || !xrs || !W || !gamma || !Y)
    return fail(BITNET_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(Xq) || !aligned16(xs) || !aligned16(xrs) || !aligned16(W) || !aligned16(gamma) ||
      !aligned16(Y) || (resid && !aligned16(resid)))
    return fail(BITNET_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  return BITNET_OK;
}

// Device address of the no-allocation FFN scratch (bitnet_ffn_noalloc), per
// device ordinal, looked up once per context.
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

}  // namespace
}  // namespace bitnet

using namespace bitnet;

extern "C" {

size_t bitnet_packed_row_bytes(int K) {
  if (K <= 0) return 0;
  return (size_t)16 * (size_t)((K + 63) / 64);
}

size_t bitnet_pack_workspace_size(int N, int K) {
  (void)N;
  (void)K;
  // one-launch path: two tagged words per CTA's partial sum and the two
  // gamma words; three-launch path: partials
  const size_t fused = (size_t)(2 * kPackMaxGrid + 2) * sizeof(unsigned long long);
  const size_t split = (size_t)kPackPartialBlocks * sizeof(double);
  return fused > split ? fused : split;
}

int bitnet_pack_weights(const void* W, int w_dtype, int N, int K, uint8_t* packed, float* gamma,
                        void* workspace, size_t ws_bytes, bitnet_stream_t stream) {
  g_last_error.clear();
  if (N < 0) return fail(BITNET_ERR_INVALID_ARG, "N=%d must be >= 0", N);
  if (int rc = check_k(K)) return rc;
  if (w_dtype != BITNET_F32 && w_dtype != BITNET_BF16)
    return fail(BITNET_ERR_INVALID_ARG, "weight dtype must be F32 or BF16");
  if (!W || !packed || !gamma) return fail(BITNET_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(W) || !aligned16(packed) || !aligned16(gamma))
    return fail(BITNET_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (workspace == nullptr || ws_bytes < bitnet_pack_workspace_size(N, K))
    return fail(BITNET_ERR_WORKSPACE, "workspace of %zu bytes needed",
                bitnet_pack_workspace_size(N, K));
  if (!aligned16(workspace)) return fail(BITNET_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = w_dtype == BITNET_BF16;
  const long long count = (long long)N * K;
  double* partials = reinterpret_cast<double*>(workspace);
  if (N > 0) {
    // one cooperative launch: two CTAs of 512 threads per SM, each staging
    // up to half of the SM's shared memory of its weights
    DeviceInfo di;
    if (int rc = device_info(di)) return rc;
    void (*kf)(const void*, int, int, int, long long, unsigned long long*, unsigned long long, int,
               float*, uint8_t*) = bf16 ? pack_fused_kernel<true> : pack_fused_kernel<false>;
    int smem = (di.smem_per_sm / 2 - 2048) & ~1023;
    if (smem > kPackMaxStage) smem = kPackMaxStage;
    if (smem > di.max_smem_optin) smem = di.max_smem_optin & ~1023;
    if (smem < 0) smem = 0;
    if (int rc = set_smem_attr((const void*)kf, (size_t)smem)) return rc;
    int per_sm = 0;
    if (int rc = occupancy(per_sm, (const void*)kf, kPackFusedThreads, (size_t)smem)) return rc;
    const int G = std::min(std::min(per_sm, 2) * di.sms, kPackMaxGrid);
    if (G >= di.sms) {
      unsigned long long* xw = reinterpret_cast<unsigned long long*>(workspace);
      const int ldw = (int)bitnet_packed_row_bytes(K);
      const unsigned long long epoch = next_epoch();
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)G);
      cfg.blockDim = dim3(kPackFusedThreads);
      cfg.dynamicSmemBytes = (size_t)smem;
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeCooperative;
      attr[0].val.cooperative = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      BN_CHECK_CUDA(cudaLaunchKernelEx(&cfg, kf, W, N, K, ldw, count, xw, epoch, smem, gamma,
                                       packed));
      return BITNET_OK;
    }
  }
  if (int rc = launch_pdl(bf16 ? absmean_partial_kernel<true> : absmean_partial_kernel<false>,
                          dim3(kPackPartialBlocks), dim3(kPackThreads), 0, st, W, count,
                          partials))
    return rc;
  if (int rc = launch_pdl(absmean_final_kernel, dim3(1), dim3(kPackThreads), 0, st,
                          (const double*)partials, (int)kPackPartialBlocks, count, gamma))
    return rc;
  if (N == 0) return BITNET_OK;
  const int ldw = (int)bitnet_packed_row_bytes(K);
  const long long words = (long long)N * (ldw / 4);
  DeviceInfo di;
  if (int rc = device_info(di)) return rc;
  long long blocks = (words + kPackThreads - 1) / kPackThreads;
  if (blocks > (long long)di.sms * 32) blocks = (long long)di.sms * 32;
  return launch_pdl(bf16 ? pack_kernel<true> : pack_kernel<false>, dim3((int)blocks),
                    dim3(kPackThreads), 0, st, W, N, K, ldw, (const float*)gamma, packed);
}

static int validate_tw2(const void* a, const void* b, int N, int K) {
  if (a == nullptr || b == nullptr) return fail(BITNET_ERR_INVALID_ARG, "null pointer");
  if (N < 0) return fail(BITNET_ERR_INVALID_ARG, "N=%d must be >= 0", N);
  if (int rc = check_k(K)) return rc;
  if (!aligned16(a) || !aligned16(b))
    return fail(BITNET_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  return BITNET_OK;
}

int bitnet_export_tw2(const uint8_t* packed, int N, int K, uint8_t* tw2, bitnet_stream_t stream) {
  g_last_error.clear();
  if (int rc = validate_tw2(packed, tw2, N, K)) return rc;
  if (N == 0) return BITNET_OK;
  DeviceInfo di;
  if (int rc = device_info(di)) return rc;
  const int ldw_words = (int)(bitnet_packed_row_bytes(K) / 4), tw2_words = K / 16;
  const int64_t total = (int64_t)N * tw2_words;
  const int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)di.sms * 8);
  export_tw2_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint32_t*>(packed), N, ldw_words, tw2_words,
      reinterpret_cast<uint32_t*>(tw2));
  BN_CHECK_CUDA(cudaGetLastError());
  return BITNET_OK;
}

int bitnet_import_tw2(const uint8_t* tw2, int N, int K, uint8_t* packed, bitnet_stream_t stream) {
  g_last_error.clear();
  if (int rc = validate_tw2(tw2, packed, N, K)) return rc;
  if (N == 0) return BITNET_OK;
  DeviceInfo di;
  if (int rc = device_info(di)) return rc;
  const int ldw_words = (int)(bitnet_packed_row_bytes(K) / 4), tw2_words = K / 16;
  const int64_t total = (int64_t)N * ldw_words;
  const int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)di.sms * 8);
  import_tw2_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint32_t*>(tw2), N, ldw_words, tw2_words,
      reinterpret_cast<uint32_t*>(packed));
  BN_CHECK_CUDA(cudaGetLastError());
  return BITNET_OK;
}

int bitnet_quant_act(const void* X, int x_dtype, int M, int K, int prelude,
                     const float* norm_gain, float eps, int8_t* Xq, float* x_scale,
                     int32_t* x_rowsum, bitnet_stream_t stream) {
  g_last_error.clear();
  if (M < 0) return fail(BITNET_ERR_INVALID_ARG, "M=%d must be >= 0", M);
  if (int rc = check_k(K)) return rc;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16)
    return fail(BITNET_ERR_INVALID_ARG, "activation dtype must be F32 or BF16");
  if (prelude != BITNET_PRELUDE_NONE && prelude != BITNET_PRELUDE_RMSNORM &&
      prelude != BITNET_PRELUDE_FWHT)
    return fail(BITNET_ERR_INVALID_ARG, "unknown prelude %d", prelude);
  if (prelude == BITNET_PRELUDE_FWHT && (K & (K - 1)) != 0)
    return fail(BITNET_ERR_INVALID_ARG, "FWHT width K=%d is not a power of two", K);
  if (norm_gain != nullptr && prelude != BITNET_PRELUDE_RMSNORM)
    return fail(BITNET_ERR_INVALID_ARG, "norm_gain is only used by the RMSNorm prelude");
  if (prelude == BITNET_PRELUDE_RMSNORM && !(eps >= 0.0f && std::isfinite(eps)))
    return fail(BITNET_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (M == 0) return BITNET_OK;
  if (!X || !Xq || !x_scale) return fail(BITNET_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(X) || !aligned16(Xq) || !aligned16(x_scale) ||
      (x_rowsum && !aligned16(x_rowsum)) || (norm_gain && !aligned16(norm_gain)))
    return fail(BITNET_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  return launch_quant(X, x_dtype == BITNET_BF16, M, K, prelude, norm_gain, eps, Xq, x_scale,
                      x_rowsum, reinterpret_cast<cudaStream_t>(stream));
}

int bitnet_plan_linear(int M, int N, int K, int epilogue, int sms, int* out) {
  g_last_error.clear();
  if (out == nullptr) return fail(BITNET_ERR_INVALID_ARG, "out is NULL");
  if (M <= 0 || N <= 0 || sms <= 0)
    return fail(BITNET_ERR_INVALID_ARG, "M=%d, N=%d and sms=%d must be positive", M, N, sms);
  if (int rc = check_k(K)) return rc;
  const int ldw = (int)bitnet_packed_row_bytes(K);
  const int flags = epilogue & ~BITNET_EPI_TYPE_MASK;
  int o[5] = {0, 0, 0, 0, 0};
  const int tiles_n = (N + 127) / 128;
  int S = 0;
  if (takes_stream(M, N, K, ldw, flags)) {
    const StreamShape sh = stream_shape(M, N, K, ldw, flags, sms);
    o[0] = sh.flat ? BITNET_PLAN_FLAT : BITNET_PLAN_STREAM;
    o[1] = sh.mt;
    o[2] = sh.grid;
    o[3] = sh.flat ? sh.R : sh.L;
    o[4] = sh.flat ? (sh.bulk ? 1 : 0) : sh.warps;
  } else if (M <= 16 && (S = decode_cluster_size(M, K, tiles_n, flags, sms)) > 0) {
    o[0] = BITNET_PLAN_GEMV_TC;
    o[1] = kDecTokens;
    o[2] = tiles_n * S;
    o[3] = S;
    o[4] = tiles_n;
  } else if (M <= 16) {
    const int rows_per_cta = (kGemvThreads / 32) * kGemvRows;
    o[0] = BITNET_PLAN_GEMV;
    o[1] = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16;
    o[2] = (N + rows_per_cta - 1) / rows_per_cta;
  } else {
    const int bn = (flags & EPI_SILU) ? 128 : token_tile(M, N, sms);
    const int tiles = ((M + bn - 1) / bn) * tiles_n;
    o[0] = BITNET_PLAN_GEMM_TC;
    o[1] = bn;
    o[2] = tiles < sms ? tiles : sms;
    o[3] = tiles;
  }
  for (int k = 0; k < 5; ++k) out[k] = o[k];
  return BITNET_OK;
}

int bitnet_linear(const int8_t* Xq, const float* x_scale, const int32_t* x_rowsum,
                  const uint8_t* packed, const float* gamma, int M, int N, int K, void* Y,
                  int epilogue, const void* residual, bitnet_stream_t stream) {
  g_last_error.clear();
  if (int rc = validate_linear(Xq, x_scale, x_rowsum, packed, gamma, M, N, K, Y, epilogue,
                               residual))
    return rc;
  if (M == 0 || N == 0) return BITNET_OK;
  LinearParams p;
  p.Xq = Xq; p.xs = x_scale; p.xrs = x_rowsum; p.W = packed; p.gamma = gamma;
  p.M = M; p.N = N; p.K = K; p.ldw = (int)bitnet_packed_row_bytes(K);
  p.Y = Y; p.out_type = epilogue & BITNET_EPI_TYPE_MASK;
  p.flags = epilogue & ~BITNET_EPI_TYPE_MASK; p.resid = residual;
  if (p.flags & LAUNCH_PDL_INPUTS) p.flags |= LAUNCH_PDL;
  if (M > 16) {
    p.w_early = (p.flags & LAUNCH_PDL) ? 1 : 0;
    p.flags &= ~(LAUNCH_PDL | LAUNCH_PDL_INPUTS);
  }
  single_segment(p);
  return launch_linear(p, reinterpret_cast<cudaStream_t>(stream));
}

int bitnet_linear_multi(const int8_t* Xq, const float* x_scale, const int32_t* x_rowsum,
                        int count, const uint8_t* const* packed, const float* const* gamma,
                        const int* N, int M, int K, void* const* Y, int epilogue,
                        bitnet_stream_t stream) {
  g_last_error.clear();
  if (count < 1 || count > kMaxSegments)
    return fail(BITNET_ERR_INVALID_ARG, "count=%d must be in [1, %d]", count, kMaxSegments);
  if (packed == nullptr || gamma == nullptr || N == nullptr || Y == nullptr)
    return fail(BITNET_ERR_INVALID_ARG, "null pointer array");
  if (epilogue & BITNET_EPI_RESIDUAL)
    return fail(BITNET_ERR_UNSUPPORTED, "no residual for several projections");
  int total = 0;
  for (int i = 0; i < count; ++i) {
    if (N[i] < 1) return fail(BITNET_ERR_INVALID_ARG, "N[%d]=%d must be >= 1", i, N[i]);
    if (int rc = validate_linear(Xq, x_scale, x_rowsum, packed[i], gamma[i], M, N[i], K, Y[i],
                                 epilogue, nullptr))
      return rc;
    if (total > (1 << 30) - N[i]) return fail(BITNET_ERR_INVALID_ARG, "too many rows");
    total += N[i];
  }
  if (M == 0) return BITNET_OK;
  LinearParams p;
  p.Xq = Xq; p.xs = x_scale; p.xrs = x_rowsum; p.W = packed[0]; p.gamma = gamma[0];
  p.M = M; p.N = total; p.K = K; p.ldw = (int)bitnet_packed_row_bytes(K);
  p.Y = Y[0]; p.out_type = epilogue & BITNET_EPI_TYPE_MASK;
  p.flags = epilogue & ~BITNET_EPI_TYPE_MASK; p.resid = nullptr;
  if (p.flags & LAUNCH_PDL_INPUTS) p.flags |= LAUNCH_PDL;
  if (M > 16) p.flags &= ~(LAUNCH_PDL | LAUNCH_PDL_INPUTS);
  p.nseg = count;
  p.seg_row0[0] = 0;
  for (int i = 0; i < count; ++i) {
    p.seg_row0[i + 1] = p.seg_row0[i] + N[i];
    p.seg_W[i] = packed[i];
    p.seg_gamma[i] = gamma[i];
    p.seg_Y[i] = Y[i];
  }
  return launch_linear(p, reinterpret_cast<cudaStream_t>(stream));
}

size_t bitnet_ffn_workspace_size(int M, int H, int I, int variant) {
  if (M < 0 || H <= 0 || I <= 0) return 0;
  const size_t m = (size_t)M;
  size_t total = 0;
  total += align256(m * (size_t)H);            // codes of x
  total += align256(m * 4) * 2;                // scale and rowsum of x
  total += align256(m * (size_t)I * 4);        // fp32 hidden activation
  total += align256(m * (size_t)I);            // codes of the hidden activation
  total += align256(m * 4) * 2;                // its scale and rowsum
  // decode (M <= 16): the up projection's fp32 output (four-launch route),
  // and the persistent launch's per-CTA partial sums and exchange flags
  if ((variant & ~BITNET_FFN_SINGLE_LAUNCH) == BITNET_FFN_RELU2_GLU && M <= 16) {
    total += align256(m * (size_t)I * 4);
    total += align256(sizeof(FdControl));
  }
  return total;
}

int bitnet_ffn(const void* X, int x_dtype, int M, int H, int I, const uint8_t* W_gate,
               const float* gamma_gate, const uint8_t* W_up, const float* gamma_up,
               const uint8_t* W_down, const float* gamma_down, const float* pre_norm_gain,
               const float* sub_norm_gain, float eps, int variant, void* Y, int y_dtype,
               void* workspace, size_t ws_bytes, bitnet_stream_t stream) {
  g_last_error.clear();
  if (M < 0) return fail(BITNET_ERR_INVALID_ARG, "M=%d must be >= 0", M);
  if (int rc = check_k(H)) return rc;
  if (int rc = check_k(I)) return rc;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16)
    return fail(BITNET_ERR_INVALID_ARG, "x dtype must be F32 or BF16");
  if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16)
    return fail(BITNET_ERR_INVALID_ARG, "y dtype must be F32 or BF16");
  const bool single = (variant & BITNET_FFN_SINGLE_LAUNCH) != 0;
  const int variant_flags = variant;
  variant &= ~BITNET_FFN_SINGLE_LAUNCH;
  if (variant != BITNET_FFN_RELU2_GLU && variant != BITNET_FFN_HADAMARD_SILU)
    return fail(BITNET_ERR_INVALID_ARG, "unknown FFN variant %d", variant_flags);
  if (variant == BITNET_FFN_RELU2_GLU) {
    if (x_dtype != y_dtype)
      return fail(BITNET_ERR_UNSUPPORTED, "the residual FFN needs x and y of one dtype");
    if (!W_up || !gamma_up) return fail(BITNET_ERR_INVALID_ARG, "W_up / gamma_up missing");
    if (!(eps >= 0.0f && std::isfinite(eps)))
      return fail(BITNET_ERR_INVALID_ARG, "eps must be finite and >= 0");
  } else {
    if (W_up || gamma_up)
      return fail(BITNET_ERR_INVALID_ARG, "the Hadamard FFN has no up projection");
    if ((H & (H - 1)) || (I & (I - 1)))
      return fail(BITNET_ERR_INVALID_ARG, "H-BitLinear widths must be powers of two");
    if (pre_norm_gain || sub_norm_gain)
      return fail(BITNET_ERR_INVALID_ARG, "the Hadamard FFN takes no norm gains");
  }
  if (M == 0) return BITNET_OK;
  if (!X || !W_gate || !gamma_gate || !W_down || !gamma_down || !Y)
    return fail(BITNET_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(X) || !aligned16(Y) || !aligned16(W_gate) || !aligned16(W_down) ||
      !aligned16(gamma_gate) || !aligned16(gamma_down) || (W_up && !aligned16(W_up)) ||
      (gamma_up && !aligned16(gamma_up)) || (pre_norm_gain && !aligned16(pre_norm_gain)) ||
      (sub_norm_gain && !aligned16(sub_norm_gain)))
    return fail(BITNET_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = bitnet_ffn_workspace_size(M, H, I, variant);
  if (workspace == nullptr || ws_bytes < need)
    return fail(BITNET_ERR_WORKSPACE, "workspace of %zu bytes needed", need);
  if (!aligned16(workspace)) return fail(BITNET_ERR_INVALID_ARG, "workspace must be 16-byte aligned");

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t m = (size_t)M;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int8_t* xq = reinterpret_cast<int8_t*>(ws);            ws += align256(m * H);
  float* xs = reinterpret_cast<float*>(ws);              ws += align256(m * 4);
  int32_t* xrs = reinterpret_cast<int32_t*>(ws);         ws += align256(m * 4);
  float* hid = reinterpret_cast<float*>(ws);             ws += align256(m * I * 4);
  int8_t* hq = reinterpret_cast<int8_t*>(ws);            ws += align256(m * I);
  float* hs = reinterpret_cast<float*>(ws);              ws += align256(m * 4);
  int32_t* hrs = reinterpret_cast<int32_t*>(ws);         ws += align256(m * 4);
  float* hid_up = reinterpret_cast<float*>(ws);          // decode GLU only
  ws += align256(m * I * 4);
  FdControl* fd_ctl = reinterpret_cast<FdControl*>(ws);  // decode GLU only
  const bool xbf = x_dtype == BITNET_BF16;

  LinearParams p1;
  p1.Xq = xq; p1.xs = xs; p1.xrs = xrs; p1.W = W_gate; p1.gamma = gamma_gate;
  p1.M = M; p1.N = I; p1.K = H; p1.ldw = (int)bitnet_packed_row_bytes(H);
  p1.Y = hid; p1.out_type = OUT_F32; p1.resid = nullptr;
  LinearParams p2;
  p2.Xq = hq; p2.xs = hs; p2.xrs = hrs; p2.W = W_down; p2.gamma = gamma_down;
  p2.M = M; p2.N = H; p2.K = I; p2.ldw = (int)bitnet_packed_row_bytes(I);
  p2.Y = Y; p2.out_type = y_dtype == BITNET_BF16 ? OUT_BF16 : OUT_F32;
  // each GEMM below follows this call's own quantiser, which writes no
  // weights and lets it launch only after everything before it completed
  p1.w_early = 1;
  p2.w_early = 1;
  single_segment(p1);
  single_segment(p2);

  if (variant == BITNET_FFN_RELU2_GLU && M <= 16 && single) {
    // Decode: the whole FFN in one persistent launch when the shape fits it
    FfnDecodeParams fp = {};
    fp.X = X; fp.x_bf16 = xbf ? 1 : 0; fp.M = M; fp.H = H; fp.I = I;
    fp.Wg = W_gate; fp.Wu = W_up; fp.Wd = W_down;
    fp.gamma_g = gamma_gate; fp.gamma_u = gamma_up; fp.gamma_d = gamma_down;
    fp.pre_gain = pre_norm_gain; fp.sub_gain = sub_norm_gain; fp.eps = eps;
    fp.Y = Y; fp.y_bf16 = y_dtype == BITNET_BF16 ? 1 : 0;
    fp.hid = hid; fp.hq = hq; fp.hs = hs; fp.hrs = hrs;
    fp.ctl = fd_ctl;
    fp.ldwH = (int)bitnet_packed_row_bytes(H); fp.ldwI = (int)bitnet_packed_row_bytes(I);
    const int rc = launch_ffn_decode(fp, st);
    if (rc != BITNET_ERR_UNSUPPORTED) return rc;
  }
  if (variant == BITNET_FFN_RELU2_GLU && M <= 16) {
    // Decode: gate and up as two projections of one decode launch (fp32
    // outputs), relu(g)^2 * u formed by the sub-norm quantiser as it loads
    // them, the down projection with the residual.  Each launch after the
    // first streams its weights while its predecessor finishes (PDL).
    if (int rc = launch_quant(X, xbf, M, H, PRE_RMSNORM, pre_norm_gain, eps, xq, xs, xrs, st))
      return rc;
    p1.N = 2 * I;                              // rows of both projections
    p1.nseg = 2;
    p1.seg_row0[0] = 0; p1.seg_row0[1] = I; p1.seg_row0[2] = 2 * I;
    p1.seg_W[1] = W_up; p1.seg_gamma[1] = gamma_up; p1.seg_Y[1] = hid_up;
    // (each decode launch is followed by a quantiser: the early trigger lets
    // it be resident when the launch completes)
    p1.flags = LAUNCH_PDL | LAUNCH_TRIGGER_EARLY;
    if (int rc = launch_linear(p1, st)) return rc;
    if (int rc = launch_quant(hid, false, M, I, PRE_GLU_RMSNORM, sub_norm_gain, eps, hq, hs, hrs,
                              st, hid_up))
      return rc;
    p2.flags = EPI_RESIDUAL | LAUNCH_PDL | LAUNCH_TRIGGER_EARLY;
    p2.resid = X;
    return launch_linear(p2, st);
  }
  if (variant == BITNET_FFN_RELU2_GLU) {
    if (int rc = launch_quant(X, xbf, M, H, PRE_RMSNORM, pre_norm_gain, eps, xq, xs, xrs, st))
      return rc;
    p1.flags = 0;
    if (int rc = launch_tc_cfg<TcGlu>(p1, W_up, gamma_up, st)) return rc;
    if (int rc = launch_quant(hid, false, M, I, PRE_RMSNORM, sub_norm_gain, eps, hq, hs, hrs, st))
      return rc;
    p2.flags = EPI_RESIDUAL;
    p2.resid = X;
    return launch_linear(p2, st);
  }
  // H-BitLinear FFN: W1 writes its plain fp32 output; the second
  // quantiser applies the SiLU as it loads the hidden rows (the same fp32
  // operations the GEMM epilogue would apply, so the same values), then the
  // transform.
  if (int rc = launch_quant(X, xbf, M, H, PRE_FWHT, nullptr, 0.0f, xq, xs, xrs, st)) return rc;
  p1.flags = 0;
  if (int rc = launch_linear(p1, st)) return rc;
  if (int rc = launch_quant(hid, false, M, I, PRE_SILU_FWHT, nullptr, 0.0f, hq, hs, hrs, st))
    return rc;
  p2.flags = 0;
  p2.resid = nullptr;
  return launch_linear(p2, st);
}

size_t bitnet_block_tail_workspace_size(int M, int H, int I) {
  if (M < 0 || H <= 0 || I <= 0) return 0;
  const size_t m = (size_t)M;
  return align256(m * (size_t)I * 4) + align256(m * (size_t)I) + 2 * align256(m * 4) +
         align256(sizeof(FdControl)) + align256(m * (size_t)H * 4);
}

int bitnet_block_tail(const void* A, const void* X, int dtype, int M, int H, int I,
                      const uint8_t* W_o, const float* gamma_o, const uint8_t* W_gate,
                      const float* gamma_gate, const uint8_t* W_up, const float* gamma_up,
                      const uint8_t* W_down, const float* gamma_down, const float* attn_norm_gain,
                      const float* post_norm_gain, const float* sub_norm_gain, float eps,
                      void* H_out, void* Y, void* workspace, size_t ws_bytes,
                      bitnet_stream_t stream) {
  g_last_error.clear();
  if (M < 0) return fail(BITNET_ERR_INVALID_ARG, "M=%d must be >= 0", M);
  if (int rc = check_k(H)) return rc;
  if (int rc = check_k(I)) return rc;
  if (dtype != BITNET_F32 && dtype != BITNET_BF16)
    return fail(BITNET_ERR_INVALID_ARG, "dtype must be F32 or BF16");
  if (!(eps >= 0.0f && std::isfinite(eps)))
    return fail(BITNET_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (M == 0) return BITNET_OK;
  if (!A || !X || !W_o || !gamma_o || !W_gate || !gamma_gate || !W_up || !gamma_up || !W_down ||
      !gamma_down || !Y)
    return fail(BITNET_ERR_INVALID_ARG, "null pointer argument");
  const void* ptrs[] = {A, X, W_o, gamma_o, W_gate, gamma_gate, W_up, gamma_up, W_down,
                        gamma_down, Y, H_out, attn_norm_gain, post_norm_gain, sub_norm_gain};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return fail(BITNET_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (M > 16 || H % 128 != 0 || I % 128 != 0)
    return fail(BITNET_ERR_UNSUPPORTED,
                "the fused block tail runs at decode sizes (M <= 16, H and I multiples of 128); "
                "compose bitnet_quant_act, bitnet_linear and bitnet_ffn otherwise");
  const size_t need = bitnet_block_tail_workspace_size(M, H, I);
  if (workspace == nullptr || ws_bytes < need)
    return fail(BITNET_ERR_WORKSPACE, "workspace of %zu bytes needed", need);
  if (!aligned16(workspace)) return fail(BITNET_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  const size_t m = (size_t)M;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  FfnDecodeParams fp = {};
  fp.hid = reinterpret_cast<float*>(ws);                  ws += align256(m * I * 4);
  fp.hq = reinterpret_cast<int8_t*>(ws);                  ws += align256(m * I);
  fp.hs = reinterpret_cast<float*>(ws);                   ws += align256(m * 4);
  fp.hrs = reinterpret_cast<int32_t*>(ws);                ws += align256(m * 4);
  fp.ctl = reinterpret_cast<FdControl*>(ws);              ws += align256(sizeof(FdControl));
  fp.hbuf = reinterpret_cast<float*>(ws);
  fp.X = X; fp.A = A; fp.x_bf16 = dtype == BITNET_BF16 ? 1 : 0;
  fp.M = M; fp.H = H; fp.I = I;
  fp.Wo = W_o; fp.gamma_o = gamma_o;
  fp.Wg = W_gate; fp.Wu = W_up; fp.Wd = W_down;
  fp.gamma_g = gamma_gate; fp.gamma_u = gamma_up; fp.gamma_d = gamma_down;
  fp.attn_gain = attn_norm_gain; fp.pre_gain = post_norm_gain; fp.sub_gain = sub_norm_gain;
  fp.eps = eps; fp.Y = Y; fp.H_out = H_out; fp.y_bf16 = fp.x_bf16;
  fp.ldwH = (int)bitnet_packed_row_bytes(H); fp.ldwI = (int)bitnet_packed_row_bytes(I);
  const int rc = launch_ffn_decode(fp, reinterpret_cast<cudaStream_t>(stream), true);
  if (rc == BITNET_ERR_UNSUPPORTED)
    return fail(BITNET_ERR_UNSUPPORTED, "staged weights and codes exceed shared memory "
                "(M=%d, H=%d, I=%d)", M, H, I);
  return rc;
}

const char* bitnet_last_error(void) { return g_last_error.c_str(); }

int bitnet_check_device_error(bitnet_stream_t stream) {
  g_last_error.clear();
  BN_CHECK_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  unsigned int word = 0, zero = 0;
  BN_CHECK_CUDA(cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word)));
  if (word != 0) {
    BN_CHECK_CUDA(cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)));
    if (word & DEV_ERR_TIMEOUT)
      return fail(BITNET_ERR_TIMEOUT, "a bounded device-side wait gave up (error word 0x%x)", word);
    return fail(BITNET_ERR_CUDA, "device error word 0x%x", word);
  }
  return BITNET_OK;
}

void bitnet_release_cache(void) {
  {
    std::lock_guard<std::mutex> lock(g_map_mu);
    g_map_cache.clear();
  }
  // per-context state: looked up / set again on the next call
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    for (int d = 0; d < kMaxDevices; ++d) g_noalloc_ptr[d] = nullptr;
  }
  g_dec_attr_set.store(0, std::memory_order_release);
  {
    std::lock_guard<std::mutex> lock(g_attr_mu);
    g_smem_set.clear();
    g_occupancy.clear();
  }
}

const char* bitnet_version(void) { return "bitnet-b200 0.1.0 (sm_100a)"; }

}  // extern "C"

// The timeout diagnostic lives below the C ABI block so it can use the
// kernel-side wait helper directly.
namespace bitnet {
__device__ int g_wait_probe_result = 0;

__global__ void wait_timeout_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // Nobody ever arrives on `bar`: the bounded wait must give up.
  const bool done = mbar_wait(&bar, 0, &abort_flag, limit_ns);
  if (threadIdx.x == 0) g_wait_probe_result = done ? 1 : 0;
}
}  // namespace bitnet

extern "C" int bitnet_debug_wait_timeout(unsigned timeout_us, bitnet_stream_t stream) {
  g_last_error.clear();
  if (timeout_us < 1 || timeout_us > 1000000)
    return fail(BITNET_ERR_INVALID_ARG, "timeout_us must be in [1, 1000000]");
  wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)timeout_us * 1000ull);
  BN_CHECK_CUDA(cudaGetLastError());
  return BITNET_OK;
}

// ------------------------------------------------------------------------
// FFN without a workspace argument (bitnet_ffn_noalloc): the scratch is this
// file-scope device array.  In host code `g_ffn_noalloc_scratch` is only a
// host-side stand-in for the symbol, never a device address, so its device
// address is looked up with cudaGetSymbolAddress once per device (with that
// device current) and passed on as the workspace pointer.
namespace bitnet {
static __device__ __align__(256) uint8_t g_ffn_noalloc_scratch[BITNET_FFN_NOALLOC_SCRATCH_BYTES];


int noalloc_scratch(void** out) {
  int dev = 0;
  BN_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices)
    return fail(BITNET_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_ffn_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(BITNET_ERR_CUDA, "cudaGetSymbolAddress of the FFN scratch failed: %s",
                  cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return BITNET_OK;
}
}  // namespace bitnet

extern "C" int bitnet_ffn_noalloc(const void* X, int x_dtype, int M, int H, int I,
                                  const uint8_t* W_gate, const float* gamma_gate,
                                  const uint8_t* W_up, const float* gamma_up,
                                  const uint8_t* W_down, const float* gamma_down,
                                  const float* pre_norm_gain, const float* sub_norm_gain,
                                  float eps, int variant, void* Y, int y_dtype,
                                  bitnet_stream_t stream) {
  g_last_error.clear();
  const size_t need = bitnet_ffn_workspace_size(M, H, I, variant);
  if (need > (size_t)BITNET_FFN_NOALLOC_SCRATCH_BYTES)
    return fail(BITNET_ERR_WORKSPACE,
                "M=%d, H=%d, I=%d needs %zu bytes of scratch; the built-in scratch holds %u "
                "(use bitnet_ffn with a workspace)",
                M, H, I, need, (unsigned)BITNET_FFN_NOALLOC_SCRATCH_BYTES);
  if (M <= 0)   // nothing to launch; bitnet_ffn validates the arguments
    return bitnet_ffn(X, x_dtype, M, H, I, W_gate, gamma_gate, W_up, gamma_up, W_down,
                      gamma_down, pre_norm_gain, sub_norm_gain, eps, variant, Y, y_dtype,
                      nullptr, 0, stream);
  void* scratch = nullptr;
  if (int rc = noalloc_scratch(&scratch)) return rc;
  return bitnet_ffn(X, x_dtype, M, H, I, W_gate, gamma_gate, W_up, gamma_up, W_down, gamma_down,
                    pre_norm_gain, sub_norm_gain, eps, variant, Y, y_dtype, scratch,
                    (size_t)BITNET_FFN_NOALLOC_SCRATCH_BYTES, stream);
}
