// flashnorm.cu — the C ABI (include/flashnorm.h): argument validation, tile selection, TMA tensor maps
// and kernel launches for the FlashNorm path on sm_100a. Every computation happens in the kernels of
// fused_gemm.cuh, gemv.cuh and elementwise.cuh; this file only checks, plans and enqueues.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>

#include "../../include/flashnorm.h"
#include "decode_fp8.cuh"
#include "decode_tc.cuh"
#include "elementwise.cuh"
#include "fused_gemm.cuh"
#include "fp8.cuh"
#include "fused_gemm_pair.cuh"
#include "gemv.cuh"
#include "postnorm_pair.cuh"
#include "postnorm_split.cuh"

namespace {

thread_local char g_last_error[512] = "";

fn_status fail(fn_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

fn_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FN_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;

int device_sm_count(int* dev_out) {
  static int sms[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  if (sms[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    sms[dev] = v;
  }
  *dev_out = dev;
  return sms[dev];
}

// Every kernel is launched with programmatic stream serialization: it may be scheduled while the
// previous kernel of the stream drains, runs its prologue (barriers, tensor memory), and then waits in
// the kernel (griddepcontrol.wait) for that kernel's completion before it touches global memory.
// cluster > 1 adds a cluster dimension.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          unsigned cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda dependency).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn_ptr = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn_ptr = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn_ptr;
}

// An encoded tensor map is a pure function of its arguments, so calls that pass the same buffer with the
// same geometry reuse the previous encoding: a small per-thread cache keyed on every argument (a buffer
// freed and allocated again at the same address with the same geometry gets a map that is still right).
struct MapKey {
  void* ptr;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3];
  int dtype, rank, swizzle, promo;
};
constexpr int kMapCacheSlots = 64;
struct MapCacheEntry {
  MapKey key;
  CUtensorMap map;
  bool valid;
};

CUresult encode_cached(CUtensorMap* map, CUtensorMapDataType dtype, int rank, void* ptr, const cuuint64_t* dims,
                       const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swizzle,
                       CUtensorMapL2promotion promo) {
  MapKey k;
  std::memset(&k, 0, sizeof(k));  // padding included: the key is compared byte for byte
  k.ptr = ptr;
  for (int i = 0; i < rank; ++i) k.dims[i] = dims[i], k.box[i] = box[i];
  for (int i = 0; i + 1 < rank; ++i) k.strides[i] = strides[i];
  k.dtype = static_cast<int>(dtype);
  k.rank = rank;
  k.swizzle = static_cast<int>(swizzle);
  k.promo = static_cast<int>(promo);
  uint64_t h = 1469598103934665603ull;  // FNV-1a over the key's bytes
  const unsigned char* b = reinterpret_cast<const unsigned char*>(&k);
  for (size_t i = 0; i < sizeof(k); ++i) h = (h ^ b[i]) * 1099511628211ull;
  thread_local MapCacheEntry cache[kMapCacheSlots];
  MapCacheEntry& e = cache[h % kMapCacheSlots];
  if (e.valid && std::memcmp(&e.key, &k, sizeof(k)) == 0) {
    *map = e.map;
    return CUDA_SUCCESS;
  }
  EncodeTiledFn enc = encode_fn();
  if (!enc) return CUDA_ERROR_NOT_FOUND;
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, dtype, static_cast<cuuint32_t>(rank), ptr, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r == CUDA_SUCCESS) {
    e.key = k;
    e.map = *map;
    e.valid = true;
  }
  return r;
}

// 2-D bf16 K-major operand [rows, k] with a (64 x box_rows) box and 128-byte swizzle.
fn_status make_operand_map(CUtensorMap* map, const void* ptr, int64_t k, int64_t rows, int box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(k) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(fn::kBK), static_cast<cuuint32_t>(box_rows)};
  CUresult r = encode_cached(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
                             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
  if (r == CUDA_ERROR_NOT_FOUND) return fail(FN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (r != CUDA_SUCCESS) return fail(FN_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return FN_OK;
}

// 2-D one-byte operand [rows, k] (FP8 E4M3 codes) with a (128 x box_rows) box and 128-byte swizzle.
fn_status make_u8_map(CUtensorMap* map, const void* ptr, int64_t k, int64_t rows, int box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(k)};
  cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  CUresult r = encode_cached(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
                             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
  if (r == CUDA_ERROR_NOT_FOUND) return fail(FN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (r != CUDA_SUCCESS) return fail(FN_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return FN_OK;
}

// NVFP4 W* [rows][groups x 144 bytes] (fp8.cuh's storage): one 144-byte group of 128 rows per box, no
// swizzle (the converters' reads of 144-byte rows fall on distinct banks as they are).
fn_status make_q4_map(CUtensorMap* map, const void* ptr, int64_t row_bytes, int64_t rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(fn::kNvfp4GroupBytes), static_cast<cuuint32_t>(fn::kD8Rows)};
  CUresult r = encode_cached(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
                             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
  if (r == CUDA_ERROR_NOT_FOUND) return fail(FN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (r != CUDA_SUCCESS) return fail(FN_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return FN_OK;
}

// 3-D fp32 [planes][rows][cols] (the split post-norm's partial products) with a 32-column x 128-row box
// and 128-byte swizzle, for TMA stores.
fn_status make_partial_map(CUtensorMap* map, void* ptr, int64_t cols, int64_t rows, int64_t planes) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 4, static_cast<cuuint64_t>(cols * rows) * 4};
  cuuint32_t box[3] = {32u, 128u, 1u};
  CUresult r = encode_cached(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box,
                             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE);
  if (r == CUDA_ERROR_NOT_FOUND) return fail(FN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (r != CUDA_SUCCESS) return fail(FN_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return FN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fn_status check_ptr(const void* p, const char* name) {
  if (p == nullptr) return fail(FN_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(FN_ERR_ALIGN, "%s is not 16-byte aligned", name);
  return FN_OK;
}

constexpr int64_t kMaxDim = (int64_t{1} << 31) - 1;

fn_status check_common(const void* x, const void* w, const void* y, int64_t M, int64_t d, float eps, int out_dtype) {
  if (M < 0 || M > kMaxDim) return fail(FN_ERR_INVALID_ARG, "M = %lld out of range", (long long)M);
  if (d < 8 || d > kMaxDim || d % 8 != 0)
    return fail(FN_ERR_INVALID_ARG, "d = %lld must be a positive multiple of 8", (long long)d);
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return fail(FN_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (out_dtype != FN_BF16 && out_dtype != FN_F32) return fail(FN_ERR_INVALID_ARG, "out_dtype %d unknown", out_dtype);
  fn_status st;
  if (M > 0) {
    if ((st = check_ptr(x, "x")) != FN_OK) return st;
    if ((st = check_ptr(y, "y")) != FN_OK) return st;
  }
  if ((st = check_ptr(w, "W*")) != FN_OK) return st;
  return FN_OK;
}

// ------------------------------------------------------------------------------------------------
// Tensor-core path
// ------------------------------------------------------------------------------------------------

// Accumulator width: fewest waves of tiles over the SMs, weighted by the tile width plus a fixed
// per-tile cost (the x tile and the epilogue do not shrink with bn).
int choose_bn(int64_t M, int64_t n_rows, int sms, int step) {
  const int64_t m_tiles = (M + fn::kBM - 1) / fn::kBM;
  const int64_t n_cap = ((n_rows + step - 1) / step) * step;
  const int top = n_cap < 256 ? static_cast<int>(n_cap) : 256;
  int best = top;
  int64_t best_cost = INT64_MAX;
  for (int bn = top; bn >= step && (bn >= 64 || bn == top); bn -= step) {
    const int64_t tiles = m_tiles * ((n_rows + bn - 1) / bn);
    const int64_t waves = (tiles + sms - 1) / sms;
    const int64_t cost = waves * (bn + 64);
    if (cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

template <int MAX_BN, int STAGES, int EPI, bool SCALE, bool OUT_F32>
fn_status launch_gemm_t(const CUtensorMap& tx, const CUtensorMap& tw, const fn::GemmParams& p, int sms, int dev,
                        cudaStream_t stream) {
  auto kern = fn::k_fused_gemm<MAX_BN, STAGES, EPI, SCALE, OUT_F32>;
  constexpr int smem = fn::gemm_smem_bytes<MAX_BN, STAGES>();
  static bool configured[kMaxDevices] = {false};
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    configured[dev] = true;
  }
  const int tiles = p.num_m_tiles * p.num_n_tiles;
  const int grid = tiles < sms ? tiles : sms;
  cudaError_t e = launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(fn::gemm_threads(EPI, SCALE)), smem,
                                stream, 1, tx, tw, p);
  if (e != cudaSuccess) return cuda_fail(e, "fused GEMM launch");
  return FN_OK;
}

// ---- CTA-pair (2-SM MMA) variant ------------------------------------------------------------------

template <int STAGES, int EPI, bool SCALE, bool OUT_F32>
fn_status launch_gemm_pair_t(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& tw2,
                             const fn::GemmParams& p, int sms, int dev, cudaStream_t stream) {
  auto kern = fn::k_fused_gemm_pair<STAGES, EPI, SCALE, OUT_F32>;
  constexpr int smem = fn::gemm_pair_smem_bytes<STAGES>();
  static bool configured[kMaxDevices] = {false};
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (pair GEMM)");
    configured[dev] = true;
  }
  const int tiles = p.num_m_tiles * p.num_n_tiles;
  const int pairs = tiles < sms / 2 ? tiles : sms / 2;
  cudaError_t e = launch_kernel(kern, dim3(static_cast<unsigned>(2 * pairs)), dim3(fn::gemm_threads(EPI, SCALE)),
                                smem, stream, 2, tx, tw, tw2, p);
  if (e != cudaSuccess) return cuda_fail(e, "pair GEMM launch");
  return FN_OK;
}

fn_status run_pair_path(const void* x, const void* w, void* y, int64_t M, int64_t d, int64_t n_rows, int64_t n_out,
                        float eps, int out_dtype, int epi, bool scale, cudaStream_t stream,
                        const float* ln_colsum = nullptr, const float* ln_bias = nullptr) {
  int dev = 0;
  const int sms = device_sm_count(&dev);
  if (sms <= 1) return fail(FN_ERR_CUDA, "cannot query the current device");
  // Pair tiles are 256 rows; the choice of width counts pairs of SMs. A tile's output columns are a
  // whole number of the epilogue's 64-byte chunks (32 bf16 outputs, i.e. 64 W* rows for the GLU).
  const int step = epi == fn::EPI_GLU ? 2 * fn::pair_chunk_cols(out_dtype == FN_F32) : 32;
  const int bn = choose_bn((M + 1) / 2, n_rows, sms / 2, step);
  const int64_t num_m_tiles = (M + 2 * fn::kBM - 1) / (2 * fn::kBM);
  const int64_t num_n_tiles = (n_rows + bn - 1) / bn;
  const int64_t tiles = num_m_tiles * num_n_tiles;
  const int64_t pairs = tiles < sms / 2 ? tiles : sms / 2;
  // Pairs in groups of two sharing each W* tile (L2 reuse) when there are several waves to run and the
  // row blocks and pairs pair up evenly.
  const int group = (tiles > pairs && num_m_tiles % 2 == 0 && pairs % 2 == 0) ? 2 : 1;
  const int64_t gtiles = tiles / group, groups = pairs / group;
  // A last wave that fills at most half of the groups is run as half tiles, one per group.
  int64_t num_main = gtiles;
  const int64_t rem = gtiles % groups;
  if (gtiles > groups && rem > 0 && 2 * rem <= groups && (bn / 2) % step == 0) num_main = gtiles - rem;
  CUtensorMap tx, tw, tw2;
  fn_status st = make_operand_map(&tx, x, d, M, fn::kBM);
  if (st != FN_OK) return st;
  st = make_operand_map(&tw, w, d, n_rows, bn / 2);
  if (st != FN_OK) return st;
  st = make_operand_map(&tw2, w, d, n_rows, num_main < gtiles ? bn / 4 : bn / 2);
  if (st != FN_OK) return st;
  fn::GemmParams p;
  p.y = y;
  p.g2 = nullptr;
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(d);
  p.n_out = static_cast<int>(n_out);
  p.ldy = static_cast<int>(n_out);
  p.bn = bn;
  p.head_dim = 0;
  p.num_m_tiles = static_cast<int>(num_m_tiles);
  p.num_n_tiles = static_cast<int>(num_n_tiles);
  p.group = group;
  p.num_main = static_cast<int>(num_main);
  p.eps = eps;
  p.ln_colsum = ln_colsum;
  p.ln_bias = ln_bias;
  const bool f32 = out_dtype == FN_F32;
#define FN_PAIR(EPI, SC)                                                                                        \
  (f32 ? launch_gemm_pair_t<fn::kPairStages, EPI, SC, true>(tx, tw, tw2, p, sms, dev, stream)                  \
       : launch_gemm_pair_t<fn::kPairStages, EPI, SC, false>(tx, tw, tw2, p, sms, dev, stream))
  if (epi == fn::EPI_LINEAR) return scale ? FN_PAIR(fn::EPI_LINEAR, true) : FN_PAIR(fn::EPI_LINEAR, false);
  if (epi == fn::EPI_LN) return FN_PAIR(fn::EPI_LN, true);
  return scale ? FN_PAIR(fn::EPI_GLU, true) : FN_PAIR(fn::EPI_GLU, false);
#undef FN_PAIR
}

// RoPE applied by the post-norm epilogue (see flashnorm_linear_postnorm_rope).
struct RopeArgs {
  const float* cs;
  const int* positions;
  int n_rope_heads;
  int max_pos;
};

// epi: fn::EpiKind; scale: apply the deferred 1/rms (sum of squares warpgroup on).
fn_status run_tensor_path(const void* x, const void* w, void* y, const void* g2, int64_t M, int64_t d,
                          int64_t n_rows, int64_t n_out, int64_t head_dim, float eps, int out_dtype, int epi,
                          bool scale, cudaStream_t stream, const RopeArgs* rope = nullptr) {
  int dev = 0;
  const int sms = device_sm_count(&dev);
  if (sms <= 0) return fail(FN_ERR_CUDA, "cannot query the current device");
  int bn;
  if (epi == fn::EPI_POSTNORM) {
    bn = head_dim <= 256 ? static_cast<int>((256 / head_dim) * head_dim) : static_cast<int>(head_dim);
    if (bn > n_rows) bn = static_cast<int>(n_rows);  // n_rows is a multiple of head_dim
  } else {
    bn = choose_bn(M, n_rows, sms, epi == fn::EPI_GLU ? 32 : 16);
  }
  CUtensorMap tx, tw;
  fn_status st = make_operand_map(&tx, x, d, M, fn::kBM);
  if (st != FN_OK) return st;
  st = make_operand_map(&tw, w, d, n_rows, bn <= 256 ? bn : bn / 2);
  if (st != FN_OK) return st;

  fn::GemmParams p;
  p.y = y;
  p.g2 = static_cast<const uint16_t*>(g2);
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(d);
  p.n_out = static_cast<int>(n_out);
  p.ldy = static_cast<int>(n_out);
  p.bn = bn;
  p.head_dim = static_cast<int>(head_dim);
  p.num_m_tiles = static_cast<int>((M + fn::kBM - 1) / fn::kBM);
  p.num_n_tiles = static_cast<int>((n_rows + bn - 1) / bn);
  p.eps = eps;
  if (rope != nullptr) {
    p.rope_cs = rope->cs;
    p.positions = rope->positions;
    p.n_rope_heads = rope->n_rope_heads;
    p.max_pos = rope->max_pos;
  }
  const bool f32 = out_dtype == FN_F32;

#define FN_LAUNCH(MAXBN, ST, EPI, SC)                                                        \
  (f32 ? launch_gemm_t<MAXBN, ST, EPI, SC, true>(tx, tw, p, sms, dev, stream)               \
       : launch_gemm_t<MAXBN, ST, EPI, SC, false>(tx, tw, p, sms, dev, stream))
  if (epi == fn::EPI_LINEAR) return scale ? FN_LAUNCH(256, 4, fn::EPI_LINEAR, true) : FN_LAUNCH(256, 4, fn::EPI_LINEAR, false);
  if (epi == fn::EPI_GLU) return scale ? FN_LAUNCH(256, 4, fn::EPI_GLU, true) : FN_LAUNCH(256, 4, fn::EPI_GLU, false);
  if (bn <= 256) return FN_LAUNCH(256, 4, fn::EPI_POSTNORM, false);
  return FN_LAUNCH(512, 2, fn::EPI_POSTNORM, false);
#undef FN_LAUNCH
}

// ------------------------------------------------------------------------------------------------
// Wide-head post-norm on CTA pairs: one cluster of 2 x 2 x KS CTAs per 256-row tile and head
// ------------------------------------------------------------------------------------------------

// Clusters of `csize` CTAs of the wide-head kernel that can be resident at once on this device.
template <bool OUT_F32>
int postnorm_pair_max_clusters(int csize, int dev) {
  static int cache[kMaxDevices][fn::kPpMaxKS + 1] = {{0}};
  const int slot = csize / (2 * fn::kPpNP);  // K ranges per cluster
  if (cache[dev][slot] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(csize));
    cfg.blockDim = dim3(fn::kPpThreads);
    cfg.dynamicSmemBytes = fn::postnorm_pair_smem_bytes();
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = static_cast<unsigned>(csize);
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn::k_postnorm_pair<OUT_F32>, &cfg) != cudaSuccess || n < 0) {
      (void)cudaGetLastError();
      n = 0;
    }
    cache[dev][slot] = n > 0 ? n : -1;  // -1: this cluster size cannot run
  }
  return cache[dev][slot];
}

template <bool OUT_F32>
fn_status run_postnorm_pair_t(const void* x, const void* w, const void* g2, void* y, int64_t M, int64_t d, int64_t N,
                              int64_t head_dim, float eps2, cudaStream_t stream) {
  int dev = 0;
  const int sms = device_sm_count(&dev);
  if (sms <= 0) return fail(FN_ERR_CUDA, "cannot query the current device");
  auto kern = fn::k_postnorm_pair<OUT_F32>;
  constexpr int smem = fn::postnorm_pair_smem_bytes();
  static bool configured[kMaxDevices] = {false};
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (wide-head post-norm)");
    configured[dev] = true;
  }
  fn::PostnormPairParams p;
  p.y = y;
  p.g2 = static_cast<const uint16_t*>(g2);
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(d);
  p.N = static_cast<int>(N);
  p.head_dim = static_cast<int>(head_dim);
  p.num_m_tiles = static_cast<int>((M + 255) / 256);
  p.eps2 = eps2;
  const int64_t clusters = p.num_m_tiles * (N / head_dim);
  const int64_t num_kb = (d + 63) / 64;
  const int64_t nw = head_dim / 2;
  // K ranges per cluster: the split with the fewest (waves x k-blocks per range + a fixed cost of about
  // six k-blocks for the pipeline fill, the reduce-scatter and the stores), among those whose K ranges
  // are not empty and whose slices are at least one 16-column chunk wide. Clusters of 12 (KS = 3) and 16
  // are non-portable sizes; on a B200 at most 7 clusters of 16 are resident at once.
  int best_ks = 0;
  int64_t best_cost = INT64_MAX;
  for (int ks = fn::kPpMaxKS; ks >= 1; --ks) {
    if (nw / ks < 16 || ks > num_kb) continue;
    const int maxc = postnorm_pair_max_clusters<OUT_F32>(2 * fn::kPpNP * ks, dev);
    if (maxc <= 0) continue;
    const int64_t waves = (clusters + maxc - 1) / maxc;
    const int64_t cost = waves * ((num_kb + ks - 1) / ks + 6);
    if (cost < best_cost) {
      best_cost = cost;
      best_ks = ks;
    }
  }
  if (best_ks == 0) return fail(FN_ERR_UNSUPPORTED, "no cluster shape of the wide-head kernel can run on this device");
  p.ks = best_ks;
  const int64_t ctas = clusters * 2 * fn::kPpNP * best_ks;
  if (ctas > INT32_MAX) return fail(FN_ERR_UNSUPPORTED, "too many tiles");
  CUtensorMap tx, tw;
  fn_status st = make_operand_map(&tx, x, d, M, 128);
  if (st != FN_OK) return st;
  st = make_operand_map(&tw, w, d, N, static_cast<int>(head_dim / 4));
  if (st != FN_OK) return st;
  cudaError_t e = launch_kernel(kern, dim3(static_cast<unsigned>(ctas)), dim3(fn::kPpThreads), smem, stream,
                                static_cast<unsigned>(2 * fn::kPpNP * best_ks), tx, tw, p);
  if (e != cudaSuccess) return cuda_fail(e, "wide-head post-norm launch");
  return FN_OK;
}

fn_status run_postnorm_pair(const void* x, const void* w, const void* g2, void* y, int64_t M, int64_t d, int64_t N,
                            int64_t head_dim, float eps2, int out_dtype, cudaStream_t stream) {
  return out_dtype == FN_F32 ? run_postnorm_pair_t<true>(x, w, g2, y, M, d, N, head_dim, eps2, stream)
                             : run_postnorm_pair_t<false>(x, w, g2, y, M, d, N, head_dim, eps2, stream);
}

// ------------------------------------------------------------------------------------------------
// Wide-head post-norm with the contraction split over independent CTA pairs (workspace) + finalize
// ------------------------------------------------------------------------------------------------

// CTA pairs of the split GEMM that can be resident at once on this device.
int postnorm_split_max_pairs(int dev) {
  static int cache[kMaxDevices] = {0};
  if (cache[dev] == 0) {
    cudaError_t e = cudaFuncSetAttribute(fn::k_postnorm_split_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         fn::postnorm_split_smem_bytes());
    int n = 0;
    if (e == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2);
      cfg.blockDim = dim3(fn::kPsThreads);
      cfg.dynamicSmemBytes = fn::postnorm_split_smem_bytes();
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 2;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      e = cudaOccupancyMaxActiveClusters(&n, fn::k_postnorm_split_gemm, &cfg);
    }
    if (e != cudaSuccess || n < 0) {
      (void)cudaGetLastError();
      n = 0;
    }
    cache[dev] = n > 0 ? n : -1;
  }
  return cache[dev];
}

// K ranges of the split kernel for this shape: as many as keep all CTA pairs in one wave (at most
// kPsMaxKS, each range at least four 64-deep k-blocks). 0 where fewer than two fit: there the cluster
// kernel, which keeps its partial sums on chip, has enough row tiles to fill the device by itself. Also 0
// for heads that are not a multiple of 64 wide (the cluster kernel takes those).
int postnorm_split_ks(int64_t M, int64_t d, int64_t N, int64_t head_dim) {
  // the partial product leaves in 32-column boxes: each pair's head_dim / 2 columns must fill whole boxes
  if (head_dim <= 256 || head_dim % 64 != 0 || M <= 0) return 0;
  int dev = 0;
  if (device_sm_count(&dev) <= 0) return 0;
  const int max_pairs = postnorm_split_max_pairs(dev);
  if (max_pairs <= 0) return 0;
  const int64_t pairs_per_range = ((M + 255) / 256) * (N / head_dim) * 2;
  const int64_t num_kb = (d + 63) / 64;
  int64_t ks = max_pairs / pairs_per_range;
  if (ks > fn::kPsMaxKS) ks = fn::kPsMaxKS;
  while (ks > 1 && num_kb < 4 * ks) --ks;
  return ks >= 2 ? static_cast<int>(ks) : 0;
}

fn_status run_postnorm_split(const void* x, const void* w, const void* g2, void* y, int64_t M, int64_t d, int64_t N,
                             int64_t head_dim, float eps2, int out_dtype, int ks, void* ws, cudaStream_t stream) {
  int dev = 0;
  const int sms = device_sm_count(&dev);
  if (sms <= 0) return fail(FN_ERR_CUDA, "cannot query the current device");
  fn::PostnormSplitParams p;
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(d);
  p.N = static_cast<int>(N);
  p.head_dim = static_cast<int>(head_dim);
  p.num_m_tiles = static_cast<int>((M + 255) / 256);
  p.heads = static_cast<int>(N / head_dim);
  p.ks = ks;
  const int64_t ctas = static_cast<int64_t>(p.num_m_tiles) * p.heads * 2 * ks * 2;
  if (ctas > INT32_MAX) return fail(FN_ERR_UNSUPPORTED, "too many tiles");
  CUtensorMap tx, tw;
  fn_status st = make_operand_map(&tx, x, d, M, 128);
  if (st != FN_OK) return st;
  st = make_operand_map(&tw, w, d, N, static_cast<int>(head_dim / 4));
  if (st != FN_OK) return st;
  CUtensorMap tws;
  st = make_partial_map(&tws, ws, N, M, ks);
  if (st != FN_OK) return st;
  // the attribute was set when the occupancy was queried (postnorm_split_max_pairs)
  cudaError_t e = launch_kernel(fn::k_postnorm_split_gemm, dim3(static_cast<unsigned>(ctas)), dim3(fn::kPsThreads),
                                fn::postnorm_split_smem_bytes(), stream, 2u, tx, tw, tws, p);
  if (e != cudaSuccess) return cuda_fail(e, "wide-head split GEMM launch");
  fn::PostnormFinalizeParams f;
  f.ws = static_cast<const float*>(ws);
  f.g2 = static_cast<const uint16_t*>(g2);
  f.y = y;
  f.M = p.M;
  f.N = p.N;
  f.head_dim = p.head_dim;
  f.heads = p.heads;
  f.ks = ks;
  f.eps2 = eps2;
  const int64_t items = M * p.heads;
  int64_t blocks = (items + fn::kPfWarps - 1) / fn::kPfWarps;
  if (blocks > 8LL * sms) blocks = 8LL * sms;
  const dim3 fgrid(static_cast<unsigned>(blocks)), fblock(fn::kPfWarps * 32);
#define FN_FIN(KS)                                                                                    \
  case KS:                                                                                            \
    e = out_dtype == FN_F32 ? launch_kernel(fn::k_postnorm_finalize<KS, true>, fgrid, fblock, 0, stream, 1u, f) \
                            : launch_kernel(fn::k_postnorm_finalize<KS, false>, fgrid, fblock, 0, stream, 1u, f); \
    break
  switch (ks) {
    FN_FIN(2);
    FN_FIN(3);
    FN_FIN(4);
    FN_FIN(5);
    FN_FIN(6);
    FN_FIN(7);
    FN_FIN(8);
    default:
      return fail(FN_ERR_UNSUPPORTED, "split post-norm with %d K ranges", ks);
  }
#undef FN_FIN
  if (e != cudaSuccess) return cuda_fail(e, "wide-head post-norm finalize launch");
  return FN_OK;
}

// ------------------------------------------------------------------------------------------------
// GEMV (decode) path
// ------------------------------------------------------------------------------------------------

template <int MT, int R, bool GLU, bool OUT_F32>
fn_status launch_gemv_t(const void* x, const void* w, void* y, int64_t M, int64_t d, int64_t n_units, float eps,
                        int sms, int dev, cudaStream_t stream) {
  auto kern = fn::k_gemv<MT, R, GLU, OUT_F32>;
  const int smem = fn::gemv_smem_bytes<MT>(static_cast<int>(d));
  static int configured[kMaxDevices] = {0};
  if (smem > 48 * 1024 && configured[dev] < smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (gemv)");
    configured[dev] = smem;
  }
  const int64_t groups = (n_units + R - 1) / R;
  const int64_t blocks_needed = (groups + 7) / 8;
  int per_sm = (228 * 1024) / (smem + 1024);
  if (per_sm > 8) per_sm = 8;
  if (per_sm < 1) per_sm = 1;
  int64_t grid = static_cast<int64_t>(sms) * per_sm;
  if (blocks_needed < grid) grid = blocks_needed;
  cudaError_t e = launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(fn::kGemvThreads),
                                static_cast<size_t>(smem), stream, 1, static_cast<const uint16_t*>(x),
                                static_cast<const uint16_t*>(w), y, static_cast<int>(M), static_cast<int>(d),
                                static_cast<int>(n_units), static_cast<int>(n_units), eps);
  if (e != cudaSuccess) return cuda_fail(e, "GEMV launch");
  return FN_OK;
}

constexpr int kGemvSmemLimit = 227 * 1024;

int gemv_mt(int64_t M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

bool gemv_fits(int64_t M, int64_t d) {
  return static_cast<int64_t>(gemv_mt(M)) * d * 2 + 64 <= kGemvSmemLimit;
}

fn_status run_gemv(const void* x, const void* w, void* y, int64_t M, int64_t d, int64_t n_units, float eps,
                   int out_dtype, bool glu, cudaStream_t stream) {
  int dev = 0;
  const int sms = device_sm_count(&dev);
  if (sms <= 0) return fail(FN_ERR_CUDA, "cannot query the current device");
  const bool f32 = out_dtype == FN_F32;
  const int mt = gemv_mt(M);
#define FN_GEMV(MT, R)                                                                                       \
  (glu ? (f32 ? launch_gemv_t<MT, R, true, true>(x, w, y, M, d, n_units, eps, sms, dev, stream)             \
              : launch_gemv_t<MT, R, true, false>(x, w, y, M, d, n_units, eps, sms, dev, stream))           \
       : (f32 ? launch_gemv_t<MT, R, false, true>(x, w, y, M, d, n_units, eps, sms, dev, stream)            \
              : launch_gemv_t<MT, R, false, false>(x, w, y, M, d, n_units, eps, sms, dev, stream)))
  switch (mt) {
    case 1: return FN_GEMV(1, 4);
    case 2: return FN_GEMV(2, 4);
    case 4: return FN_GEMV(4, 2);
    case 8: return FN_GEMV(8, 2);
    default: return FN_GEMV(16, 1);
  }
#undef FN_GEMV
}

// FP8 E4M3 weights (decode GEMV)
template <int MT, int R, bool OUT_F32>
fn_status launch_gemv_fp8_t(const void* x, const void* q, const void* scales, void* y, int64_t M, int64_t d,
                            int64_t N, float eps, int sms, int dev, cudaStream_t stream) {
  auto kern = fn::k_gemv_fp8<MT, R, OUT_F32>;
  const int smem = fn::gemv_smem_bytes<MT>(static_cast<int>(d));
  static int configured[kMaxDevices] = {0};
  if (smem > 48 * 1024 && configured[dev] < smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (fp8 gemv)");
    configured[dev] = smem;
  }
  const int64_t groups = (N + R - 1) / R;
  const int64_t blocks_needed = (groups + 7) / 8;
  int per_sm = (228 * 1024) / (smem + 1024);
  if (per_sm > 8) per_sm = 8;
  if (per_sm < 1) per_sm = 1;
  int64_t grid = static_cast<int64_t>(sms) * per_sm;
  if (blocks_needed < grid) grid = blocks_needed;
  cudaError_t e = launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(fn::kGemvThreads),
                                static_cast<size_t>(smem), stream, 1, static_cast<const uint16_t*>(x),
                                static_cast<const uint8_t*>(q), static_cast<const float*>(scales), y,
                                static_cast<int>(M), static_cast<int>(d), static_cast<int>(N), eps);
  if (e != cudaSuccess) return cuda_fail(e, "fp8 GEMV launch");
  return FN_OK;
}

// ------------------------------------------------------------------------------------------------
// FP8 decode on the tensor cores
// ------------------------------------------------------------------------------------------------

template <int STAGES, int KSPLIT, bool OUT_F32, int FMT = fn::kFmtFp8>
fn_status launch_decode_fp8_t(const CUtensorMap& tq, const CUtensorMap& tx, const fn::DecodeFp8Params& p, int slabs,
                              int dev, cudaStream_t stream) {
  auto kern = fn::k_decode_fp8<STAGES, KSPLIT, OUT_F32, FMT>;
  constexpr int smem = fn::decode_fp8_smem_bytes<STAGES, KSPLIT, FMT>();
  static bool configured[kMaxDevices] = {false};
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (fp8 decode)");
    configured[dev] = true;
  }
  // KSPLIT == 0: p.ksplit independent CTAs per slab (no cluster)
  const int ks = KSPLIT == 0 ? p.ksplit : KSPLIT;
  cudaError_t e = launch_kernel(kern, dim3(static_cast<unsigned>(slabs * ks)), dim3(fn::kD8Threads), smem, stream,
                                KSPLIT == 0 ? 1 : KSPLIT, tq, tx, p);
  if (e != cudaSuccess) return cuda_fail(e, "fp8 decode launch");
  return FN_OK;
}

// K ranges per slab of the quantized decode kernel with a workspace: enough independent CTAs for two on
// every SM (each holds 4-5 stages: two fit one SM's shared and tensor memory), while there are at most as
// many slabs as SMs; 1 (no split, no workspace) otherwise. k_stage: k per pipeline stage (128 for FP8,
// 256 for NVFP4); a range holds whole stages.
int fp8_ws_ksplit(int64_t N, int64_t d, int sms, int k_stage = fn::kD8KStage) {
  const int64_t slabs = (N + fn::kD8Rows - 1) / fn::kD8Rows;
  const int64_t units = (d + k_stage - 1) / k_stage;
  if (slabs > fn::kD8MaxWsSlabs || slabs > sms) return 1;
  int64_t ks = (2 * static_cast<int64_t>(sms)) / slabs;
  ks = std::min<int64_t>(std::min<int64_t>(ks, units), 16);
  return ks >= 2 ? static_cast<int>(ks) : 1;
}

int64_t fp8_ws_bytes(int64_t N, int ks) {
  if (ks < 2) return 0;
  const int64_t slabs = (N + fn::kD8Rows - 1) / fn::kD8Rows;
  return fn::kD8WsCounterBytes + slabs * ks * (fn::kD8Rows * fn::kD8Tok + fn::kD8Tok) * 4;
}

fn_status run_decode_fp8(const void* x, const void* q, const void* scales, void* y, int64_t M, int64_t d, int64_t N,
                         float eps, int out_dtype, void* workspace, cudaStream_t stream) {
  int dev = 0;
  const int sms = device_sm_count(&dev);
  if (sms <= 0) return fail(FN_ERR_CUDA, "cannot query the current device");
  const int64_t slabs = (N + fn::kD8Rows - 1) / fn::kD8Rows;
  const int64_t units = (d + fn::kD8KStage - 1) / fn::kD8KStage;
  // With a workspace: K in fp8_ws_ksplit ranges of independent CTAs, two on every SM. Without one, K is
  // split in a cluster as for the bf16 decode kernel: in two while there are at most as many slabs as SMs
  // (two 5-stage CTAs fit one SM), in four when there are few slabs; otherwise one 10-stage CTA per slab.
  // (A cluster of three, two 4-stage CTAs on every SM, took 23.9 us against 17.3 us on the Llama-7B QKV
  // codes: clusters of three do not all fit at once.)
  int ksplit = 1;
  const int ws_ks = workspace != nullptr ? fp8_ws_ksplit(N, d, sms) : 1;
  if (ws_ks >= 2) {
    ksplit = ws_ks;
  } else {
    if (slabs <= sms && units >= 2) ksplit = 2;
    if (slabs * 4 <= sms && units >= 4) ksplit = 4;
  }
  CUtensorMap tq, tx;
  fn_status st = make_u8_map(&tq, q, d, N, fn::kD8Rows);
  if (st != FN_OK) return st;
  st = make_operand_map(&tx, x, d, M, fn::kD8Tok);
  if (st != FN_OK) return st;
  fn::DecodeFp8Params p;
  p.y = y;
  p.scales = static_cast<const float*>(scales);
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(d);
  p.N = static_cast<int>(N);
  p.ldy = static_cast<int>(N);
  p.ksplit = ksplit;
  p.eps = eps;
  p.counters = nullptr;
  p.part = p.part_ss = nullptr;
  const int sl = static_cast<int>(slabs);
  const bool f32 = out_dtype == FN_F32;
#define FN_D8(ST, KS)                                                                                          \
  (f32 ? launch_decode_fp8_t<ST, KS, true>(tq, tx, p, sl, dev, stream)                                         \
       : launch_decode_fp8_t<ST, KS, false>(tq, tx, p, sl, dev, stream))
  if (ws_ks >= 2) {
    p.counters = static_cast<unsigned*>(workspace);
    p.part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + fn::kD8WsCounterBytes);
    p.part_ss = p.part + slabs * ksplit * fn::kD8Rows * fn::kD8Tok;
    return FN_D8(5, 0);
  }
  if (ksplit == 1) return FN_D8(10, 1);
  if (ksplit == 2) return FN_D8(5, 2);
  return FN_D8(4, 4);
#undef FN_D8
}

// NVFP4 W* on the tensor cores: the same kernel with the 4-bit widening and 256-k stages (two units). With
// a workspace, the K split over independent CTAs (four 26 KB stages each: two CTAs fit one SM); without
// one, one CTA per slab over all of K (eight stages).
fn_status run_decode_nvfp4(const void* x, const void* q4, const void* s2, void* y, int64_t M, int64_t d, int64_t N,
                           float eps, int out_dtype, void* workspace, cudaStream_t stream) {
  int dev = 0;
  const int sms = device_sm_count(&dev);
  if (sms <= 0) return fail(FN_ERR_CUDA, "cannot query the current device");
  const int64_t slabs = (N + fn::kD8Rows - 1) / fn::kD8Rows;
  const int64_t groups = (d + fn::kNvfp4Group - 1) / fn::kNvfp4Group;
  const int ks = workspace != nullptr ? fp8_ws_ksplit(N, d, sms, fn::kNvfp4Group) : 1;
  CUtensorMap tq, tx;
  fn_status st = make_q4_map(&tq, q4, groups * fn::kNvfp4GroupBytes, N);
  if (st != FN_OK) return st;
  st = make_operand_map(&tx, x, d, M, fn::kD8Tok);
  if (st != FN_OK) return st;
  fn::DecodeFp8Params p;
  p.y = y;
  p.scales = static_cast<const float*>(s2);
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(d);
  p.N = static_cast<int>(N);
  p.ldy = static_cast<int>(N);
  p.ksplit = ks;
  p.eps = eps;
  p.counters = nullptr;
  p.part = p.part_ss = nullptr;
  const int sl = static_cast<int>(slabs);
  const bool f32 = out_dtype == FN_F32;
#define FN_D4(ST, KS)                                                                                          \
  (f32 ? launch_decode_fp8_t<ST, KS, true, fn::kFmtNvfp4>(tq, tx, p, sl, dev, stream)                          \
       : launch_decode_fp8_t<ST, KS, false, fn::kFmtNvfp4>(tq, tx, p, sl, dev, stream))
  if (ks >= 2) {
    p.counters = static_cast<unsigned*>(workspace);
    p.part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + fn::kD8WsCounterBytes);
    p.part_ss = p.part + slabs * ks * fn::kD8Rows * fn::kD8Tok;
    return FN_D4(4, 0);
  }
  return FN_D4(8, 1);
#undef FN_D4
}

// ------------------------------------------------------------------------------------------------
// Tensor-core decode path
// ------------------------------------------------------------------------------------------------

template <int STAGES, int KSPLIT, bool GLU, bool OUT_F32, bool LN>
fn_status launch_decode_t(const CUtensorMap& tw, const CUtensorMap& tx, const fn::DecodeParams& p, int slabs,
                          int dev, cudaStream_t stream) {
  auto kern = fn::k_decode_tc<STAGES, KSPLIT, GLU, OUT_F32, LN>;
  constexpr int smem = fn::decode_smem_bytes<STAGES, KSPLIT>();
  static bool configured[kMaxDevices] = {false};
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (decode)");
    configured[dev] = true;
  }
  cudaError_t e = launch_kernel(kern, dim3(static_cast<unsigned>(slabs * KSPLIT)), dim3(fn::kDecThreads), smem,
                                stream, KSPLIT, tw, tx, p);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return FN_OK;
}

// colsum / bias non-null: the LayerNorm epilogue (linear only).
fn_status run_decode_tc(const void* x, const void* w, void* y, int64_t M, int64_t d, int64_t n_rows, int64_t n_out,
                        float eps, int out_dtype, bool glu, cudaStream_t stream, const float* colsum = nullptr,
                        const float* bias = nullptr) {
  int dev = 0;
  const int sms = device_sm_count(&dev);
  if (sms <= 0) return fail(FN_ERR_CUDA, "cannot query the current device");
  const int64_t slabs = (n_rows + fn::kDecRows - 1) / fn::kDecRows;
  const int64_t num_kb = (d + 63) / 64;
  // Split K across a cluster so that more SMs stream W*: in two while there are at most as many slabs as
  // SMs (two 5-stage CTAs fit one SM), in four when there are few slabs. Llama-7B QKV (96 slabs): 22.7 ->
  // 20.5 us with the split in two; in four, 25.6 us. (In three, 288 four-stage CTAs two to an SM:
  // 27.0 us. In two with six stages, the partial sums moved into the idle W* stages: 21.8 us.)
  int ksplit = 1;
  if (slabs <= sms && num_kb >= 2) ksplit = 2;
  if (slabs * 4 <= sms && num_kb >= 4) ksplit = 4;
  CUtensorMap tw, tx;
  fn_status st = make_operand_map(&tw, w, d, n_rows, fn::kDecRows);
  if (st != FN_OK) return st;
  st = make_operand_map(&tx, x, d, M, fn::kDecTok);
  if (st != FN_OK) return st;
  fn::DecodeParams p;
  p.y = y;
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(d);
  p.n_rows = static_cast<int>(n_rows);
  p.n_out = static_cast<int>(n_out);
  p.ldy = static_cast<int>(n_out);
  p.ksplit = ksplit;
  p.eps = eps;
  p.ln_colsum = colsum;
  p.ln_bias = bias;
  const bool ln = colsum != nullptr;
  const int sl = static_cast<int>(slabs);
  const bool f32 = out_dtype == FN_F32;
#define FN_DEC(ST, KS)                                                                                          \
  (ln    ? (f32 ? launch_decode_t<ST, KS, false, true, true>(tw, tx, p, sl, dev, stream)                     \
                : launch_decode_t<ST, KS, false, false, true>(tw, tx, p, sl, dev, stream))                   \
   : glu ? (f32 ? launch_decode_t<ST, KS, true, true, false>(tw, tx, p, sl, dev, stream)                     \
                : launch_decode_t<ST, KS, true, false, false>(tw, tx, p, sl, dev, stream))                   \
         : (f32 ? launch_decode_t<ST, KS, false, true, false>(tw, tx, p, sl, dev, stream)                    \
                : launch_decode_t<ST, KS, false, false, false>(tw, tx, p, sl, dev, stream)))
  if (ksplit == 1) return FN_DEC(12, 1);
  if (ksplit == 2) return FN_DEC(5, 2);
  return FN_DEC(3, 4);
#undef FN_DEC
}

fn_status projection(const void* x, const void* w, void* y, int64_t M, int64_t d, int64_t n_rows, int64_t n_out,
                     float eps, int out_dtype, int path, bool glu, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (path != FN_PATH_AUTO && path != FN_PATH_TENSOR && path != FN_PATH_GEMV && path != FN_PATH_DECODE &&
      path != FN_PATH_PAIR)
    return fail(FN_ERR_INVALID_ARG, "path %d unknown", path);
  if (M == 0) return FN_OK;
  if (path == FN_PATH_DECODE) {
    if (M > FN_DECODE_MAX_M) return fail(FN_ERR_UNSUPPORTED, "decode path takes M <= %d", FN_DECODE_MAX_M);
    return run_decode_tc(x, w, y, M, d, n_rows, n_out, eps, out_dtype, glu, s);
  }
  // Prefill: CTA pairs (2-SM MMA) whenever there is more than one 128-row tile of x.
  if (path == FN_PATH_PAIR || (path == FN_PATH_AUTO && M > fn::kBM))
    return run_pair_path(x, w, y, M, d, n_rows, n_out, eps, out_dtype, glu ? fn::EPI_GLU : fn::EPI_LINEAR, true, s);
  if (path == FN_PATH_AUTO && M <= FN_DECODE_MAX_M)
    return run_decode_tc(x, w, y, M, d, n_rows, n_out, eps, out_dtype, glu, s);
  bool use_gemv = path == FN_PATH_GEMV;
  if (use_gemv) {
    if (M > FN_DECODE_MAX_M) return fail(FN_ERR_UNSUPPORTED, "GEMV path takes M <= %d", FN_DECODE_MAX_M);
    if (!gemv_fits(M, d)) return fail(FN_ERR_UNSUPPORTED, "GEMV path: x [%lld, %lld] does not fit in shared memory",
                                      (long long)M, (long long)d);
    return run_gemv(x, w, y, M, d, n_out, eps, out_dtype, glu, s);
  }
  return run_tensor_path(x, w, y, nullptr, M, d, n_rows, n_out, 0, eps, out_dtype,
                         glu ? fn::EPI_GLU : fn::EPI_LINEAR, true, s);
}

fn_status check_postnorm(const void* x, const void* Wstar, const void* g2, const void* y, int64_t M, int64_t d,
                         int64_t N, int64_t head_dim, float eps2, int out_dtype) {
  fn_status st = check_common(x, Wstar, y, M, d, eps2, out_dtype);
  if (st != FN_OK) return st;
  if (head_dim < 16 || head_dim % 16 != 0) return fail(FN_ERR_INVALID_ARG, "head_dim = %lld must be a positive multiple of 16", (long long)head_dim);
  if (head_dim > 512) return fail(FN_ERR_UNSUPPORTED, "head_dim = %lld > 512 (one tensor memory)", (long long)head_dim);
  if (head_dim > 256 && head_dim % 32 != 0) return fail(FN_ERR_UNSUPPORTED, "head_dim in (256, 512] must be a multiple of 32");
  if (N < head_dim || N > kMaxDim || N % head_dim != 0) return fail(FN_ERR_INVALID_ARG, "N = %lld must be a multiple of head_dim", (long long)N);
  return check_ptr(g2, "g2");
}

}  // namespace

extern "C" {

fn_status flashnorm_fold_weights(const void* W, const void* g, void* Wstar, int64_t d, int64_t N, int glu,
                                 void* stream) {
  g_last_error[0] = '\0';
  if (d < 8 || d > kMaxDim || d % 8 != 0) return fail(FN_ERR_INVALID_ARG, "d = %lld must be a positive multiple of 8", (long long)d);
  if (N < 8 || N > kMaxDim || N % 8 != 0) return fail(FN_ERR_INVALID_ARG, "N = %lld must be a positive multiple of 8", (long long)N);
  if (glu != 0 && glu != 1) return fail(FN_ERR_INVALID_ARG, "glu must be 0 or 1");
  if (glu && (N % 32 != 0)) return fail(FN_ERR_INVALID_ARG, "GLU fold needs N = 2F with F %% 16 == 0");
  fn_status st;
  if ((st = check_ptr(W, "W")) != FN_OK) return st;
  if ((st = check_ptr(g, "g")) != FN_OK) return st;
  if ((st = check_ptr(Wstar, "Wstar")) != FN_OK) return st;
  dim3 grid(static_cast<unsigned>((N + fn::kFoldTile - 1) / fn::kFoldTile),
            static_cast<unsigned>((d + fn::kFoldTile - 1) / fn::kFoldTile));
  if (grid.y > 65535) return fail(FN_ERR_UNSUPPORTED, "d too large for the fold grid");
  cudaError_t e = launch_kernel(fn::k_fold, grid, dim3(256), 0, static_cast<cudaStream_t>(stream), 1,
                                static_cast<const uint16_t*>(W), static_cast<const uint16_t*>(g),
                                static_cast<uint16_t*>(Wstar), static_cast<int>(d), static_cast<int>(N), glu);
  if (e != cudaSuccess) return cuda_fail(e, "fold launch");
  return FN_OK;
}

fn_status flashnorm_linear_ex(const void* x, const void* Wstar, void* y, int64_t M, int64_t d, int64_t N, float eps,
                              int out_dtype, int path, void* stream) {
  g_last_error[0] = '\0';
  fn_status st = check_common(x, Wstar, y, M, d, eps, out_dtype);
  if (st != FN_OK) return st;
  if (N < 8 || N > kMaxDim || N % 8 != 0) return fail(FN_ERR_INVALID_ARG, "N = %lld must be a positive multiple of 8", (long long)N);
  return projection(x, Wstar, y, M, d, N, N, eps, out_dtype, path, false, stream);
}

fn_status flashnorm_linear(const void* x, const void* Wstar, void* y, int64_t M, int64_t d, int64_t N, float eps,
                           int out_dtype, void* stream) {
  return flashnorm_linear_ex(x, Wstar, y, M, d, N, eps, out_dtype, FN_PATH_AUTO, stream);
}

fn_status flashnorm_glu_ex(const void* x, const void* Wstar_gu, void* y, int64_t M, int64_t d, int64_t F, float eps,
                           int out_dtype, int path, void* stream) {
  g_last_error[0] = '\0';
  fn_status st = check_common(x, Wstar_gu, y, M, d, eps, out_dtype);
  if (st != FN_OK) return st;
  if (F < 16 || F > kMaxDim / 2 || F % 16 != 0) return fail(FN_ERR_INVALID_ARG, "F = %lld must be a positive multiple of 16", (long long)F);
  return projection(x, Wstar_gu, y, M, d, 2 * F, F, eps, out_dtype, path, true, stream);
}

fn_status flashnorm_glu(const void* x, const void* Wstar_gu, void* y, int64_t M, int64_t d, int64_t F, float eps,
                        int out_dtype, void* stream) {
  return flashnorm_glu_ex(x, Wstar_gu, y, M, d, F, eps, out_dtype, FN_PATH_AUTO, stream);
}

fn_status flashnorm_postnorm_workspace_bytes(int64_t M, int64_t d, int64_t N, int64_t head_dim, int64_t* bytes) {
  g_last_error[0] = '\0';
  if (bytes == nullptr) return fail(FN_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = 0;
  if (M < 0 || M > kMaxDim) return fail(FN_ERR_INVALID_ARG, "M = %lld out of range", (long long)M);
  if (d < 8 || d > kMaxDim || d % 8 != 0) return fail(FN_ERR_INVALID_ARG, "d = %lld must be a positive multiple of 8", (long long)d);
  if (head_dim < 16 || head_dim % 16 != 0 || head_dim > 512) return fail(FN_ERR_INVALID_ARG, "head_dim = %lld out of range", (long long)head_dim);
  if (N < head_dim || N > kMaxDim || N % head_dim != 0) return fail(FN_ERR_INVALID_ARG, "N = %lld must be a multiple of head_dim", (long long)N);
  const int ks = postnorm_split_ks(M, d, N, head_dim);
  *bytes = static_cast<int64_t>(ks) * M * N * 4;
  return FN_OK;
}

fn_status flashnorm_linear_postnorm_ws(const void* x, const void* Wstar, const void* g2, void* y, int64_t M, int64_t d,
                                       int64_t N, int64_t head_dim, float eps2, int out_dtype, void* workspace,
                                       int64_t workspace_bytes, void* stream) {
  g_last_error[0] = '\0';
  fn_status st = check_postnorm(x, Wstar, g2, y, M, d, N, head_dim, eps2, out_dtype);
  if (st != FN_OK) return st;
  if (workspace_bytes < 0) return fail(FN_ERR_INVALID_ARG, "workspace_bytes is negative");
  if (M == 0) return FN_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (head_dim > 256) {
    const int ks = workspace != nullptr ? postnorm_split_ks(M, d, N, head_dim) : 0;
    if (ks > 0) {
      const int64_t need = static_cast<int64_t>(ks) * M * N * 4;
      if (workspace_bytes < need)
        return fail(FN_ERR_INVALID_ARG, "workspace of %lld bytes; this shape needs %lld",
                    (long long)workspace_bytes, (long long)need);
      if ((st = check_ptr(workspace, "workspace")) != FN_OK) return st;
      return run_postnorm_split(x, Wstar, g2, y, M, d, N, head_dim, eps2, out_dtype, ks, workspace, s);
    }
    return run_postnorm_pair(x, Wstar, g2, y, M, d, N, head_dim, eps2, out_dtype, s);
  }
  return run_tensor_path(x, Wstar, y, g2, M, d, N, N, head_dim, eps2, out_dtype, fn::EPI_POSTNORM, false, s);
}

fn_status flashnorm_linear_postnorm(const void* x, const void* Wstar, const void* g2, void* y, int64_t M, int64_t d,
                                    int64_t N, int64_t head_dim, float eps2, int out_dtype, void* stream) {
  return flashnorm_linear_postnorm_ws(x, Wstar, g2, y, M, d, N, head_dim, eps2, out_dtype, nullptr, 0, stream);
}

fn_status flashnorm_linear_postnorm_rope(const void* x, const void* Wstar, const void* g2, const void* rope_cs,
                                         const void* positions, void* y, int64_t M, int64_t d, int64_t N,
                                         int64_t head_dim, int64_t n_rope_heads, int64_t max_pos, float eps2,
                                         int out_dtype, void* stream) {
  g_last_error[0] = '\0';
  fn_status st = check_common(x, Wstar, y, M, d, eps2, out_dtype);
  if (st != FN_OK) return st;
  if (head_dim < 16 || head_dim % 16 != 0) return fail(FN_ERR_INVALID_ARG, "head_dim = %lld must be a positive multiple of 16", (long long)head_dim);
  if (head_dim > 512 || (head_dim > 256 && head_dim % 128 == 0))
    return fail(FN_ERR_UNSUPPORTED, "RoPE is fused for heads of at most 256 (and 320) features, not %lld", (long long)head_dim);
  if (head_dim > 256 && head_dim % 32 != 0) return fail(FN_ERR_UNSUPPORTED, "head_dim in (256, 512] must be a multiple of 32");
  if (N < head_dim || N > kMaxDim || N % head_dim != 0) return fail(FN_ERR_INVALID_ARG, "N = %lld must be a multiple of head_dim", (long long)N);
  if (n_rope_heads < 0 || n_rope_heads > N / head_dim)
    return fail(FN_ERR_INVALID_ARG, "n_rope_heads = %lld must be in [0, N / head_dim]", (long long)n_rope_heads);
  if (max_pos < 1 || max_pos > kMaxDim) return fail(FN_ERR_INVALID_ARG, "max_pos = %lld must be positive", (long long)max_pos);
  if ((st = check_ptr(g2, "g2")) != FN_OK) return st;
  if ((st = check_ptr(rope_cs, "rope_cs")) != FN_OK) return st;
  if (M == 0) return FN_OK;
  if (positions == nullptr) return fail(FN_ERR_INVALID_ARG, "positions is NULL");
  if ((reinterpret_cast<uintptr_t>(positions) & 3u) != 0) return fail(FN_ERR_ALIGN, "positions is not 4-byte aligned");
  const RopeArgs rope = {static_cast<const float*>(rope_cs), static_cast<const int*>(positions),
                         static_cast<int>(n_rope_heads), static_cast<int>(max_pos)};
  return run_tensor_path(x, Wstar, y, g2, M, d, N, N, head_dim, eps2, out_dtype, fn::EPI_POSTNORM, false,
                         static_cast<cudaStream_t>(stream), &rope);
}

fn_status flashnorm_fold_layernorm(const void* W, const void* gamma, const void* beta, void* Wstar, void* colsum,
                                   void* bias, int64_t d, int64_t N, void* stream) {
  g_last_error[0] = '\0';
  fn_status st;
  // everything is validated before the first launch
  if ((st = check_ptr(colsum, "colsum")) != FN_OK) return st;
  if ((st = check_ptr(bias, "bias")) != FN_OK) return st;
  if (beta != nullptr && (st = check_ptr(beta, "beta")) != FN_OK) return st;
  st = flashnorm_fold_weights(W, gamma, Wstar, d, N, 0, stream);  // validates W, gamma, Wstar, d, N, then folds
  if (st != FN_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_kernel(fn::k_ln_colsum, dim3(static_cast<unsigned>((N + 7) / 8)), dim3(256), 0, s, 1,
                                static_cast<const uint16_t*>(Wstar), static_cast<float*>(colsum), static_cast<int>(d),
                                static_cast<int>(N));
  if (e == cudaSuccess)
    e = launch_kernel(fn::k_ln_bias, dim3(static_cast<unsigned>((N + 255) / 256)), dim3(256), 0, s, 1,
                      static_cast<const uint16_t*>(W), static_cast<const uint16_t*>(beta), static_cast<float*>(bias),
                      static_cast<int>(d), static_cast<int>(N));
  if (e != cudaSuccess) return cuda_fail(e, "LayerNorm fold launch");
  return FN_OK;
}

fn_status flashnorm_layernorm_linear(const void* x, const void* Wstar, const void* colsum, const void* bias, void* y,
                                     int64_t M, int64_t d, int64_t N, float eps, int out_dtype, void* stream) {
  g_last_error[0] = '\0';
  fn_status st = check_common(x, Wstar, y, M, d, eps, out_dtype);
  if (st != FN_OK) return st;
  if (N < 8 || N > kMaxDim || N % 8 != 0) return fail(FN_ERR_INVALID_ARG, "N = %lld must be a positive multiple of 8", (long long)N);
  if ((st = check_ptr(colsum, "colsum")) != FN_OK) return st;
  if ((st = check_ptr(bias, "bias")) != FN_OK) return st;
  if (M == 0) return FN_OK;
  // decode-sized batches on the tensor-core decode kernel (the weights stream once), larger on CTA pairs
  if (M <= FN_DECODE_MAX_M)
    return run_decode_tc(x, Wstar, y, M, d, N, N, eps, out_dtype, false, static_cast<cudaStream_t>(stream),
                         static_cast<const float*>(colsum), static_cast<const float*>(bias));
  return run_pair_path(x, Wstar, y, M, d, N, N, eps, out_dtype, fn::EPI_LN, true, static_cast<cudaStream_t>(stream),
                       static_cast<const float*>(colsum), static_cast<const float*>(bias));
}

fn_status flashnorm_fold_weights_fp8(const void* W, const void* g, void* Q, void* scales, int64_t d, int64_t N,
                                     void* stream) {
  g_last_error[0] = '\0';
  if (d < 16 || d > kMaxDim || d % 16 != 0) return fail(FN_ERR_INVALID_ARG, "d = %lld must be a positive multiple of 16", (long long)d);
  if (N < 8 || N > kMaxDim || N % 8 != 0) return fail(FN_ERR_INVALID_ARG, "N = %lld must be a positive multiple of 8", (long long)N);
  fn_status st;
  if ((st = check_ptr(W, "W")) != FN_OK) return st;
  if ((st = check_ptr(g, "g")) != FN_OK) return st;
  if ((st = check_ptr(Q, "Q")) != FN_OK) return st;
  if ((st = check_ptr(scales, "scales")) != FN_OK) return st;
  dim3 grid(static_cast<unsigned>((N + fn::kFoldTile - 1) / fn::kFoldTile),
            static_cast<unsigned>((d + fn::kFoldTile - 1) / fn::kFoldTile));
  if (grid.y > 65535) return fail(FN_ERR_UNSUPPORTED, "d too large for the fold grid");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_kernel(fn::k_fp8_scales, dim3(static_cast<unsigned>((N + 255) / 256)), dim3(256), 0, s, 1,
                                static_cast<const uint16_t*>(W), static_cast<const uint16_t*>(g),
                                static_cast<float*>(scales), static_cast<int>(d), static_cast<int>(N), fn::kE4m3Max);
  if (e == cudaSuccess)
    e = launch_kernel(fn::k_fold_fp8, grid, dim3(256), 0, s, 1, static_cast<const uint16_t*>(W),
                      static_cast<const uint16_t*>(g), static_cast<const float*>(scales), static_cast<uint8_t*>(Q),
                      static_cast<int>(d), static_cast<int>(N));
  if (e != cudaSuccess) return cuda_fail(e, "fp8 fold launch");
  return FN_OK;
}

fn_status flashnorm_fp8_workspace_bytes(int64_t M, int64_t d, int64_t N, int64_t* bytes) {
  g_last_error[0] = '\0';
  if (bytes == nullptr) return fail(FN_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = 0;
  if (M < 0 || M > kMaxDim) return fail(FN_ERR_INVALID_ARG, "M = %lld out of range", (long long)M);
  if (d < 16 || d > kMaxDim || d % 16 != 0) return fail(FN_ERR_INVALID_ARG, "d = %lld must be a positive multiple of 16", (long long)d);
  if (N < 8 || N > kMaxDim || N % 8 != 0) return fail(FN_ERR_INVALID_ARG, "N = %lld must be a positive multiple of 8", (long long)N);
  if (M == 0 || M > FN_DECODE_MAX_M) return FN_OK;
  int dev = 0;
  const int sms = device_sm_count(&dev);
  if (sms <= 0) return fail(FN_ERR_CUDA, "cannot query the current device");
  *bytes = fp8_ws_bytes(N, fp8_ws_ksplit(N, d, sms));
  return FN_OK;
}

fn_status flashnorm_linear_fp8_ws(const void* x, const void* Q, const void* scales, void* y, int64_t M, int64_t d,
                                  int64_t N, float eps, int out_dtype, int path, void* workspace,
                                  int64_t workspace_bytes, void* stream) {
  g_last_error[0] = '\0';
  if (path != FN_PATH_AUTO && path != FN_PATH_DECODE && path != FN_PATH_GEMV)
    return fail(FN_ERR_INVALID_ARG, "fp8 path %d: AUTO, DECODE or GEMV", path);
  fn_status st = check_common(x, Q, y, M, d, eps, out_dtype);
  if (st != FN_OK) return st;
  if (d % 16 != 0) return fail(FN_ERR_INVALID_ARG, "d = %lld must be a multiple of 16", (long long)d);
  if (N < 8 || N > kMaxDim || N % 8 != 0) return fail(FN_ERR_INVALID_ARG, "N = %lld must be a positive multiple of 8", (long long)N);
  if (M > FN_DECODE_MAX_M) return fail(FN_ERR_UNSUPPORTED, "the fp8 path is the decode GEMV: M <= %d", FN_DECODE_MAX_M);
  if ((st = check_ptr(scales, "scales")) != FN_OK) return st;
  if (workspace_bytes < 0) return fail(FN_ERR_INVALID_ARG, "workspace_bytes is negative");
  if (M == 0) return FN_OK;
  void* ws = nullptr;  // the workspace, where the tensor-core kernel's K split uses one for this shape
  if (workspace != nullptr && path != FN_PATH_GEMV) {
    int dev = 0;
    const int sms = device_sm_count(&dev);
    if (sms <= 0) return fail(FN_ERR_CUDA, "cannot query the current device");
    const int64_t need = fp8_ws_bytes(N, fp8_ws_ksplit(N, d, sms));
    if (need > 0) {
      if (workspace_bytes < need)
        return fail(FN_ERR_INVALID_ARG, "workspace of %lld bytes; this shape needs %lld", (long long)workspace_bytes,
                    (long long)need);
      if ((st = check_ptr(workspace, "workspace")) != FN_OK) return st;
      ws = workspace;
    }
  }
  // AUTO: the tensor-core kernel, whose time does not grow with M (the GEMV's does: 29 us at 4 tokens,
  // 125 us at 16), except for one token without a workspace, where the CUDA-core GEMV (16.2 us for the
  // Llama-7B QKV codes) beats the cluster-split kernel (18.0 us).
  if (path == FN_PATH_DECODE || (path == FN_PATH_AUTO && (M > 1 || ws != nullptr)))
    return run_decode_fp8(x, Q, scales, y, M, d, N, eps, out_dtype, ws, static_cast<cudaStream_t>(stream));
  if (!gemv_fits(M, d)) return fail(FN_ERR_UNSUPPORTED, "x [%lld, %lld] does not fit in shared memory", (long long)M, (long long)d);
  int dev = 0;
  const int sms = device_sm_count(&dev);
  if (sms <= 0) return fail(FN_ERR_CUDA, "cannot query the current device");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool f32 = out_dtype == FN_F32;
#define FN_G8(MT, R)                                                                          \
  (f32 ? launch_gemv_fp8_t<MT, R, true>(x, Q, scales, y, M, d, N, eps, sms, dev, s)          \
       : launch_gemv_fp8_t<MT, R, false>(x, Q, scales, y, M, d, N, eps, sms, dev, s))
  switch (gemv_mt(M)) {
    case 1: return FN_G8(1, 4);
    case 2: return FN_G8(2, 4);
    case 4: return FN_G8(4, 2);
    case 8: return FN_G8(8, 2);
    default: return FN_G8(16, 1);
  }
#undef FN_G8
}

fn_status flashnorm_fold_weights_nvfp4(const void* W, const void* g, void* Q4, void* s2, int64_t d, int64_t N,
                                       void* stream) {
  g_last_error[0] = '\0';
  if (d < 16 || d > kMaxDim || d % 16 != 0) return fail(FN_ERR_INVALID_ARG, "d = %lld must be a positive multiple of 16", (long long)d);
  if (N < 8 || N > kMaxDim || N % 8 != 0) return fail(FN_ERR_INVALID_ARG, "N = %lld must be a positive multiple of 8", (long long)N);
  fn_status st;
  if ((st = check_ptr(W, "W")) != FN_OK) return st;
  if ((st = check_ptr(g, "g")) != FN_OK) return st;
  if ((st = check_ptr(Q4, "Q4")) != FN_OK) return st;
  if ((st = check_ptr(s2, "s2")) != FN_OK) return st;
  const int64_t groups = (d + fn::kNvfp4Group - 1) / fn::kNvfp4Group;
  if (groups > 65535) return fail(FN_ERR_UNSUPPORTED, "d too large for the fold grid");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_kernel(fn::k_fp8_scales, dim3(static_cast<unsigned>((N + 255) / 256)), dim3(256), 0, s, 1,
                                static_cast<const uint16_t*>(W), static_cast<const uint16_t*>(g),
                                static_cast<float*>(s2), static_cast<int>(d), static_cast<int>(N), fn::kNvfp4ScaleDiv);
  if (e == cudaSuccess)
    e = launch_kernel(fn::k_fold_nvfp4, dim3(static_cast<unsigned>((N + 31) / 32), static_cast<unsigned>(groups)),
                      dim3(256), 0, s, 1, static_cast<const uint16_t*>(W), static_cast<const uint16_t*>(g),
                      static_cast<const float*>(s2), static_cast<uint8_t*>(Q4), static_cast<int>(d),
                      static_cast<int>(N));
  if (e != cudaSuccess) return cuda_fail(e, "nvfp4 fold launch");
  return FN_OK;
}

fn_status flashnorm_nvfp4_workspace_bytes(int64_t M, int64_t d, int64_t N, int64_t* bytes) {
  g_last_error[0] = '\0';
  if (bytes == nullptr) return fail(FN_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = 0;
  if (M < 0 || M > kMaxDim) return fail(FN_ERR_INVALID_ARG, "M = %lld out of range", (long long)M);
  if (d < 16 || d > kMaxDim || d % 16 != 0) return fail(FN_ERR_INVALID_ARG, "d = %lld must be a positive multiple of 16", (long long)d);
  if (N < 8 || N > kMaxDim || N % 8 != 0) return fail(FN_ERR_INVALID_ARG, "N = %lld must be a positive multiple of 8", (long long)N);
  if (M == 0 || M > FN_DECODE_MAX_M) return FN_OK;
  int dev = 0;
  const int sms = device_sm_count(&dev);
  if (sms <= 0) return fail(FN_ERR_CUDA, "cannot query the current device");
  *bytes = fp8_ws_bytes(N, fp8_ws_ksplit(N, d, sms, fn::kNvfp4Group));
  return FN_OK;
}

fn_status flashnorm_linear_nvfp4(const void* x, const void* Q4, const void* s2, void* y, int64_t M, int64_t d,
                                 int64_t N, float eps, int out_dtype, void* workspace, int64_t workspace_bytes,
                                 void* stream) {
  g_last_error[0] = '\0';
  fn_status st = check_common(x, Q4, y, M, d, eps, out_dtype);
  if (st != FN_OK) return st;
  if (d % 16 != 0) return fail(FN_ERR_INVALID_ARG, "d = %lld must be a multiple of 16", (long long)d);
  if (N < 8 || N > kMaxDim || N % 8 != 0) return fail(FN_ERR_INVALID_ARG, "N = %lld must be a positive multiple of 8", (long long)N);
  if (M > FN_DECODE_MAX_M) return fail(FN_ERR_UNSUPPORTED, "the nvfp4 path is decode only: M <= %d", FN_DECODE_MAX_M);
  if ((st = check_ptr(s2, "s2")) != FN_OK) return st;
  if (workspace_bytes < 0) return fail(FN_ERR_INVALID_ARG, "workspace_bytes is negative");
  if (M == 0) return FN_OK;
  void* ws = nullptr;
  if (workspace != nullptr) {
    int dev = 0;
    const int sms = device_sm_count(&dev);
    if (sms <= 0) return fail(FN_ERR_CUDA, "cannot query the current device");
    const int64_t need = fp8_ws_bytes(N, fp8_ws_ksplit(N, d, sms, fn::kNvfp4Group));
    if (need > 0) {
      if (workspace_bytes < need)
        return fail(FN_ERR_INVALID_ARG, "workspace of %lld bytes; this shape needs %lld", (long long)workspace_bytes,
                    (long long)need);
      if ((st = check_ptr(workspace, "workspace")) != FN_OK) return st;
      ws = workspace;
    }
  }
  return run_decode_nvfp4(x, Q4, s2, y, M, d, N, eps, out_dtype, ws, static_cast<cudaStream_t>(stream));
}

fn_status flashnorm_linear_fp8_ex(const void* x, const void* Q, const void* scales, void* y, int64_t M, int64_t d,
                                  int64_t N, float eps, int out_dtype, int path, void* stream) {
  return flashnorm_linear_fp8_ws(x, Q, scales, y, M, d, N, eps, out_dtype, path, nullptr, 0, stream);
}

fn_status flashnorm_linear_fp8(const void* x, const void* Q, const void* scales, void* y, int64_t M, int64_t d,
                               int64_t N, float eps, int out_dtype, void* stream) {
  return flashnorm_linear_fp8_ex(x, Q, scales, y, M, d, N, eps, out_dtype, FN_PATH_AUTO, stream);
}

fn_status flashnorm_rope_table(void* rope_cs, int64_t max_pos, int64_t head_dim, double base, void* stream) {
  g_last_error[0] = '\0';
  if (max_pos < 1 || max_pos > kMaxDim) return fail(FN_ERR_INVALID_ARG, "max_pos = %lld must be positive", (long long)max_pos);
  if (head_dim < 2 || head_dim % 2 != 0 || head_dim > 65536)
    return fail(FN_ERR_INVALID_ARG, "head_dim = %lld must be even", (long long)head_dim);
  if (!(base > 1.0) || !std::isfinite(base)) return fail(FN_ERR_INVALID_ARG, "base must be finite and > 1");
  fn_status st;
  if ((st = check_ptr(rope_cs, "rope_cs")) != FN_OK) return st;
  const long long n = static_cast<long long>(max_pos) * (head_dim / 2);
  const long long blocks = std::min<long long>((n + 255) / 256, 148LL * 16);
  cudaError_t e = launch_kernel(fn::k_rope_table, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                                static_cast<cudaStream_t>(stream), 1, static_cast<float*>(rope_cs),
                                static_cast<int>(max_pos), static_cast<int>(head_dim), base);
  if (e != cudaSuccess) return cuda_fail(e, "rope table launch");
  return FN_OK;
}

fn_status flashnorm_rmsnorm(const void* x, const void* g, void* xn, int64_t M, int64_t d, float eps, void* stream) {
  g_last_error[0] = '\0';
  if (M < 0 || M > kMaxDim) return fail(FN_ERR_INVALID_ARG, "M out of range");
  if (d < 8 || d > kMaxDim || d % 8 != 0) return fail(FN_ERR_INVALID_ARG, "d must be a positive multiple of 8");
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return fail(FN_ERR_INVALID_ARG, "eps must be finite and >= 0");
  fn_status st;
  if ((st = check_ptr(g, "g")) != FN_OK) return st;
  if (M == 0) return FN_OK;
  if ((st = check_ptr(x, "x")) != FN_OK) return st;
  if ((st = check_ptr(xn, "xn")) != FN_OK) return st;
  const int64_t blocks = (M + 7) / 8;
  cudaError_t e = launch_kernel(fn::k_rmsnorm, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                                static_cast<cudaStream_t>(stream), 1, static_cast<const uint16_t*>(x),
                                static_cast<const uint16_t*>(g), static_cast<uint16_t*>(xn), static_cast<int>(M),
                                static_cast<int>(d), eps);
  if (e != cudaSuccess) return cuda_fail(e, "rmsnorm launch");
  return FN_OK;
}

static fn_status unfused(const void* x, const void* g, const void* Wk, void* xn_ws, void* y, int64_t M, int64_t d,
                         int64_t n_rows, int64_t n_out, float eps, int out_dtype, bool glu, void* stream) {
  fn_status st = check_common(x, Wk, y, M, d, eps, out_dtype);
  if (st != FN_OK) return st;
  if ((st = check_ptr(g, "g")) != FN_OK) return st;
  if (M == 0) return FN_OK;
  if ((st = check_ptr(xn_ws, "xn_ws")) != FN_OK) return st;
  st = flashnorm_rmsnorm(x, g, xn_ws, M, d, eps, stream);
  if (st != FN_OK) return st;
  // the same GEMM kernel the fused path picks, with the deferred scale switched off
  if (M > fn::kBM)
    return run_pair_path(xn_ws, Wk, y, M, d, n_rows, n_out, 0.0f, out_dtype, glu ? fn::EPI_GLU : fn::EPI_LINEAR,
                         false, static_cast<cudaStream_t>(stream));
  return run_tensor_path(xn_ws, Wk, y, nullptr, M, d, n_rows, n_out, 0, 0.0f, out_dtype,
                         glu ? fn::EPI_GLU : fn::EPI_LINEAR, false, static_cast<cudaStream_t>(stream));
}

fn_status flashnorm_linear_unfused(const void* x, const void* g, const void* W_kmajor, void* xn_ws, void* y,
                                   int64_t M, int64_t d, int64_t N, float eps, int out_dtype, void* stream) {
  g_last_error[0] = '\0';
  if (N < 8 || N > kMaxDim || N % 8 != 0) return fail(FN_ERR_INVALID_ARG, "N must be a positive multiple of 8");
  return unfused(x, g, W_kmajor, xn_ws, y, M, d, N, N, eps, out_dtype, false, stream);
}

fn_status flashnorm_glu_unfused(const void* x, const void* g, const void* W_kmajor_gu, void* xn_ws, void* y,
                                int64_t M, int64_t d, int64_t F, float eps, int out_dtype, void* stream) {
  g_last_error[0] = '\0';
  if (F < 16 || F > kMaxDim / 2 || F % 16 != 0) return fail(FN_ERR_INVALID_ARG, "F must be a positive multiple of 16");
  return unfused(x, g, W_kmajor_gu, xn_ws, y, M, d, 2 * F, F, eps, out_dtype, true, stream);
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// Unfused baseline without a caller workspace. The scratch for the normalised activations lives in
// this file's device image; host code reaches it only through the address that cudaGetSymbolAddress
// returns on the current device (the symbol itself is a host-side stand-in, not a device pointer).
// ------------------------------------------------------------------------------------------------
static __device__ __align__(256) uint16_t g_noalloc_xn[FN_NOALLOC_MAX_ELEMS];

namespace {

// Device address of g_noalloc_xn on the current device, looked up once per device.
fn_status noalloc_scratch(void** out) {
  static void* addr[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FN_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_xn);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    addr[dev] = p;
  }
  *out = addr[dev];
  return FN_OK;
}

}  // namespace

extern "C" {

fn_status flashnorm_linear_unfused_noalloc(const void* x, const void* g, const void* W_kmajor, void* y, int64_t M,
                                           int64_t d, int64_t N, float eps, int out_dtype, void* stream) {
  g_last_error[0] = '\0';
  if (N < 8 || N > kMaxDim || N % 8 != 0) return fail(FN_ERR_INVALID_ARG, "N must be a positive multiple of 8");
  fn_status st = check_common(x, W_kmajor, y, M, d, eps, out_dtype);
  if (st != FN_OK) return st;
  if (M > 0 && M > FN_NOALLOC_MAX_ELEMS / d)
    return fail(FN_ERR_UNSUPPORTED, "no-alloc scratch holds %lld elements; M * d = %lld is larger",
                (long long)FN_NOALLOC_MAX_ELEMS, (long long)(M * d));
  if (M == 0) return FN_OK;
  void* xn = nullptr;
  if ((st = noalloc_scratch(&xn)) != FN_OK) return st;
  return unfused(x, g, W_kmajor, xn, y, M, d, N, N, eps, out_dtype, false, stream);
}

fn_status flashnorm_check_device_error(void* stream) {
  g_last_error[0] = '\0';
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int h = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&h, fn::g_device_status, sizeof(h), 0, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  if (h != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(fn::g_device_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
    if (h & fn::kStatusTimeout) return fail(FN_ERR_TIMEOUT, "a kernel gave up on a bounded wait");
    if (h & fn::kStatusBadPosition)
      return fail(FN_ERR_INVALID_ARG, "a RoPE position was outside [0, max_pos); those rows were written as NaN");
  }
  return FN_OK;
}

fn_status flashnorm_selftest_timeout(int64_t limit_us, void* stream) {
  g_last_error[0] = '\0';
  if (limit_us < 1 || limit_us > 10000000) return fail(FN_ERR_INVALID_ARG, "limit_us must be in [1, 1e7]");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_kernel(fn::k_wait_selftest, dim3(1), dim3(32), 0, s, 1,
                                static_cast<unsigned long long>(limit_us) * 1000ull);
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return flashnorm_check_device_error(stream);
}

const char* flashnorm_status_string(int status) {
  switch (status) {
    case FN_OK: return "FN_OK";
    case FN_ERR_INVALID_ARG: return "FN_ERR_INVALID_ARG: an argument is out of range";
    case FN_ERR_UNSUPPORTED: return "FN_ERR_UNSUPPORTED: no kernel for this request";
    case FN_ERR_ALIGN: return "FN_ERR_ALIGN: a pointer is not 16-byte aligned";
    case FN_ERR_CUDA: return "FN_ERR_CUDA: a CUDA call failed";
    case FN_ERR_TIMEOUT: return "FN_ERR_TIMEOUT: a device-side wait ran out";
    default: return "unknown status";
  }
}

const char* flashnorm_last_error(void) { return g_last_error; }

int flashnorm_version(void) { return 100; }

}  // extern "C"
