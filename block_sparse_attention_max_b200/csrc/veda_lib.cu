// veda_lib.cu -- the C ABI of include/veda.h: argument checks, launch configuration,
// tensor-map encoding and the per-device status word. Kernels live in k_*.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <string>

#include "../../include/veda.h"
#include "k_attn.cuh"
#include "k_heat.cuh"
#include "k_bwd.cuh"
#include "k_fp8.cuh"
#include "k_gather.cuh"
#include "k_scores.cuh"
#include "k_select.cuh"
#include "veda_ptx.cuh"

namespace veda {

namespace {
thread_local std::string t_last_error;

struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int sms = 0;
  bool attrs_set = false;
  int per_sm_copy = 1, per_sm_unpermute = 1, per_sm_pool = 1, per_sm_permpool = 1;   // resident CTAs per SM
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

// Signature of the driver's cuTensorMapEncodeTiled (obtained through the runtime's
// driver entry-point query, so the library needs no link against libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
}  // namespace

void set_last_error(const std::string& msg) { t_last_error = msg; }

namespace {

veda_status fail(veda_status st, const std::string& msg) {
  set_last_error(msg);
  return st;
}

veda_status cuda_fail(cudaError_t e, const char* what) {
  return fail(VEDA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// Current device: must be compute capability 10.0 (B200). Sets one-time kernel attributes.
veda_status current_device(int& sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(VEDA_ERR_UNSUPPORTED, "device ordinal out of range");
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.probed) {
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    d.supported = (major == 10 && minor == 0);
    d.probed = true;
  }
  if (!d.supported)
    return fail(VEDA_ERR_UNSUPPORTED, "the kernels are built for sm_100a (compute capability 10.0) only");
  if (!d.attrs_set) {
    struct { const void* f; int bytes; } attrs[] = {
        {reinterpret_cast<const void*>(attn::attn_fwd_kernel), static_cast<int>(attn::kSmemBytes)},
        {reinterpret_cast<const void*>(heat::heat_kernel), static_cast<int>(attn::kSmemBytes)},
        {reinterpret_cast<const void*>(fp8::attn_fwd_fp8_kernel), static_cast<int>(fp8::kSmemBytes)},
        {reinterpret_cast<const void*>(bwd::bwd_kernel<bwd::kModeDQ>), static_cast<int>(bwd::kSmemBytesDQ)},
        {reinterpret_cast<const void*>(bwd::bwd_kernel<bwd::kModeDKDV>), static_cast<int>(bwd::kSmemBytesDKDV)},
        {reinterpret_cast<const void*>(sgemm::nt_gemm_3xtf32_kernel), static_cast<int>(sgemm::kSmemBytes)},
        {reinterpret_cast<const void*>(select_kernel), static_cast<int>(kSelMaxSmem)},
    };
    for (auto& x : attrs) {
      e = cudaFuncSetAttribute(x.f, cudaFuncAttributeMaxDynamicSharedMemorySize, x.bytes);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    }
    // the attention kernel re-splits its registers between warpgroups (setmaxnreg); the
    // split assumes the launch allocation it was built for, so refuse any other build
    const void* split_kernels[] = {reinterpret_cast<const void*>(attn::attn_fwd_kernel),
                                   reinterpret_cast<const void*>(heat::heat_kernel),
                                   reinterpret_cast<const void*>(fp8::attn_fwd_fp8_kernel),
                                   reinterpret_cast<const void*>(bwd::bwd_kernel<bwd::kModeDQ>),
                                   reinterpret_cast<const void*>(bwd::bwd_kernel<bwd::kModeDKDV>)};
    for (const void* f : split_kernels) {
      cudaFuncAttributes fa{};
      if ((e = cudaFuncGetAttributes(&fa, f)) != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
      if (fa.numRegs != attn::kLaunchRegs)
        return fail(VEDA_ERR_UNSUPPORTED, "attention/heat kernel built with " + std::to_string(fa.numRegs) +
                                              " registers per thread; its register split needs " +
                                              std::to_string(attn::kLaunchRegs));
    }
    // persistent grids: as many CTAs as can be resident at once
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.per_sm_copy, permute_kernel, kCopyThreads, 0)) != cudaSuccess ||
        (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.per_sm_unpermute, unpermute_kernel, kCopyThreads, 0)) != cudaSuccess ||
        (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.per_sm_pool, pool_kernel, kPoolThreads, 0)) != cudaSuccess ||
        (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.per_sm_permpool, permute_pool_kernel, kPoolThreads, 0)) != cudaSuccess)
      return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    d.per_sm_copy = d.per_sm_copy < 1 ? 1 : d.per_sm_copy;
    d.per_sm_unpermute = d.per_sm_unpermute < 1 ? 1 : d.per_sm_unpermute;
    d.per_sm_pool = d.per_sm_pool < 1 ? 1 : d.per_sm_pool;
    d.per_sm_permpool = d.per_sm_permpool < 1 ? 1 : d.per_sm_permpool;
    d.attrs_set = true;
  }
  sms = d.sms;
  return VEDA_OK;
}

const DeviceInfo& device_info() {
  int dev = 0;
  cudaGetDevice(&dev);
  return g_dev[dev];
}

// The library's second stream of the current device and a fork / join event pair, created on
// first use and kept until exit (the backward runs its two independent kernels on both).
veda_status side_stream(cudaStream_t& s, cudaEvent_t& fork, cudaEvent_t& join) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(VEDA_ERR_UNSUPPORTED, "device ordinal out of range");
  static cudaStream_t streams[kMaxDevices] = {};
  static cudaEvent_t forks[kMaxDevices] = {}, joins[kMaxDevices] = {};
  std::lock_guard<std::mutex> lk(g_mu);
  if (streams[dev] == nullptr) {
    if ((e = cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&forks[dev], cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&joins[dev], cudaEventDisableTiming)) != cudaSuccess)
      return cuda_fail(e, "side stream");
  }
  s = streams[dev];
  fork = forks[dev];
  join = joins[dev];
  return VEDA_OK;
}

veda_status get_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return VEDA_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
    return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found");
  g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  return VEDA_OK;
}

// 2D map over rows of 128 bf16 (256 B): box 64 columns x 128 rows, 128-byte swizzle.
veda_status encode_rows(CUtensorMap& m, const void* base, uint64_t rows) {
  const cuuint64_t dims[2] = {128, rows};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(r) + ")");
  return VEDA_OK;
}

// e4m3 tiles: rows of 128 bytes, one 128 x 128 box per tile, 128-byte swizzle
veda_status encode_rows8(CUtensorMap& m, const void* base, uint64_t rows) {
  const cuuint64_t dims[2] = {128, rows};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(r) + ")");
  return VEDA_OK;
}

// fp32 matrix of `cols` columns (row stride cols * 4 bytes, a multiple of 16) and `rows` rows:
// box 32 columns (128 bytes) x 128 rows, 128-byte swizzle. Rows past the end read as zero.
veda_status encode_f32_rows(CUtensorMap& m, const void* base, uint64_t cols, uint64_t rows) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 4};
  const cuuint32_t box[2] = {32, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(&m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(r) + ")");
  return VEDA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

veda_status launched(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return VEDA_OK;
}

int grid_for(int64_t units, int sms, int per_sm) {
  const int64_t g = static_cast<int64_t>(sms) * per_sm;
  return static_cast<int>(units < g ? units : g);
}

}  // namespace
}  // namespace veda

using namespace veda;

extern "C" {

int32_t veda_abi_version(void) { return VEDA_ABI_VERSION; }

const char* veda_status_string(veda_status s) {
  switch (s) {
    case VEDA_OK: return "ok";
    case VEDA_ERR_INVALID_ARG: return "invalid argument";
    case VEDA_ERR_UNSUPPORTED: return "unsupported device or shape";
    case VEDA_ERR_CUDA: return "CUDA error";
    case VEDA_ERR_TIMEOUT: return "a kernel wait timed out";
    case VEDA_ERR_DEVICE_CHECK: return "a kernel found invalid data";
  }
  return "unknown status";
}

const char* veda_last_error(void) { return t_last_error.c_str(); }

veda_status veda_permute_tiles(const void* x, void* x_tiled, const int32_t* tile_map, int32_t B,
                               int32_t N, int32_t H, int32_t D, int32_t Npad, veda_stream_t stream) {
  if (!x || !x_tiled || !tile_map || B <= 0 || N <= 0 || H <= 0 || Npad <= 0 || Npad % 128)
    return fail(VEDA_ERR_INVALID_ARG, "veda_permute_tiles: bad pointer or size");
  if (D != 128) return fail(VEDA_ERR_UNSUPPORTED, "head_dim must be 128");
  if (!aligned(x, 16) || !aligned(x_tiled, 16)) return fail(VEDA_ERR_INVALID_ARG, "veda_permute_tiles: buffers must be 16-byte aligned");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  GatherArgs a{static_cast<const uint8_t*>(x), static_cast<uint8_t*>(x_tiled), tile_map, B, N, H, Npad,
               Npad / 128, static_cast<int64_t>(B) * H * (Npad / 128)};
  permute_kernel<<<grid_for(a.units, sms, device_info().per_sm_copy), kCopyThreads, 0,
                   reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return launched("permute_kernel");
}

veda_status veda_permute_pool(const void* x, void* x_tiled, const int32_t* tile_map, const int32_t* tile_valid,
                              float* pooled, int32_t B, int32_t N, int32_t H, int32_t D, int32_t Npad,
                              veda_stream_t stream) {
  if (!x || !x_tiled || !tile_map || !tile_valid || !pooled || B <= 0 || N <= 0 || H <= 0 || Npad <= 0 ||
      Npad % 128)
    return fail(VEDA_ERR_INVALID_ARG, "veda_permute_pool: bad pointer or size");
  if (D != 128) return fail(VEDA_ERR_UNSUPPORTED, "head_dim must be 128");
  if (!aligned(x, 16) || !aligned(x_tiled, 16) || !aligned(pooled, 4))
    return fail(VEDA_ERR_INVALID_ARG, "veda_permute_pool: misaligned buffer");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  PermPoolArgs p{{static_cast<const uint8_t*>(x), static_cast<uint8_t*>(x_tiled), tile_map, B, N, H, Npad,
                  Npad / 128, static_cast<int64_t>(B) * H * (Npad / 128)},
                 tile_valid, pooled};
  const int64_t pp_ctas = (p.g.units + kPoolThreads / 32 - 1) / (kPoolThreads / 32);
  permute_pool_kernel<<<grid_for(pp_ctas, sms, device_info().per_sm_permpool), kPoolThreads, 0,
                        reinterpret_cast<cudaStream_t>(stream)>>>(p);
  return launched("permute_pool_kernel");
}

veda_status veda_unpermute(const void* o_tiled, void* o, const int32_t* tile_map, int32_t B, int32_t N,
                           int32_t H, int32_t D, int32_t Npad, veda_stream_t stream) {
  if (!o_tiled || !o || !tile_map || B <= 0 || N <= 0 || H <= 0 || Npad <= 0 || Npad % 128)
    return fail(VEDA_ERR_INVALID_ARG, "veda_unpermute: bad pointer or size");
  if (D != 128) return fail(VEDA_ERR_UNSUPPORTED, "head_dim must be 128");
  if (!aligned(o, 16) || !aligned(o_tiled, 16)) return fail(VEDA_ERR_INVALID_ARG, "veda_unpermute: buffers must be 16-byte aligned");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  GatherArgs a{static_cast<const uint8_t*>(o_tiled), static_cast<uint8_t*>(o), tile_map, B, N, H, Npad,
               Npad / 128, static_cast<int64_t>(B) * H * (Npad / 128)};
  unpermute_kernel<<<grid_for(a.units, sms, device_info().per_sm_unpermute), kCopyThreads, 0,
                     reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return launched("unpermute_kernel");
}

veda_status veda_tile_pool(const void* x_tiled, const int32_t* tile_valid, float* pooled, int32_t B,
                           int32_t H, int32_t nT, int32_t D, veda_stream_t stream) {
  if (!x_tiled || !tile_valid || !pooled || B <= 0 || H <= 0 || nT <= 0)
    return fail(VEDA_ERR_INVALID_ARG, "veda_tile_pool: bad pointer or size");
  if (D != 128) return fail(VEDA_ERR_UNSUPPORTED, "head_dim must be 128");
  if (!aligned(x_tiled, 16) || !aligned(pooled, 4)) return fail(VEDA_ERR_INVALID_ARG, "veda_tile_pool: misaligned buffer");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  PoolArgs a{static_cast<const uint8_t*>(x_tiled), tile_valid, pooled, B, H, nT,
             static_cast<int64_t>(B) * H * nT};
  const int64_t pool_ctas = (a.units + kPoolThreads / 32 - 1) / (kPoolThreads / 32);
  pool_kernel<<<grid_for(pool_ctas, sms, device_info().per_sm_pool), kPoolThreads, 0,
                reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return launched("pool_kernel");
}

size_t veda_block_scores_workspace_bytes(int32_t B, int32_t H, int32_t nT, int32_t D) {
  if (B <= 0 || H <= 0 || nT <= 0 || D <= 0) return 0;
  return static_cast<size_t>(2) * B * H * nT * D * sizeof(float);
}

veda_status veda_block_scores(const float* pooled_q, const float* pooled_k, const float* Wq, const float* Wk,
                              float* scores, void* workspace, size_t workspace_bytes, int32_t B, int32_t H,
                              int32_t nT, int32_t D, veda_stream_t stream) {
  if (!pooled_q || !pooled_k || !Wq || !Wk || !scores || !workspace || B <= 0 || H <= 0 || nT <= 0)
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_scores: bad pointer or size");
  if (D != 128) return fail(VEDA_ERR_UNSUPPORTED, "head_dim must be 128");
  if (workspace_bytes < veda_block_scores_workspace_bytes(B, H, nT, D))
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_scores: workspace too small");
  if (!aligned(pooled_q, 16) || !aligned(pooled_k, 16) || !aligned(Wq, 16) || !aligned(Wk, 16) ||
      !aligned(workspace, 256))
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_scores: misaligned buffer");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  if ((st = get_encoder()) != VEDA_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* hat = static_cast<float*>(workspace);             // [2][B][H][nT][128]: qhat, khat
  const int64_t BH = static_cast<int64_t>(B) * H;
  const int32_t tiles_m = (nT + 127) / 128;
  // projection: hat[which] = mean + pooled . W^T   (M = nT, N = 128, K = 384)
  CUtensorMap mPq, mPk, mWq, mWk;
  if ((st = encode_f32_rows(mPq, pooled_q, 384, static_cast<uint64_t>(BH) * nT)) != VEDA_OK ||
      (st = encode_f32_rows(mPk, pooled_k, 384, static_cast<uint64_t>(BH) * nT)) != VEDA_OK ||
      (st = encode_f32_rows(mWq, Wq, 384, static_cast<uint64_t>(H) * 128)) != VEDA_OK ||
      (st = encode_f32_rows(mWk, Wk, 384, static_cast<uint64_t>(H) * 128)) != VEDA_OK)
    return st;
  sgemm::Args p{};
  p.mode = sgemm::kModeProject;
  p.nT = nT; p.N = 128; p.k_chunks = 384 / 32;
  p.tiles_m = tiles_m; p.tiles_n = 1;
  p.BH = static_cast<int32_t>(BH); p.H = H;
  p.tiles = 2 * BH * tiles_m;
  p.out = hat;
  sgemm::nt_gemm_3xtf32_kernel<<<grid_for(p.tiles, sms, 1), sgemm::kThreads, sgemm::kSmemBytes, s>>>(
      mPq, mPk, mWq, mWk, p);
  st = launched("projection");
  if (st != VEDA_OK) return st;
  // scores = qhat . khat^T  (M = N = nT, K = 128)
  CUtensorMap mHat;
  if ((st = encode_f32_rows(mHat, hat, 128, static_cast<uint64_t>(2 * BH) * nT)) != VEDA_OK) return st;
  sgemm::Args q{};
  q.mode = sgemm::kModeScores;
  q.nT = nT; q.N = nT; q.k_chunks = 128 / 32;
  q.tiles_m = tiles_m; q.tiles_n = tiles_m;
  q.BH = static_cast<int32_t>(BH); q.H = H;
  q.tiles = BH * tiles_m * tiles_m;
  q.out = scores;
  sgemm::nt_gemm_3xtf32_kernel<<<grid_for(q.tiles, sms, 1), sgemm::kThreads, sgemm::kSmemBytes, s>>>(
      mHat, mHat, mHat, mHat, q);
  return launched("scores");
}

// Scratch of veda_block_scores_noalloc: part of the library's device image, so no call
// ever allocates. Host code must not pass `g_noalloc_scratch` itself to a kernel (on the
// host it is only a stand-in symbol); its device address is looked up once per device and
// context, with that device current, and cached together with the context it belongs to.
static __device__ __align__(256) unsigned char g_noalloc_scratch[VEDA_NOALLOC_SCORES_BYTES];
struct NoallocSlot {
  CUcontext ctx;   // context the address was looked up in
  void* ptr;       // device address of g_noalloc_scratch in that context
};
static NoallocSlot g_noalloc[kMaxDevices] = {};
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
static CtxGetCurrentFn g_ctx_current = nullptr;

// Current context of the calling thread (null before the runtime has created one).
static veda_status current_context(CUcontext& ctx) {
  if (g_ctx_current == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
      return fail(VEDA_ERR_CUDA, "cuCtxGetCurrent entry point not found");
    g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(fn);
  }
  ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS) return fail(VEDA_ERR_CUDA, "cuCtxGetCurrent failed");
  return VEDA_OK;
}

veda_status veda_block_scores_noalloc(const float* pooled_q, const float* pooled_k, const float* Wq,
                                      const float* Wk, float* scores, int32_t B, int32_t H, int32_t nT,
                                      int32_t D, veda_stream_t stream) {
  if (B <= 0 || H <= 0 || nT <= 0)
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_scores_noalloc: bad size");
  const size_t need = veda_block_scores_workspace_bytes(B, H, nT, D);
  if (need > VEDA_NOALLOC_SCORES_BYTES)
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_scores_noalloc: 2*B*H*nT*D*4 = " + std::to_string(need) +
                                          " bytes exceeds the built-in scratch of " +
                                          std::to_string(VEDA_NOALLOC_SCORES_BYTES) + " bytes");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(VEDA_ERR_UNSUPPORTED, "device ordinal out of range");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    CUcontext ctx = nullptr;
    veda_status st = current_context(ctx);
    if (st != VEDA_OK) return st;
    NoallocSlot& slot = g_noalloc[dev];
    if (slot.ptr == nullptr || ctx == nullptr || slot.ctx != ctx) {
      // first call on this device, or its context was replaced (e.g. after a device reset,
      // which reloads the library's module): look the address up again, `dev` current
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || p == nullptr) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
      if ((st = current_context(ctx)) != VEDA_OK) return st;
      slot.ctx = ctx;
      slot.ptr = p;
    }
    scratch = slot.ptr;
  }
  return veda_block_scores(pooled_q, pooled_k, Wq, Wk, scores, scratch, VEDA_NOALLOC_SCORES_BYTES, B, H, nT, D,
                           stream);
}

veda_status veda_select_blocks(const float* scores, const int32_t* tile_valid, const int32_t* tile_segment,
                               const int32_t* nT_per_head, int32_t n_segments, const int32_t* rho_num,
                               const int32_t* rho_den, int32_t* full_cnt, int32_t* full_idx, int32_t* part_cnt,
                               int32_t* part_idx, int32_t list_stride, int32_t B, int32_t H, int32_t nT,
                               veda_stream_t stream) {
  if (!scores || !tile_valid || !tile_segment || !nT_per_head || !rho_num || !rho_den || !full_cnt ||
      !full_idx || !part_cnt || !part_idx || B <= 0 || H <= 0 || nT <= 0)
    return fail(VEDA_ERR_INVALID_ARG, "veda_select_blocks: bad pointer or size");
  if (nT > VEDA_MAX_TILES) return fail(VEDA_ERR_INVALID_ARG, "veda_select_blocks: nT above VEDA_MAX_TILES");
  if (n_segments < 1 || n_segments > VEDA_MAX_SEGMENTS)
    return fail(VEDA_ERR_INVALID_ARG, "veda_select_blocks: n_segments out of range");
  int64_t bound = 1;
  for (int s = 0; s < n_segments; ++s) {
    if (rho_den[s] < 1 || rho_num[s] < 0 || rho_num[s] > rho_den[s])
      return fail(VEDA_ERR_INVALID_ARG, "veda_select_blocks: density must be num/den with 0 <= num <= den");
    bound += (static_cast<int64_t>(nT) * rho_num[s] + rho_den[s] - 1) / rho_den[s];
  }
  if (bound > nT) bound = nT;
  if (list_stride < bound)
    return fail(VEDA_ERR_INVALID_ARG, "veda_select_blocks: list_stride below the largest possible row budget");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  SelectArgs a{};
  a.scores = scores; a.valid = tile_valid; a.segment = tile_segment; a.nT_per_head = nT_per_head;
  a.full_cnt = full_cnt; a.full_idx = full_idx; a.part_cnt = part_cnt; a.part_idx = part_idx;
  a.stride = list_stride; a.B = B; a.H = H; a.nT = nT; a.n_seg = n_segments;
  for (int s = 0; s < kMaxSeg; ++s) {
    a.rho_num[s] = s < n_segments ? rho_num[s] : 0;
    a.rho_den[s] = s < n_segments ? rho_den[s] : 1;
  }
  const int64_t rows = static_cast<int64_t>(B) * H * nT;
  if (rows > INT32_MAX) return fail(VEDA_ERR_INVALID_ARG, "veda_select_blocks: too many rows");
  select_kernel<<<static_cast<unsigned>((rows + kSelWarps - 1) / kSelWarps), kSelThreads,
                  kSelWarps * sel_warp_bytes(nT, n_segments), reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return launched("select_kernel");
}

veda_status veda_block_sparse_attn_fwd(const void* q, const void* k, const void* v, const int32_t* tile_valid,
                                       const int32_t* full_cnt, const int32_t* full_idx, const int32_t* part_cnt,
                                       const int32_t* part_idx, int32_t list_stride, float softmax_scale, void* o,
                                       float* lse, int32_t B, int32_t H, int32_t nT, int32_t D,
                                       veda_stream_t stream) {
  if (!q || !k || !v || !tile_valid || !full_cnt || !full_idx || !part_cnt || !part_idx || !o || B <= 0 ||
      H <= 0 || nT <= 0 || list_stride <= 0)
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_sparse_attn_fwd: bad pointer or size");
  if (D != 128) return fail(VEDA_ERR_UNSUPPORTED, "head_dim must be 128");
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_sparse_attn_fwd: softmax_scale must be positive and finite");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16))
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_sparse_attn_fwd: Q/K/V/O must be 16-byte aligned");
  const int64_t rows = static_cast<int64_t>(B) * H * nT * 128;
  if (rows > INT32_MAX) return fail(VEDA_ERR_INVALID_ARG, "veda_block_sparse_attn_fwd: too many rows");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  if ((st = get_encoder()) != VEDA_OK) return st;
  CUtensorMap tq, tk, tv;
  if ((st = encode_rows(tq, q, rows)) != VEDA_OK) return st;
  if ((st = encode_rows(tk, k, rows)) != VEDA_OK) return st;
  if ((st = encode_rows(tv, v, rows)) != VEDA_OK) return st;
  attn::Args a{};
  a.valid = tile_valid; a.full_cnt = full_cnt; a.full_idx = full_idx; a.part_cnt = part_cnt; a.part_idx = part_idx;
  a.o = static_cast<__nv_bfloat16*>(o); a.lse = lse;
  a.stride = list_stride; a.H = H; a.nT = nT;
  a.items = static_cast<int64_t>(B) * H * nT;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  attn::attn_fwd_kernel<<<grid_for(a.items, sms, 1), attn::kThreads, attn::kSmemBytes,
                          reinterpret_cast<cudaStream_t>(stream)>>>(tq, tk, tv, a);
  return launched("attn_fwd_kernel");
}

veda_status veda_quantize_fp8(const void* x_tiled, void* codes, float* scale, int32_t B, int32_t H, int32_t nT,
                             int32_t D, int32_t transpose_tiles, veda_stream_t stream) {
  if (!x_tiled || !codes || !scale || B <= 0 || H <= 0 || nT <= 0)
    return fail(VEDA_ERR_INVALID_ARG, "veda_quantize_fp8: bad pointer or size");
  if (D != 128) return fail(VEDA_ERR_UNSUPPORTED, "head_dim must be 128");
  if (transpose_tiles != 0 && transpose_tiles != 1)
    return fail(VEDA_ERR_INVALID_ARG, "veda_quantize_fp8: transpose_tiles must be 0 or 1");
  if (!aligned(x_tiled, 16) || !aligned(codes, 16) || !aligned(scale, 4))
    return fail(VEDA_ERR_INVALID_ARG, "veda_quantize_fp8: x_tiled / codes must be 16-byte aligned");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t bh = static_cast<int64_t>(B) * H;
  cudaError_t e = cudaMemsetAsync(scale, 0, static_cast<size_t>(bh) * sizeof(float), s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(scale)");
  fp8::QuantArgs q{};
  q.x = static_cast<const __nv_bfloat16*>(x_tiled);
  q.codes = static_cast<uint8_t*>(codes);
  q.amax_bits = reinterpret_cast<uint32_t*>(scale);
  q.scale = scale;
  q.bh = bh;
  q.rows = static_cast<int64_t>(nT) * 128;
  q.transpose = transpose_tiles;
  const int64_t chunks = (q.rows * 128 + fp8::kAmaxChunk - 1) / fp8::kAmaxChunk;
  fp8::amax_kernel<<<grid_for(bh * chunks, sms, 8), fp8::kQuantThreads, 0, s>>>(q);
  if ((st = launched("amax_kernel")) != VEDA_OK) return st;
  fp8::quant_kernel<<<grid_for(bh * nT, sms, 8), fp8::kQuantThreads, 0, s>>>(q);
  if ((st = launched("quant_kernel")) != VEDA_OK) return st;
  fp8::scale_kernel<<<static_cast<int>((bh + 255) / 256), 256, 0, s>>>(q.amax_bits, bh);
  return launched("scale_kernel");
}

veda_status veda_block_sparse_attn_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* q_scale,
                                           const float* k_scale, const float* v_scale, const int32_t* tile_valid,
                                           const int32_t* full_cnt, const int32_t* full_idx,
                                           const int32_t* part_cnt, const int32_t* part_idx, int32_t list_stride,
                                           float softmax_scale, void* o, float* lse, int32_t B, int32_t H,
                                           int32_t nT, int32_t D, veda_stream_t stream) {
  if (!q8 || !k8 || !vt8 || !q_scale || !k_scale || !v_scale || !tile_valid || !full_cnt || !full_idx ||
      !part_cnt || !part_idx || !o || B <= 0 || H <= 0 || nT <= 0 || list_stride <= 0)
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_sparse_attn_fwd_fp8: bad pointer or size");
  if (D != 128) return fail(VEDA_ERR_UNSUPPORTED, "head_dim must be 128");
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_sparse_attn_fwd_fp8: softmax_scale must be positive and finite");
  if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(vt8, 16) || !aligned(o, 16))
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_sparse_attn_fwd_fp8: Q/K/V codes and O must be 16-byte aligned");
  const int64_t rows = static_cast<int64_t>(B) * H * nT * 128;
  if (rows > INT32_MAX) return fail(VEDA_ERR_INVALID_ARG, "veda_block_sparse_attn_fwd_fp8: too many rows");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  if ((st = get_encoder()) != VEDA_OK) return st;
  CUtensorMap tq, tk, tv;
  if ((st = encode_rows8(tq, q8, rows)) != VEDA_OK) return st;
  if ((st = encode_rows8(tk, k8, rows)) != VEDA_OK) return st;
  if ((st = encode_rows8(tv, vt8, rows)) != VEDA_OK) return st;
  fp8::Args p{};
  p.a.valid = tile_valid; p.a.full_cnt = full_cnt; p.a.full_idx = full_idx; p.a.part_cnt = part_cnt;
  p.a.part_idx = part_idx; p.a.o = static_cast<__nv_bfloat16*>(o); p.a.lse = lse;
  p.a.stride = list_stride; p.a.H = H; p.a.nT = nT;
  p.a.items = static_cast<int64_t>(B) * H * nT;
  p.a.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.q_scale = q_scale; p.k_scale = k_scale; p.v_scale = v_scale;
  fp8::attn_fwd_fp8_kernel<<<grid_for(p.a.items, sms, 1), fp8::kThreads, fp8::kSmemBytes,
                              reinterpret_cast<cudaStream_t>(stream)>>>(tq, tk, tv, p);
  return launched("attn_fwd_fp8_kernel");
}

veda_status veda_block_heat(const void* q, const void* k, const int32_t* tile_valid, const int32_t* full_cnt,
                            const int32_t* full_idx, const int32_t* part_cnt, const int32_t* part_idx,
                            int32_t list_stride, const float* lse, float softmax_scale, float* heat, int32_t B,
                            int32_t H, int32_t nT, int32_t D, veda_stream_t stream) {
  if (!q || !k || !tile_valid || !full_cnt || !full_idx || !part_cnt || !part_idx || !lse || !heat || B <= 0 ||
      H <= 0 || nT <= 0 || list_stride <= 0)
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_heat: bad pointer or size");
  if (D != 128) return fail(VEDA_ERR_UNSUPPORTED, "head_dim must be 128");
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_heat: softmax_scale must be positive and finite");
  if (!aligned(q, 16) || !aligned(k, 16))
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_heat: Q/K must be 16-byte aligned");
  const int64_t rows = static_cast<int64_t>(B) * H * nT * 128;
  if (rows > INT32_MAX) return fail(VEDA_ERR_INVALID_ARG, "veda_block_heat: too many rows");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  if ((st = get_encoder()) != VEDA_OK) return st;
  CUtensorMap tq, tk;
  if ((st = encode_rows(tq, q, rows)) != VEDA_OK) return st;
  if ((st = encode_rows(tk, k, rows)) != VEDA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t heat_bytes = static_cast<size_t>(B) * H * nT * nT * sizeof(float);
  cudaError_t e = cudaMemsetAsync(heat, 0, heat_bytes, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(heat)");
  heat::HeatArgs p{};
  p.a.valid = tile_valid; p.a.full_cnt = full_cnt; p.a.full_idx = full_idx; p.a.part_cnt = part_cnt;
  p.a.part_idx = part_idx; p.a.stride = list_stride; p.a.H = H; p.a.nT = nT;
  p.a.items = static_cast<int64_t>(B) * H * nT;
  p.lse = lse;
  p.heat = heat;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  heat::heat_kernel<<<grid_for(p.a.items, sms, 1), attn::kThreads, attn::kSmemBytes, s>>>(tq, tk, p);
  return launched("heat_kernel");
}

veda_status veda_mask_quality(const float* heat, const int32_t* tile_valid, const int32_t* nT_per_head,
                              const int32_t* pred_full_cnt, const int32_t* pred_full_idx,
                              const int32_t* pred_part_cnt, const int32_t* pred_part_idx, int32_t pred_stride,
                              const int32_t* orc_full_cnt, const int32_t* orc_full_idx,
                              const int32_t* orc_part_cnt, const int32_t* orc_part_idx, int32_t orc_stride,
                              float* mass_rows, float* recall_rows, float* totals, int32_t B, int32_t H,
                              int32_t nT, veda_stream_t stream) {
  if (!heat || !tile_valid || !nT_per_head || !pred_full_cnt || !pred_full_idx || !pred_part_cnt ||
      !pred_part_idx || !orc_full_cnt || !orc_full_idx || !orc_part_cnt || !orc_part_idx || !mass_rows ||
      !recall_rows || !totals || B <= 0 || H <= 0 || nT <= 0 || pred_stride <= 0 || orc_stride <= 0)
    return fail(VEDA_ERR_INVALID_ARG, "veda_mask_quality: bad pointer or size");
  if (nT > heat::kQualMaxTiles) return fail(VEDA_ERR_INVALID_ARG, "veda_mask_quality: nT exceeds VEDA_MAX_TILES");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(totals, 0, 4 * sizeof(float), s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(totals)");
  heat::QualityArgs qa{};
  qa.heat = heat; qa.valid = tile_valid; qa.nT_per_head = nT_per_head;
  qa.pfc = pred_full_cnt; qa.pfi = pred_full_idx; qa.ppc = pred_part_cnt; qa.ppi = pred_part_idx;
  qa.ofc = orc_full_cnt; qa.ofi = orc_full_idx; qa.opc = orc_part_cnt; qa.opi = orc_part_idx;
  qa.pstride = pred_stride; qa.ostride = orc_stride;
  qa.mass_rows = mass_rows; qa.recall_rows = recall_rows; qa.totals = totals;
  qa.H = H; qa.nT = nT;
  qa.rows = static_cast<int64_t>(B) * H * nT;
  const int64_t blocks = (qa.rows + heat::kQualWarps - 1) / heat::kQualWarps;
  if (blocks > INT32_MAX) return fail(VEDA_ERR_INVALID_ARG, "veda_mask_quality: too many rows");
  heat::mask_quality_kernel<<<static_cast<unsigned>(blocks), 32 * heat::kQualWarps, 0, s>>>(qa);
  return launched("mask_quality_kernel");
}

veda_status veda_transpose_lists(const int32_t* full_cnt, const int32_t* full_idx, const int32_t* part_cnt,
                                 const int32_t* part_idx, int32_t list_stride, const int32_t* nT_per_head,
                                 int32_t* t_cnt, int32_t* t_idx, int32_t t_stride, int32_t B, int32_t H, int32_t nT,
                                 veda_stream_t stream) {
  if (!full_cnt || !full_idx || !part_cnt || !part_idx || !nT_per_head || !t_cnt || !t_idx || B <= 0 || H <= 0 ||
      nT <= 0 || list_stride <= 0 || t_stride <= 0)
    return fail(VEDA_ERR_INVALID_ARG, "veda_transpose_lists: bad pointer or size");
  if (t_stride < nT && t_stride < list_stride)
    return fail(VEDA_ERR_INVALID_ARG, "veda_transpose_lists: t_stride must be >= nT");
  const int64_t rows = static_cast<int64_t>(B) * H * nT;
  const int64_t blocks = (rows + 3) / 4;
  if (blocks > INT32_MAX) return fail(VEDA_ERR_INVALID_ARG, "veda_transpose_lists: too many rows");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  bwd::transpose_lists_kernel<<<static_cast<unsigned>(blocks), 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      full_cnt, full_idx, part_cnt, part_idx, list_stride, nT_per_head, t_cnt, t_idx, t_stride, H, nT, rows);
  return launched("transpose_lists_kernel");
}

veda_status veda_block_sparse_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                       const float* lse, const int32_t* tile_valid, const int32_t* full_cnt,
                                       const int32_t* full_idx, const int32_t* part_cnt, const int32_t* part_idx,
                                       int32_t list_stride, const int32_t* t_cnt, const int32_t* t_idx,
                                       int32_t t_stride, float softmax_scale, void* dq, void* dk, void* dv,
                                       float* delta, int32_t B, int32_t H, int32_t nT, int32_t D,
                                       veda_stream_t stream) {
  if (!q || !k || !v || !o || !dout || !lse || !tile_valid || !full_cnt || !full_idx || !part_cnt || !part_idx ||
      !t_cnt || !t_idx || !dq || !dk || !dv || !delta || B <= 0 || H <= 0 || nT <= 0 || list_stride <= 0 ||
      t_stride <= 0)
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_sparse_attn_bwd: bad pointer or size");
  if (D != 128) return fail(VEDA_ERR_UNSUPPORTED, "head_dim must be 128");
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_sparse_attn_bwd: softmax_scale must be positive and finite");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 16) || !aligned(delta, 16))
    return fail(VEDA_ERR_INVALID_ARG, "veda_block_sparse_attn_bwd: tensors must be 16-byte aligned");
  const int64_t rows = static_cast<int64_t>(B) * H * nT * 128;
  if (rows > INT32_MAX) return fail(VEDA_ERR_INVALID_ARG, "veda_block_sparse_attn_bwd: too many rows");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  if ((st = get_encoder()) != VEDA_OK) return st;
  CUtensorMap tq, tk, tv, tdo;
  if ((st = encode_rows(tq, q, rows)) != VEDA_OK) return st;
  if ((st = encode_rows(tk, k, rows)) != VEDA_OK) return st;
  if ((st = encode_rows(tv, v, rows)) != VEDA_OK) return st;
  if ((st = encode_rows(tdo, dout, rows)) != VEDA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the two kernels' work-queue counters live after the B*H*nT*128 values of D
  int32_t* counters = reinterpret_cast<int32_t*>(delta + rows);
  cudaError_t ce = cudaMemsetAsync(counters, 0, 2 * sizeof(int32_t), s);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaMemsetAsync(work counters)");
  // D = rowsum(dO * O)
  const int64_t dblocks = std::min<int64_t>((rows + 15) / 16, static_cast<int64_t>(sms) * 16);
  bwd::delta_kernel<<<static_cast<unsigned>(dblocks), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(o), delta, rows);
  if ((st = launched("delta_kernel")) != VEDA_OK) return st;
  bwd::Args a{};
  a.valid = tile_valid;
  a.lse = lse;
  a.delta = delta;
  a.H = H;
  a.nT = nT;
  a.items = static_cast<int64_t>(B) * H * nT;
  a.scale = softmax_scale;
  a.next_item = counters;
  const unsigned grid = grid_for(a.items, sms, 1);
  // The two kernels are independent and each holds a whole SM per CTA. dK/dV (uneven items:
  // a key tile is listed by 0 to hundreds of query tiles) goes first on the caller's stream,
  // dQ on the library's second stream of this device, so that dQ's CTAs start on the SMs that
  // dK/dV's last items leave idle; the caller's stream then waits for both.
  cudaStream_t aux;
  cudaEvent_t ev_fork, ev_join;
  if ((st = side_stream(aux, ev_fork, ev_join)) != VEDA_OK) return st;
  // the fork / join events are shared by the device's calls: enqueue one call at a time
  static std::mutex fork_mu;
  std::lock_guard<std::mutex> fork_lk(fork_mu);
  if ((ce = cudaEventRecord(ev_fork, s)) != cudaSuccess) return cuda_fail(ce, "cudaEventRecord");
  if ((ce = cudaStreamWaitEvent(aux, ev_fork, 0)) != cudaSuccess) return cuda_fail(ce, "cudaStreamWaitEvent");
  // dK, dV: key tiles over the transposed lists (fixed K, V; streamed Q, dO)
  bwd::Args t = a;
  t.full_cnt = t_cnt; t.full_idx = t_idx; t.part_cnt = nullptr; t.part_idx = nullptr;
  t.stride = t_stride;
  t.out0 = static_cast<__nv_bfloat16*>(dv);
  t.out1 = static_cast<__nv_bfloat16*>(dk);
  t.next_item = counters + 1;
  bwd::bwd_kernel<bwd::kModeDKDV><<<grid, bwd::kThreads, bwd::kSmemBytesDKDV, s>>>(tk, tv, tq, tdo, t);
  if ((st = launched("bwd_kernel<dK,dV>")) != VEDA_OK) return st;
  // dQ: query tiles over the forward lists (fixed Q, dO; streamed K, V)
  a.full_cnt = full_cnt; a.full_idx = full_idx; a.part_cnt = part_cnt; a.part_idx = part_idx;
  a.stride = list_stride;
  a.out0 = static_cast<__nv_bfloat16*>(dq);
  a.out1 = nullptr;
  bwd::bwd_kernel<bwd::kModeDQ><<<grid, bwd::kThreads, bwd::kSmemBytesDQ, aux>>>(tq, tdo, tk, tv, a);
  if ((st = launched("bwd_kernel<dQ>")) != VEDA_OK) return st;
  if ((ce = cudaEventRecord(ev_join, aux)) != cudaSuccess) return cuda_fail(ce, "cudaEventRecord");
  if ((ce = cudaStreamWaitEvent(s, ev_join, 0)) != cudaSuccess) return cuda_fail(ce, "cudaStreamWaitEvent");
  return VEDA_OK;
}

veda_status veda_rel_error(const void* o, const void* o_ref, float* sums, int32_t B, int32_t N, int32_t H,
                           int32_t D, veda_stream_t stream) {
  if (!o || !o_ref || !sums || B <= 0 || N <= 0 || H <= 0)
    return fail(VEDA_ERR_INVALID_ARG, "veda_rel_error: bad pointer or size");
  if (D != 128) return fail(VEDA_ERR_UNSUPPORTED, "head_dim must be 128");
  if (H > heat::kErrMaxHeads) return fail(VEDA_ERR_INVALID_ARG, "veda_rel_error: too many heads");
  if (!aligned(o, 16) || !aligned(o_ref, 16) || !aligned(sums, 4))
    return fail(VEDA_ERR_INVALID_ARG, "veda_rel_error: misaligned buffer");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(sums, 0, 2 * sizeof(float) * H, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(sums)");
  const int64_t rows = static_cast<int64_t>(B) * N * H;
  const int64_t blocks = std::min<int64_t>((rows + 15) / 16, static_cast<int64_t>(sms) * 8);
  heat::rel_error_kernel<<<static_cast<unsigned>(blocks), heat::kErrThreads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(o_ref), sums, rows, H);
  return launched("rel_error_kernel");
}

// Self-test of the bounded waits: one thread waits on an mbarrier that nothing arrives
// on; the wait gives up after `limit_ns`, records the timeout and the kernel returns.
__global__ void wait_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  mbar_init(smem_u32(&bar), 1);
  fence_mbar_init();
  mbar_wait(smem_u32(&bar), 0, nullptr, 0xEE, limit_ns);
}

veda_status veda_selftest_wait_timeout(uint32_t limit_us, veda_stream_t stream) {
  if (limit_us == 0 || limit_us > 1000000)
    return fail(VEDA_ERR_INVALID_ARG, "veda_selftest_wait_timeout: limit must be 1..1000000 us");
  int sms;
  veda_status st = current_device(sms);
  if (st != VEDA_OK) return st;
  wait_selftest_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t>(limit_us) * 1000u);
  return launched("wait_selftest_kernel");
}

veda_status veda_check_device_status(veda_stream_t stream, uint32_t* detail) {
  if (detail) *detail = 0;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "read status word");
  if (v) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "clear status word");
  }
  if (detail) *detail = v;
  if (v & ST_TIMEOUT) return fail(VEDA_ERR_TIMEOUT, "a kernel wait ran out (site " + std::to_string((v >> 8) & 0xff) + ")");
  if (v) return fail(VEDA_ERR_DEVICE_CHECK, "a kernel flagged invalid data (bits " + std::to_string(v & 0xff) + ")");
  return VEDA_OK;
}

}  // extern "C"
