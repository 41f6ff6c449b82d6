// omnikv_decode_static: decode attention followed by the split-K combine, with
// the split-K partials kept in a fixed device array owned by this library
// instead of a buffer the caller allocates.
//
// Who needs it: callers that cannot make a new device allocation while
// decoding -- an inference engine that reserved (nearly) all device memory for
// its own pool at start-up, so a further cudaMalloc fails or fragments the pool;
// a plug-in whose host framework owns every allocation and forbids its
// extensions from allocating; a latency-critical loop that cannot afford
// cudaMalloc / cudaFree, which may synchronise the device.
//
// The scratch is a file-scope __device__ array of kScratchBytes (8 MiB) that
// every GPU loading this library holds until the process exits. Host code only
// sees a stand-in for it, so its device address is looked up with
// cudaGetSymbolAddress once per device and context (on the first call made with
// that device current, and again after the device's context is recreated) and
// passed to the kernels. All calls share the one array and it keeps the last
// call's contents: nothing in it needs to start at zero (every split the combine
// reads is written first by the same call), but calls that overlap on the GPU --
// on different streams, or from different host threads -- race on it.
#include <cuda_runtime.h>

#include <atomic>

#include "abi_internal.h"
#include "common.cuh"
#include "kernels.h"

using namespace omnikv;

namespace {

constexpr size_t kScratchBytes = OMNIKV_DECODE_STATIC_SCRATCH_BYTES;  // 5405 partials entries of 1552 B
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_decode_scratch[kScratchBytes];

// The array's device address per device, with the context it was looked up in:
// a device reset (or any new context of the device) loads the module again,
// possibly at another address, so the address is looked up again when the
// current context differs from the one cached.
struct ScratchAddr {
  std::atomic<void*> ctx{nullptr};
  std::atomic<void*> addr{nullptr};
};
ScratchAddr g_scratch[kMaxDevices];

using CtxGetCurrentFn = int (*)(void** ctx);  // the driver's cuCtxGetCurrent (CUresult, CUcontext*)

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(f);
  }();
  return fn;
}

// Device address of g_decode_scratch in the current context of the current device.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const CtxGetCurrentFn get = ctx_get_current();
  if (get == nullptr) return cudaErrorInitializationError;
  void* ctx = nullptr;  // null until the runtime has made its context current on this thread
  if (get(&ctx) != 0) return cudaErrorInitializationError;
  ScratchAddr& c = g_scratch[dev];
  void* p = c.addr.load(std::memory_order_acquire);
  if (p == nullptr || ctx == nullptr || c.ctx.load(std::memory_order_acquire) != ctx) {
    e = cudaGetSymbolAddress(&p, g_decode_scratch);  // makes the runtime's context current
    if (e != cudaSuccess) return e;
    if (get(&ctx) != 0 || ctx == nullptr) return cudaErrorInitializationError;
    c.addr.store(p, std::memory_order_release);
    c.ctx.store(ctx, std::memory_order_release);
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" {

omnikv_status omnikv_decode_static(const omnikv_config* cfg, const omnikv_cache* cache, const void* q, float* out,
                                   int32_t num_splits, void* stream) {
  omnikv_status st = validate_config_cache(cfg, cache);
  if (st != OMNIKV_OK) return st;
  if (!q || !out || num_splits < 0) return OMNIKV_ERR_INVALID_ARG;
  const long long per_split = (long long)cache->batch * cfg->num_q_heads * (long long)sizeof(Partial);
  const long long fit = (long long)kScratchBytes / per_split;  // splits that fit in the scratch
  if (fit < 1) return OMNIKV_ERR_CAPACITY;
  int32_t S = num_splits;
  if (S == 0) {
    S = resolve_splits(cfg, cache, 0);
    if (S > fit) S = (int32_t)fit;
  } else if (S > fit) {
    return OMNIKV_ERR_CAPACITY;
  }
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return OMNIKV_ERR_CUDA;
  DecodeParams dp;
  if ((st = prepare_decode(cfg, cache, q, scratch, S, &dp)) != OMNIKV_OK) return st;
  CombineParams cp;
  if ((st = prepare_combine(cfg, cache, scratch, S, out, &cp)) != OMNIKV_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (launch_decode(dp, cache->batch, s) != cudaSuccess) return OMNIKV_ERR_CUDA;
  if (launch_combine(cp, cache->batch, s) != cudaSuccess) return OMNIKV_ERR_CUDA;
  return OMNIKV_OK;
}

}  // extern "C"
