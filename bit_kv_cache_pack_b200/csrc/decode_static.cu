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
// sees a stand-in for it, so its device address is looked up once per device
// with cudaGetSymbolAddress (on the first call made with that device current)
// and passed to the kernels. All calls share the one array and it keeps the last
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

std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of g_decode_scratch on the current device (set up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev].store(p, std::memory_order_release);
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
