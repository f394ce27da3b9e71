// bitnet_quantize_weights_noalloc: the offline weight path for callers that
// cannot allocate device memory.
//
// bitnet_quantize_weights needs a small scratch buffer (the digit counters of
// the exact mean |W|), which its caller allocates.  Some callers cannot do
// that: a plugin running inside a host application that owns every device
// allocation, a runtime that reserves all its memory up front and forbids
// allocation afterwards, or code that must not pay the implicit device
// synchronisation a cudaMalloc/cudaFree can cause.  This variant keeps the
// scratch in a fixed array in this library's device memory instead.
//
// The array lives for as long as the library is loaded, on every device that
// uses it.  Host code cannot use the array's name as a device address, so the
// first call on each device looks the address up with cudaGetSymbolAddress
// (with that device current) and caches it.  The cached address belongs to
// the device's primary context: after cudaDeviceReset, or under a context the
// caller created itself, it no longer names the array, and this entry point
// must not be called.  All calls share the one array: the counters are cleared
// at the start of each call, and two calls whose kernels overlap on the GPU
// (for example on two streams) race on it.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/bitnet.h"

namespace bitnet {
cudaError_t run_quantize_weights(const void* W, int bf16, int64_t N, int64_t K, uint8_t* pkW,
                                 float* s_w, void* ws, cudaStream_t st);
size_t weights_workspace_bytes();
}  // namespace bitnet

namespace {

// Fixed scratch: 256 bytes, room for the ten 64-bit counters the reduction uses.
constexpr size_t kNoallocScratchBytes = 256;
static __device__ __align__(256) unsigned long long g_noalloc_scratch[kNoallocScratchBytes / 8];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return BITNET_ERR_CUDA; }
  if (dev < 0 || dev >= kMaxDevices) return BITNET_ERR_UNSUPPORTED;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return BITNET_ERR_CUDA;
  }
  if (major != 10) return BITNET_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return BITNET_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return BITNET_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int bitnet_quantize_weights_noalloc(const void* W, int w_dtype, int64_t N, int64_t K,
                                               uint8_t* pkW, float* s_w, void* stream) {
  if (!W || !pkW || !s_w) return BITNET_ERR_NULL;
  if (w_dtype != BITNET_F32 && w_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (N < 1 || K < 16 || K % 16 != 0) return BITNET_ERR_SHAPE;
  // the fixed 64-bit counters absorb at most 2^31 - 1 weights without overflow
  // (compared by division first, so that N * K is never formed when it could overflow)
  if (K > BITNET_NOALLOC_MAX_WEIGHTS / N || N * K > BITNET_NOALLOC_MAX_WEIGHTS) return BITNET_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(pkW) || (reinterpret_cast<uintptr_t>(s_w) & 3u)) return BITNET_ERR_ALIGN;
  if (bitnet::weights_workspace_bytes() > kNoallocScratchBytes) return BITNET_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != BITNET_OK) return st;
  const cudaError_t e = bitnet::run_quantize_weights(W, w_dtype == BITNET_BF16, N, K, pkW, s_w, scratch,
                                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) { cudaGetLastError(); return BITNET_ERR_CUDA; }
  return BITNET_OK;
}
