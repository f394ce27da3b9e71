// Measurement: dense int8 tensor-core throughput of this GPU, in the very
// instruction form the BitLinear GEMM issues (tcgen05.mma.cta_group::1.kind::i8,
// A from tensor memory, B from a shared-memory descriptor, int32 accumulators
// in tensor memory).  It is the denominator of the GEMM's roofline fraction,
// measured instead of derived from a bf16 figure.
//
// One CTA per SM holds all 512 tensor-memory columns: a 128 x BN int32
// accumulator and four A slices; one thread issues n_mma MMAs of
// 128 x BN x 32 back to back into the one accumulator, cycling over four
// A/B slices, then commits and waits (bounded) for them.  Operand values do
// not matter for the timing; B is filled with a fixed byte pattern.
#include "../../include/bitnet_measure.h"
#include "common.cuh"

namespace bitnet {

constexpr int PK_THREADS = 128;
constexpr size_t PK_SMEM = 256 * 128 + 1024 + 100 * 1024;   // B tile (256 rows x 128 B) + slack: one CTA per SM

template <int BN>
__global__ void __launch_bounds__(PK_THREADS, 1)
peak_i8_kernel(int n_mma, unsigned long long* __restrict__ cycles, unsigned long long* __restrict__ nanos) {
  extern __shared__ uint8_t pk_raw[];
  __shared__ __align__(8) uint64_t bar_done;
  __shared__ uint32_t tmem_base_sh;
  uint8_t* b = smem_align(pk_raw, 1024u);
  for (int i = threadIdx.x; i < BN * 128 / 4; i += PK_THREADS)
    reinterpret_cast<uint32_t*>(b)[i] = 0x9E3779B9u * (uint32_t)(i + 1);
  fence_proxy_async_smem();
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&bar_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  if (threadIdx.x == 32) {
    constexpr uint32_t IDESC = idesc_i8(128, BN);
    const uint32_t baddr = smem_u32(b);
    const long long c0 = clock64();
    const uint64_t g0 = globaltimer();
    for (int i = 0; i < n_mma; ++i) {
      const int kk = i & 3;
      mma_i8_ts(tmem, tmem + 256u + 8u * (uint32_t)kk, smem_desc_k_sw128(baddr + 32 * kk), IDESC,
                i > 0 ? 1u : 0u);
    }
    mma_commit(&bar_done);
    mbar_wait(&bar_done, 0, DEV_ERR_TIMEOUT_ACC, false);
    const long long c1 = clock64();
    const uint64_t g1 = globaltimer();
    cycles[blockIdx.x] = (unsigned long long)(c1 - c0);
    nanos[blockIdx.x] = g1 - g0;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Self-test of the bounded waits: one thread waits on an mbarrier that nothing
// will ever complete, through the same mbar_wait every pipeline uses.  After
// its time limit (about two seconds) the wait gives up, records the code in
// g_device_error and returns; the kernel then exits normally.
__global__ void wait_timeout_selftest_kernel() {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  mbar_wait(&bar, 0, DEV_ERR_TIMEOUT_FULL, false);
}

}  // namespace bitnet

extern "C" int bitnet_selftest_wait_timeout(void* stream) {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return BITNET_ERR_CUDA;
  }
  if (major != 10) return BITNET_ERR_UNSUPPORTED;
  bitnet::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  if (cudaGetLastError() != cudaSuccess) return BITNET_ERR_CUDA;
  return BITNET_OK;
}

extern "C" int bitnet_measure_i8_mma(int n_mma, int bn, int ctas, unsigned long long* cycles,
                                     unsigned long long* nanos, void* stream) {
  if (n_mma < 1 || n_mma > (1 << 24) || (bn != 128 && bn != 256) || ctas < 1 || ctas > 4096)
    return BITNET_ERR_SHAPE;
  if (!cycles || !nanos) return BITNET_ERR_NULL;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return BITNET_ERR_CUDA;
  }
  if (major != 10) return BITNET_ERR_UNSUPPORTED;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (bn == 128) {
    e = bitnet::ensure_smem_limit(reinterpret_cast<const void*>(bitnet::peak_i8_kernel<128>), bitnet::PK_SMEM);
    if (e == cudaSuccess) {
      bitnet::peak_i8_kernel<128><<<ctas, bitnet::PK_THREADS, bitnet::PK_SMEM, st>>>(n_mma, cycles, nanos);
      e = cudaGetLastError();
    }
  } else {
    e = bitnet::ensure_smem_limit(reinterpret_cast<const void*>(bitnet::peak_i8_kernel<256>), bitnet::PK_SMEM);
    if (e == cudaSuccess) {
      bitnet::peak_i8_kernel<256><<<ctas, bitnet::PK_THREADS, bitnet::PK_SMEM, st>>>(n_mma, cycles, nanos);
      e = cudaGetLastError();
    }
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return BITNET_ERR_CUDA;
  }
  return BITNET_OK;
}
