// Offline weight path: absmean ternarisation and 2-bit packing.
//
// "LLM을 1.58비트로 파인튜닝: BitNet을 이용한 극단적인 양자화", section 양자화
// 메커니즘: symmetric per-tensor quantisation whose scale is the reciprocal
// of the mean absolute weight; weights are scaled, rounded, clamped to
// [-1, 1].  Section 주요 결과: four ternary weights per byte.
//
// The mean is exact: every |w| is an integer multiple of 2^-149 (the fp32
// subnormal step), so the sum is accumulated as a big integer split into
// 32-bit digit positions held in 64-bit counters (each addend is < 2^32 and
// at most 2^31 elements are summed, so no counter overflows, and integer
// addition makes the result independent of the order).  The sum is rounded
// once to fp64 (nearest, ties to even), divided by N*K in fp64 and rounded to
// fp32; s_w = 1 / max(mean, 1e-5) in fp32.  q = clamp(rint(w * s_w), -1, 1).
//
// Packing: codes are 2-bit two's complement (-1 -> 0b11, 0 -> 0, +1 -> 0b01);
// in each little-endian 32-bit word of 16 consecutive weights, weight 4j + i
// sits at bits 8i + 2j.
#include "common.cuh"

namespace bitnet {

constexpr int WQ_DIGITS = 10;           // 320 bits of 2^-149 units (max sum < 2^(277+31))

// The counters live in registers: a switch on the digit index (weights of
// one tensor share one or two exponent groups, so the branch hardly diverges).
struct Digits {
  uint64_t c[WQ_DIGITS];
};

// Adds |w| (given as its fp32 bit pattern) to the digit counters.
BN_DEV void digits_add(Digits& acc, uint32_t bits) {
  bits &= 0x7FFFFFFFu;
  const uint32_t ex = bits >> 23;
  const uint32_t man = (bits & 0x7FFFFFu) | (ex ? 0x800000u : 0u);
  const uint32_t sh = ex ? ex - 1 : 0;             // value = man << sh (units of 2^-149)
  const uint64_t v = (uint64_t)man << (sh & 31);
  const uint64_t lo = (uint32_t)v, hi = v >> 32;
  switch (sh >> 5) {                               // 0 .. 7 (sh <= 254)
#define BN_DIGIT_CASE(D) case D: acc.c[D] += lo; acc.c[D + 1] += hi; break;
    BN_DIGIT_CASE(0) BN_DIGIT_CASE(1) BN_DIGIT_CASE(2) BN_DIGIT_CASE(3)
    BN_DIGIT_CASE(4) BN_DIGIT_CASE(5) BN_DIGIT_CASE(6) BN_DIGIT_CASE(7)
#undef BN_DIGIT_CASE
  }
}

template <typename TIn>
__global__ void __launch_bounds__(256)
absmean_digits_kernel(const TIn* __restrict__ W, size_t n16, uint64_t* __restrict__ ws) {
  __shared__ unsigned long long sacc[WQ_DIGITS];
  if (threadIdx.x < WQ_DIGITS) sacc[threadIdx.x] = 0ull;
  __syncthreads();
  Digits acc;
#pragma unroll
  for (int i = 0; i < WQ_DIGITS; ++i) acc.c[i] = 0;
  // four independent 16-byte loads in flight per thread (integer sums: any
  // grouping gives the same counters; padding chunks add zero)
  constexpr int U = 4;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < n16; i0 += U * stride) {
    uint4 u[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const size_t i = i0 + k * stride;
      u[k] = i < n16 ? ldg_nc_v4(reinterpret_cast<const uint8_t*>(W) + 16 * i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if constexpr (sizeof(TIn) == 4) {
        digits_add(acc, u[k].x); digits_add(acc, u[k].y); digits_add(acc, u[k].z); digits_add(acc, u[k].w);
      } else {
        digits_add(acc, u[k].x << 16); digits_add(acc, u[k].x & 0xFFFF0000u);
        digits_add(acc, u[k].y << 16); digits_add(acc, u[k].y & 0xFFFF0000u);
        digits_add(acc, u[k].z << 16); digits_add(acc, u[k].z & 0xFFFF0000u);
        digits_add(acc, u[k].w << 16); digits_add(acc, u[k].w & 0xFFFF0000u);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < WQ_DIGITS; ++i) {
    // warp-level sum first (integers: any order is exact), then one shared atomic per warp
    unsigned long long x = acc.c[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if ((threadIdx.x & 31) == 0 && x) atomicAdd(&sacc[i], x);
  }
  __syncthreads();
  if (threadIdx.x < WQ_DIGITS && sacc[threadIdx.x])
    atomicAdd(reinterpret_cast<unsigned long long*>(ws) + threadIdx.x, sacc[threadIdx.x]);
}

// Exact digit sum -> fp64 (round to nearest even) -> mean -> s_w.
__global__ void absmean_finalize_kernel(const uint64_t* __restrict__ ws, double count,
                                        float* __restrict__ s_w) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  uint32_t D[WQ_DIGITS + 2];
  uint64_t carry = 0;
  for (int i = 0; i < WQ_DIGITS; ++i) {
    const uint64_t t = ws[i] + carry;              // ws[i] < 2^63, carry < 2^32
    D[i] = (uint32_t)t;
    carry = t >> 32;
  }
  D[WQ_DIGITS] = (uint32_t)carry;
  D[WQ_DIGITS + 1] = (uint32_t)(carry >> 32);
  int top = -1;                                    // index of the highest set bit
  for (int i = WQ_DIGITS + 1; i >= 0 && top < 0; --i)
    if (D[i]) top = 32 * i + 31 - __clz(D[i]);
  auto bit = [&](int p) -> uint32_t { return p < 0 ? 0u : (D[p >> 5] >> (p & 31)) & 1u; };
  double sum;
  if (top < 0) {
    sum = 0.0;
  } else if (top <= 52) {
    const uint64_t lo = (uint64_t)D[0] | ((uint64_t)D[1] << 32);
    sum = ldexp((double)lo, -149);                 // exact
  } else {
    uint64_t mant = 0;
    for (int p = top; p > top - 53; --p) mant = (mant << 1) | bit(p);
    const uint32_t rnd = bit(top - 53);
    bool sticky = false;
    for (int p = top - 54; p >= 0 && !sticky; --p) sticky = bit(p) != 0;
    if (rnd && (sticky || (mant & 1))) mant += 1;  // mant may become 2^53: still exact
    sum = ldexp((double)mant, top - 52 - 149);
  }
  const double mean = sum / count;
  const float m32 = __double2float_rn(mean);
  s_w[0] = __fdiv_rn(1.0f, fmaxf(m32, 1e-5f));
}

template <typename TIn>
__global__ void __launch_bounds__(256)
ternary_pack_kernel(const TIn* __restrict__ W, size_t ngroups, const float* __restrict__ s_w_ptr,
                    uint32_t* __restrict__ pk) {
  const size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= ngroups) return;
  const float s_w = __ldg(s_w_ptr);
  float w[16];
  const uint8_t* src = reinterpret_cast<const uint8_t*>(W) + g * 16 * sizeof(TIn);
  if constexpr (sizeof(TIn) == 4) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 u = ldg_nc_v4(src + 16 * q);
      w[4 * q] = __uint_as_float(u.x); w[4 * q + 1] = __uint_as_float(u.y);
      w[4 * q + 2] = __uint_as_float(u.z); w[4 * q + 3] = __uint_as_float(u.w);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint4 u = ldg_nc_v4(src + 16 * q);
      w[8 * q] = bf16lo(u.x); w[8 * q + 1] = bf16hi(u.x); w[8 * q + 2] = bf16lo(u.y);
      w[8 * q + 3] = bf16hi(u.y); w[8 * q + 4] = bf16lo(u.z); w[8 * q + 5] = bf16hi(u.z);
      w[8 * q + 6] = bf16lo(u.w); w[8 * q + 7] = bf16hi(u.w);
    }
  }
  uint32_t word = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int q = __float2int_rn(__fmul_rn(w[4 * j + i], s_w));
      q = max(-1, min(1, q));
      word |= (uint32_t)(q & 3) << (8 * i + 2 * j);
    }
  }
  pk[g] = word;
}

size_t weights_workspace_bytes() { return 128; }

// Ends the weight path.  The linear kernels stream their weights before they
// wait for the kernel ahead of them in the stream (programmatic dependent
// launch), and that wait alone orders memory.  This empty kernel is launched
// without the programmatic attribute, so it starts only once the kernel that
// wrote the weights has completed; and as it never signals its dependents
// early, the next kernel can start only after it has exited.  A linear kernel
// enqueued right after a weight call therefore cannot read the weights early.
__global__ void weights_ready_kernel() {}

cudaError_t enqueue_weights_ready(cudaStream_t st) {
  weights_ready_kernel<<<1, 32, 0, st>>>();
  return cudaGetLastError();
}

cudaError_t run_quantize_weights(const void* W, int bf16, int64_t N, int64_t K, uint8_t* pkW,
                                 float* s_w, void* ws, cudaStream_t st) {
  const size_t n = (size_t)N * (size_t)K;
  cudaError_t e = cudaMemsetAsync(ws, 0, WQ_DIGITS * sizeof(uint64_t), st);
  if (e != cudaSuccess) return e;
  const size_t n16 = n * (bf16 ? 2 : 4) / 16;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  size_t blocks = (n16 + 255) / 256;
  if (blocks > (size_t)sms * 8) blocks = (size_t)sms * 8;
  if (blocks < 1) blocks = 1;
  if (bf16)
    absmean_digits_kernel<uint16_t><<<(unsigned)blocks, 256, 0, st>>>(static_cast<const uint16_t*>(W), n16, static_cast<uint64_t*>(ws));
  else
    absmean_digits_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(static_cast<const float*>(W), n16, static_cast<uint64_t*>(ws));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  absmean_finalize_kernel<<<1, 32, 0, st>>>(static_cast<const uint64_t*>(ws), (double)n, s_w);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t ng = n / 16;
  const unsigned pb = (unsigned)((ng + 255) / 256);
  if (bf16)
    ternary_pack_kernel<uint16_t><<<pb, 256, 0, st>>>(static_cast<const uint16_t*>(W), ng, s_w, reinterpret_cast<uint32_t*>(pkW));
  else
    ternary_pack_kernel<float><<<pb, 256, 0, st>>>(static_cast<const float*>(W), ng, s_w, reinterpret_cast<uint32_t*>(pkW));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return enqueue_weights_ready(st);
}

}  // namespace bitnet
