// Ternary weights five per byte ("양자화(quantization) 1.58bit", section
// "1.58비트는 어디서 나온거에요?": three states carry log2(3) = 1.58 bits, so
// five weights fit in 3^5 = 243 <= 256 byte values, 1.6 bits per weight).
//
// Byte g of a row = sum_i (w[5g + i] + 1) * 3^i, i = 0..4; weights past K
// count as 0 and each row is padded to a multiple of 16 bytes with bytes of
// five zero weights (121).  The repacking reads the 2-bit packed weights of
// bitnet_quantize_weights (weight 4j + i of a 16-weight word at bits
// 8i + 2j, two's complement) and writes this format; the decode kernel reads
// it back (linear_decode.cu).
#include "decode_common.cuh"

namespace bitnet {

cudaError_t enqueue_weights_ready(cudaStream_t st);

// One thread per output byte: five 2-bit codes in, one base-3 byte out.
__global__ void __launch_bounds__(256)
trit5_pack_kernel(const uint32_t* __restrict__ pkW, int N, int K, int r5, uint8_t* __restrict__ pk5) {
  pdl_launch_dependents();
  pdl_wait();                                  // the packed weights may come from the previous kernel
  const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (size_t)N * r5) return;
  const int n = (int)(idx / r5), g = (int)(idx - (size_t)n * r5);
  const uint32_t* row = pkW + (size_t)n * (K / 16);
  int b = 0, p = 1;
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    const int k = 5 * g + i;
    int digit = 1;                             // a zero weight past K and in the padding
    if (k < K) {
      const int kk = k & 15;
      const uint32_t code = (__ldg(row + (k >> 4)) >> (8 * (kk & 3) + 2 * (kk >> 2))) & 3u;
      digit = code == 3u ? 0 : (int)code + 1;  // -1, 0, +1 -> 0, 1, 2
    }
    b += digit * p;
    p *= 3;
  }
  pk5[idx] = (uint8_t)b;
}

cudaError_t run_repack_trit5(const uint8_t* pkW, int N, int K, uint8_t* pk5, cudaStream_t st) {
  const int r5 = trit5_row_bytes(K);
  const size_t total = (size_t)N * r5;
  const unsigned blocks = (unsigned)((total + 255) / 256);
  const cudaError_t e = launch_pdl(trit5_pack_kernel, dim3(blocks), dim3(256), 0, st, 1u,
                                   reinterpret_cast<const uint32_t*>(pkW), N, K, r5, pk5);
  if (e != cudaSuccess) return e;
  return enqueue_weights_ready(st);             // the decode kernel reads pk5 before its dependency wait
}

size_t trit5_row_bytes_host(int K) { return (size_t)trit5_row_bytes(K); }

}  // namespace bitnet
