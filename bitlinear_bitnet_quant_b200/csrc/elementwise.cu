// Element-wise glue of the stacked BitLinear chain: the fp32 residual add and
// the squared-ReLU gated unit of the feed-forward block ("AI 혁신의 선두:
// 마이크로소프트의 1비트 LLM, BitNet b1.58 2B4T", section 주요 아키텍처 혁신:
// squared ReLU).  Fixed fp32 arithmetic, no contraction:
//   add:  out = a + b
//   glu:  g = max(gate, 0);  out = (g * g) * up
#include "common.cuh"

namespace bitnet {

__global__ void __launch_bounds__(256)
add_f32_kernel(const float4* __restrict__ a, const float4* __restrict__ b, float4* __restrict__ out, size_t n4) {
  pdl_launch_dependents();
  pdl_wait();                                   // inputs come from the previous kernels
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const uint4 ua = ldg_v4(a + i), ub = ldg_v4(b + i);
    const float4 x = make_float4(__uint_as_float(ua.x), __uint_as_float(ua.y), __uint_as_float(ua.z), __uint_as_float(ua.w));
    const float4 y = make_float4(__uint_as_float(ub.x), __uint_as_float(ub.y), __uint_as_float(ub.z), __uint_as_float(ub.w));
    out[i] = make_float4(__fadd_rn(x.x, y.x), __fadd_rn(x.y, y.y), __fadd_rn(x.z, y.z), __fadd_rn(x.w, y.w));
  }
}

__global__ void __launch_bounds__(256)
relu2_glu_kernel(const float4* __restrict__ gate, const float4* __restrict__ up, float4* __restrict__ out,
                 size_t n4) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const uint4 ug = ldg_v4(gate + i), uu = ldg_v4(up + i);
    const float4 g = make_float4(__uint_as_float(ug.x), __uint_as_float(ug.y), __uint_as_float(ug.z), __uint_as_float(ug.w));
    const float4 u = make_float4(__uint_as_float(uu.x), __uint_as_float(uu.y), __uint_as_float(uu.z), __uint_as_float(uu.w));
    out[i] = make_float4(relu2_times(g.x, u.x), relu2_times(g.y, u.y), relu2_times(g.z, u.z), relu2_times(g.w, u.w));
  }
}

static unsigned ew_grid(size_t n4) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  size_t blocks = (n4 + 255) / 256;
  const size_t cap = (size_t)sms * 8;
  return (unsigned)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

cudaError_t run_add_f32(const float* a, const float* b, float* out, size_t n, cudaStream_t st) {
  const size_t n4 = n / 4;
  return launch_pdl(add_f32_kernel, dim3(ew_grid(n4)), dim3(256), 0, st, 1u, reinterpret_cast<const float4*>(a),
                    reinterpret_cast<const float4*>(b), reinterpret_cast<float4*>(out), n4);
}

cudaError_t run_relu2_glu(const float* gate, const float* up, float* out, size_t n, cudaStream_t st) {
  const size_t n4 = n / 4;
  return launch_pdl(relu2_glu_kernel, dim3(ew_grid(n4)), dim3(256), 0, st, 1u,
                    reinterpret_cast<const float4*>(gate), reinterpret_cast<const float4*>(up),
                    reinterpret_cast<float4*>(out), n4);
}

}  // namespace bitnet
