// extern "C" entry points declared in include/bitnet.h: host-side validation,
// then dispatch to the kernels.  Nothing here allocates device memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/bitnet.h"
#include "common.cuh"

namespace bitnet {
__device__ int g_device_error = 0;

cudaError_t run_quantize_weights(const void* W, int bf16, int64_t N, int64_t K, uint8_t* pkW,
                                 float* s_w, void* ws, cudaStream_t st);
size_t weights_workspace_bytes();
cudaError_t run_quant_act_i8(const void* X, int bf16, int M, int K, const float* gamma, float eps,
                             int8_t* Xq, float* s_x, cudaStream_t st);
cudaError_t run_hadamard_quant_i4(const void* X, int bf16, int M, int K, int L, const float* gamma,
                                  float eps, uint8_t* Xq4, float* s_x, float* T_dbg, cudaStream_t st);
cudaError_t run_linear(const void* Xq, int act_bits, const float* s_x, const uint8_t* pkW, const float* s_w,
                       int M, int N, int K, void* Y, int y_bf16, int32_t* acc_dbg, int path, cudaStream_t st);
cudaError_t run_linear_group(const LinGroup& grp, const void* Xq, int act_bits, const float* s_x, int M, int K,
                             int y_bf16, int path, cudaStream_t st);
bool tensor_map_encoder_available();
cudaError_t run_add_quant_act_i8(const float* A, const float* B, int M, int K, const float* gamma, float eps,
                                 float* H, int8_t* Xq, float* s_x, cudaStream_t st);
cudaError_t run_glu_hadamard_quant_i4(const float* gate, const float* up, int M, int K, int L, const float* gamma,
                                      float eps, uint8_t* Xq4, float* s_x, cudaStream_t st);
cudaError_t run_bitlinear(const void* X, int x_bf16, int M, int K, const float* gamma, float eps, const uint8_t* pkW,
                          const float* s_w, int N, void* Y, int y_bf16, int8_t* Xq, float* s_x, int path,
                          cudaStream_t st);
bool decode_path_applies(int M, int K);
bool fused_path_applies(int M, int N, int K, int x_bf16);
cudaError_t run_add_f32(const float* a, const float* b, float* out, size_t n, cudaStream_t st);
cudaError_t run_repack_trit5(const uint8_t* pkW, int N, int K, uint8_t* pk5, cudaStream_t st);
size_t trit5_row_bytes_host(int K);
cudaError_t run_linear_decode_trit5(const void* Xq, int act_bits, const float* s_x, const uint8_t* pk5,
                                    const float* s_w, int M, int N, int K, void* Y, int y_bf16, int32_t* acc_dbg,
                                    cudaStream_t st);
cudaError_t run_relu2_glu(const float* gate, const float* up, float* out, size_t n, cudaStream_t st);
cudaError_t run_rope_append(float* Q, const float* K, const float* V, int B, int L, int t0, int heads, int d,
                            double base, float* Kc, float* Vc, int T_cap, cudaStream_t st);
cudaError_t run_attention(const float* Q, const float* Kc, const float* Vc, int B, int L, int t0, int heads, int d,
                          int T_cap, float* A, cudaStream_t st);
}  // namespace bitnet

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_dev_ok[kMaxDevices];   // 0 unknown, 1 sm_100, 2 other

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return BITNET_ERR_CUDA; }
  if (dev < 0 || dev >= kMaxDevices) return BITNET_ERR_UNSUPPORTED;
  int s = g_dev_ok[dev].load(std::memory_order_relaxed);
  if (s == 0) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
      cudaGetLastError();
      return BITNET_ERR_CUDA;
    }
    s = major == 10 ? 1 : 2;
    g_dev_ok[dev].store(s, std::memory_order_relaxed);
  }
  return s == 1 ? BITNET_OK : BITNET_ERR_UNSUPPORTED;
}

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return BITNET_OK;
  cudaGetLastError();
  return BITNET_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* bitnet_status_string(int status) {
  switch (status) {
    case BITNET_OK: return "ok";
    case BITNET_ERR_NULL: return "a required pointer is NULL";
    case BITNET_ERR_SHAPE: return "a size breaks the documented limits";
    case BITNET_ERR_ALIGN: return "a tensor pointer is not 16-byte aligned";
    case BITNET_ERR_DTYPE: return "unknown dtype or act_bits value";
    case BITNET_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case BITNET_ERR_UNSUPPORTED: return "no sm_100 device or TMA encoder unavailable";
    case BITNET_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

int bitnet_abi_version(void) { return 2; }

size_t bitnet_quantize_weights_workspace_size(int64_t N, int64_t K) {
  (void)N; (void)K;
  return bitnet::weights_workspace_bytes();
}

int bitnet_quantize_weights(const void* W, int w_dtype, int64_t N, int64_t K, uint8_t* pkW, float* s_w,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (!W || !pkW || !s_w) return BITNET_ERR_NULL;
  if (w_dtype != BITNET_F32 && w_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (N < 1 || K < 16 || K % 16 != 0 || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) ||
      N * K >= (int64_t(1) << 31))                       // each factor < 2^31: the product cannot overflow
    return BITNET_ERR_SHAPE;
  if (!workspace || workspace_bytes < bitnet::weights_workspace_bytes()) return BITNET_ERR_WORKSPACE;
  if (!aligned16(W) || !aligned16(pkW) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(s_w) & 3u))
    return BITNET_ERR_ALIGN;
  int d = check_device();
  if (d != BITNET_OK) return d;
  return cuda_status(bitnet::run_quantize_weights(W, w_dtype == BITNET_BF16, N, K, pkW, s_w, workspace,
                                                  static_cast<cudaStream_t>(stream)));
}

int bitnet_quant_act(const void* X, int x_dtype, int64_t M, int64_t K, const float* gamma, float eps,
                     int8_t* Xq, float* s_x, void* stream) {
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (M < 0 || M > (int64_t(1) << 30) || K < 16 || K > 16384 || K % 16 != 0) return BITNET_ERR_SHAPE;
  if (M == 0) return BITNET_OK;
  if (!X || !Xq || !s_x) return BITNET_ERR_NULL;
  if (!aligned16(X) || !aligned16(Xq) || (gamma && !aligned16(gamma)) || (reinterpret_cast<uintptr_t>(s_x) & 3u))
    return BITNET_ERR_ALIGN;
  int d = check_device();
  if (d != BITNET_OK) return d;
  return cuda_status(bitnet::run_quant_act_i8(X, x_dtype == BITNET_BF16, (int)M, (int)K, gamma, eps, Xq, s_x,
                                              static_cast<cudaStream_t>(stream)));
}

int bitnet_add_quant_act(const float* A, const float* B, int64_t M, int64_t K, const float* gamma, float eps,
                         float* H, int8_t* Xq, float* s_x, void* stream) {
  if (M < 0 || M > (int64_t(1) << 30) || K < 16 || K > 16384 || K % 16 != 0) return BITNET_ERR_SHAPE;
  if (M == 0) return BITNET_OK;
  if (!A || !B || !H || !Xq || !s_x) return BITNET_ERR_NULL;
  if (!aligned16(A) || !aligned16(B) || !aligned16(H) || !aligned16(Xq) || (gamma && !aligned16(gamma)) ||
      (reinterpret_cast<uintptr_t>(s_x) & 3u))
    return BITNET_ERR_ALIGN;
  int d = check_device();
  if (d != BITNET_OK) return d;
  return cuda_status(bitnet::run_add_quant_act_i8(A, B, (int)M, (int)K, gamma, eps, H, Xq, s_x,
                                                  static_cast<cudaStream_t>(stream)));
}

int bitnet_glu_hadamard_quant_act(const float* gate, const float* up, int64_t M, int64_t K, const float* gamma,
                                  float eps, int had_block, uint8_t* Xq4, float* s_x, void* stream) {
  if (M < 0 || M > (int64_t(1) << 30) || K < 128 || K > 16384 || K % 128 != 0) return BITNET_ERR_SHAPE;
  int64_t b = had_block;
  if (b == 0) b = K & (-K);                    // the largest power of two dividing K
  if (b < 32 || b > 8192 || (b & (b - 1)) != 0 || K % b != 0) return BITNET_ERR_SHAPE;
  if (M == 0) return BITNET_OK;
  if (!gate || !up || !Xq4 || !s_x) return BITNET_ERR_NULL;
  if (!aligned16(gate) || !aligned16(up) || !aligned16(Xq4) || (gamma && !aligned16(gamma)) ||
      (reinterpret_cast<uintptr_t>(s_x) & 3u))
    return BITNET_ERR_ALIGN;
  int d = check_device();
  if (d != BITNET_OK) return d;
  int L = 0;
  while ((int64_t(1) << L) < b) ++L;
  return cuda_status(bitnet::run_glu_hadamard_quant_i4(gate, up, (int)M, (int)K, L, gamma, eps, Xq4, s_x,
                                                       static_cast<cudaStream_t>(stream)));
}

int bitnet_hadamard_quant_act(const void* X, int x_dtype, int64_t M, int64_t K, const float* gamma, float eps,
                              int had_block, uint8_t* Xq4, float* s_x, float* T_dbg, void* stream) {
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (M < 0 || M > (int64_t(1) << 30) || K < 128 || K > 16384 || K % 128 != 0) return BITNET_ERR_SHAPE;
  int64_t b = had_block;
  if (b == 0) b = K & (-K);
  if (b < 32 || b > 8192 || (b & (b - 1)) != 0 || K % b != 0) return BITNET_ERR_SHAPE;
  if (M == 0) return BITNET_OK;
  if (!X || !Xq4 || !s_x) return BITNET_ERR_NULL;
  if (!aligned16(X) || !aligned16(Xq4) || (gamma && !aligned16(gamma)) || (T_dbg && !aligned16(T_dbg)) ||
      (reinterpret_cast<uintptr_t>(s_x) & 3u))
    return BITNET_ERR_ALIGN;
  int d = check_device();
  if (d != BITNET_OK) return d;
  int L = 0;
  while ((int64_t(1) << L) < b) ++L;
  return cuda_status(bitnet::run_hadamard_quant_i4(X, x_dtype == BITNET_BF16, (int)M, (int)K, L, gamma, eps,
                                                   Xq4, s_x, T_dbg, static_cast<cudaStream_t>(stream)));
}

// kernel: 0 = automatic, 1 = CUDA-core dp4a, 2 = tcgen05, 3 = warp-MMA decode,
// 4 = tcgen05 with 256 weight rows per CTA, 5 = persistent tcgen05 (int8)
static int linear_impl(const void* Xq, int act_bits, const float* s_x, const uint8_t* pkW, const float* s_w,
                       int64_t M, int64_t N, int64_t K, void* Y, int y_dtype, int32_t* acc_dbg, int kernel,
                       void* stream) {
  if (kernel < 0 || kernel > 5) return BITNET_ERR_SHAPE;
  if (act_bits != 8 && act_bits != 4) return BITNET_ERR_DTYPE;
  if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (M < 0 || M > (int64_t(1) << 30) || N < 1 || N > (int64_t(1) << 30) || K < 128 || K > 65536 ||
      K % 128 != 0 || M * N >= (int64_t(1) << 40))
    return BITNET_ERR_SHAPE;
  if (M == 0) return BITNET_OK;
  if (!Xq || !s_x || !pkW || !s_w || !Y) return BITNET_ERR_NULL;
  if (!aligned16(Xq) || !aligned16(pkW) || !aligned16(Y) || (acc_dbg && !aligned16(acc_dbg)) ||
      (reinterpret_cast<uintptr_t>(s_x) & 3u) || (reinterpret_cast<uintptr_t>(s_w) & 3u))
    return BITNET_ERR_ALIGN;
  if (kernel == 3 && !bitnet::decode_path_applies((int)M, (int)K)) return BITNET_ERR_SHAPE;
  if (kernel == 5 && (act_bits != 8 || M <= 64 || (K / 128) % 2 != 0)) return BITNET_ERR_SHAPE;
  int d = check_device();
  if (d != BITNET_OK) return d;
  if (!bitnet::tensor_map_encoder_available()) return BITNET_ERR_UNSUPPORTED;
  return cuda_status(bitnet::run_linear(Xq, act_bits, s_x, pkW, s_w, (int)M, (int)N, (int)K, Y,
                                        y_dtype == BITNET_BF16, acc_dbg, kernel,
                                        static_cast<cudaStream_t>(stream)));
}

int bitnet_linear(const void* Xq, int act_bits, const float* s_x, const uint8_t* pkW, const float* s_w,
                  int64_t M, int64_t N, int64_t K, void* Y, int y_dtype, int32_t* acc_dbg, void* stream) {
  return linear_impl(Xq, act_bits, s_x, pkW, s_w, M, N, K, Y, y_dtype, acc_dbg, 0, stream);
}

int bitnet_linear_kernel(const void* Xq, int act_bits, const float* s_x, const uint8_t* pkW, const float* s_w,
                         int64_t M, int64_t N, int64_t K, void* Y, int y_dtype, int32_t* acc_dbg, int kernel,
                         void* stream) {
  return linear_impl(Xq, act_bits, s_x, pkW, s_w, M, N, K, Y, y_dtype, acc_dbg, kernel, stream);
}

int bitnet_linear_group(const void* Xq, int act_bits, const float* s_x, int64_t M, int64_t K, int count,
                        const uint8_t* const* pkW, const float* const* s_w, const int64_t* N, void* const* Y,
                        int y_dtype, void* stream) {
  if (act_bits != 8 && act_bits != 4) return BITNET_ERR_DTYPE;
  if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (count < 1 || count > bitnet::GROUP_MAX) return BITNET_ERR_SHAPE;
  if (!pkW || !s_w || !N || !Y) return BITNET_ERR_NULL;
  if (M < 0 || M > (int64_t(1) << 30) || K < 128 || K > 65536 || K % 128 != 0) return BITNET_ERR_SHAPE;
  for (int g = 0; g < count; ++g)
    if (N[g] < 1 || N[g] > (int64_t(1) << 30) || M * N[g] >= (int64_t(1) << 40)) return BITNET_ERR_SHAPE;
  if (M == 0) return BITNET_OK;
  if (!Xq || !s_x) return BITNET_ERR_NULL;
  for (int g = 0; g < count; ++g) {
    if (!pkW[g] || !s_w[g] || !Y[g]) return BITNET_ERR_NULL;
    if (!aligned16(pkW[g]) || !aligned16(Y[g]) || (reinterpret_cast<uintptr_t>(s_w[g]) & 3u)) return BITNET_ERR_ALIGN;
  }
  if (!aligned16(Xq) || (reinterpret_cast<uintptr_t>(s_x) & 3u)) return BITNET_ERR_ALIGN;
  int d = check_device();
  if (d != BITNET_OK) return d;
  if (!bitnet::tensor_map_encoder_available()) return BITNET_ERR_UNSUPPORTED;
  bitnet::LinGroup grp = {};
  for (int g = 0; g < count; ++g) {
    grp.pkW[g] = pkW[g];
    grp.s_w[g] = s_w[g];
    grp.Y[g] = Y[g];
    grp.acc_dbg[g] = nullptr;
    grp.N[g] = (int)N[g];
  }
  grp.count = count;
  return cuda_status(bitnet::run_linear_group(grp, Xq, act_bits, s_x, (int)M, (int)K, y_dtype == BITNET_BF16, 0,
                                              static_cast<cudaStream_t>(stream)));
}

size_t bitnet_trit5_row_bytes(int64_t K) {
  if (K < 1 || K > (int64_t(1) << 30)) return 0;
  return bitnet::trit5_row_bytes_host((int)K);
}

int bitnet_repack_trit5(const uint8_t* pkW, int64_t N, int64_t K, uint8_t* pk5, void* stream) {
  if (N < 1 || N >= (int64_t(1) << 31) || K < 16 || K % 16 != 0 || K > (int64_t(1) << 30)) return BITNET_ERR_SHAPE;
  if (N * (int64_t)bitnet::trit5_row_bytes_host((int)K) >= (int64_t(1) << 31) || N * K / 4 >= (int64_t(1) << 31))
    return BITNET_ERR_SHAPE;
  if (!pkW || !pk5) return BITNET_ERR_NULL;
  if (!aligned16(pkW) || !aligned16(pk5)) return BITNET_ERR_ALIGN;
  int d = check_device();
  if (d != BITNET_OK) return d;
  return cuda_status(bitnet::run_repack_trit5(pkW, (int)N, (int)K, pk5, static_cast<cudaStream_t>(stream)));
}

int bitnet_linear_trit5(const void* Xq, int act_bits, const float* s_x, const uint8_t* pk5, const float* s_w,
                        int64_t M, int64_t N, int64_t K, void* Y, int y_dtype, int32_t* acc_dbg, void* stream) {
  if (act_bits != 8 && act_bits != 4) return BITNET_ERR_DTYPE;
  if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (M < 1 || M > 32 || N < 1 || N > (int64_t(1) << 30) || K < 512 || K > 16384 ||
      !bitnet::decode_path_applies((int)M, (int)K))
    return BITNET_ERR_SHAPE;
  if (!Xq || !s_x || !pk5 || !s_w || !Y) return BITNET_ERR_NULL;
  if (!aligned16(Xq) || !aligned16(pk5) || !aligned16(Y) || (acc_dbg && !aligned16(acc_dbg)) ||
      (reinterpret_cast<uintptr_t>(s_x) & 3u) || (reinterpret_cast<uintptr_t>(s_w) & 3u))
    return BITNET_ERR_ALIGN;
  int d = check_device();
  if (d != BITNET_OK) return d;
  return cuda_status(bitnet::run_linear_decode_trit5(Xq, act_bits, s_x, pk5, s_w, (int)M, (int)N, (int)K, Y,
                                                     y_dtype == BITNET_BF16, acc_dbg,
                                                     static_cast<cudaStream_t>(stream)));
}

static int elementwise_check(const float* a, const float* b, const float* out, int64_t n) {
  if (n < 0 || n % 4 != 0) return BITNET_ERR_SHAPE;
  if (n == 0) return -1;                                  // nothing to do
  if (!a || !b || !out) return BITNET_ERR_NULL;
  if (!aligned16(a) || !aligned16(b) || !aligned16(out)) return BITNET_ERR_ALIGN;
  return check_device();
}

// kernel: 0 = automatic (the quantiser, then bitnet_linear's choice), 1-3 = the
// quantiser, then that linear kernel family, 4 = the fused single kernel
static int bitlinear_impl(const void* X, int x_dtype, int64_t M, int64_t K, const float* gamma, float eps,
                          const uint8_t* pkW, const float* s_w, int64_t N, void* Y, int y_dtype, int8_t* Xq,
                          float* s_x, int kernel, void* stream) {
  if (kernel < 0 || kernel > 4) return BITNET_ERR_SHAPE;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (M < 0 || M > (int64_t(1) << 30) || N < 1 || N > (int64_t(1) << 30) || K < 128 || K > 16384 ||
      K % 128 != 0 || M * N >= (int64_t(1) << 40))
    return BITNET_ERR_SHAPE;
  if (M == 0) return BITNET_OK;
  if (!X || !pkW || !s_w || !Y || !Xq || !s_x) return BITNET_ERR_NULL;
  if (!aligned16(X) || !aligned16(pkW) || !aligned16(Y) || !aligned16(Xq) || (gamma && !aligned16(gamma)) ||
      (reinterpret_cast<uintptr_t>(s_x) & 3u) || (reinterpret_cast<uintptr_t>(s_w) & 3u))
    return BITNET_ERR_ALIGN;
  if (kernel == 3 && !bitnet::decode_path_applies((int)M, (int)K)) return BITNET_ERR_SHAPE;
  int d = check_device();
  if (d != BITNET_OK) return d;
  if (!bitnet::tensor_map_encoder_available()) return BITNET_ERR_UNSUPPORTED;
  if (kernel == 4 && !bitnet::fused_path_applies((int)M, (int)N, (int)K, x_dtype == BITNET_BF16))
    return BITNET_ERR_SHAPE;
  return cuda_status(bitnet::run_bitlinear(X, x_dtype == BITNET_BF16, (int)M, (int)K, gamma, eps, pkW, s_w, (int)N,
                                           Y, y_dtype == BITNET_BF16, Xq, s_x, kernel,
                                           static_cast<cudaStream_t>(stream)));
}

int bitnet_bitlinear(const void* X, int x_dtype, int64_t M, int64_t K, const float* gamma, float eps,
                     const uint8_t* pkW, const float* s_w, int64_t N, void* Y, int y_dtype, int8_t* Xq, float* s_x,
                     void* stream) {
  return bitlinear_impl(X, x_dtype, M, K, gamma, eps, pkW, s_w, N, Y, y_dtype, Xq, s_x, 0, stream);
}

int bitnet_bitlinear_kernel(const void* X, int x_dtype, int64_t M, int64_t K, const float* gamma, float eps,
                            const uint8_t* pkW, const float* s_w, int64_t N, void* Y, int y_dtype, int8_t* Xq,
                            float* s_x, int kernel, void* stream) {
  return bitlinear_impl(X, x_dtype, M, K, gamma, eps, pkW, s_w, N, Y, y_dtype, Xq, s_x, kernel, stream);
}

int bitnet_add(const float* a, const float* b, float* out, int64_t n, void* stream) {
  const int c = elementwise_check(a, b, out, n);
  if (c != BITNET_OK) return c < 0 ? BITNET_OK : c;
  return cuda_status(bitnet::run_add_f32(a, b, out, (size_t)n, static_cast<cudaStream_t>(stream)));
}

int bitnet_relu2_glu(const float* gate, const float* up, float* out, int64_t n, void* stream) {
  const int c = elementwise_check(gate, up, out, n);
  if (c != BITNET_OK) return c < 0 ? BITNET_OK : c;
  return cuda_status(bitnet::run_relu2_glu(gate, up, out, (size_t)n, static_cast<cudaStream_t>(stream)));
}

static int attention_shape(int64_t B, int64_t L, int64_t t0, int heads, int head_dim, int64_t T_cap) {
  if (head_dim != 128 || heads < 1 || heads > 256) return BITNET_ERR_SHAPE;
  if (B < 0 || L < 0 || t0 < 0 || T_cap < 1 || T_cap > (int64_t(1) << 24) || t0 + L > T_cap) return BITNET_ERR_SHAPE;
  if (B * T_cap * heads * head_dim >= (int64_t(1) << 40) || B * L >= (int64_t(1) << 30) || B > 65535)
    return BITNET_ERR_SHAPE;
  return BITNET_OK;
}

int bitnet_rope_append(float* Q, const float* K, const float* V, int64_t B, int64_t L, int64_t t0, int heads,
                       int head_dim, double base, float* Kc, float* Vc, int64_t T_cap, void* stream) {
  const int sh = attention_shape(B, L, t0, heads, head_dim, T_cap);
  if (sh != BITNET_OK) return sh;
  if (!(base > 1.0) || !(base < 1e300)) return BITNET_ERR_SHAPE;
  if (B == 0 || L == 0) return BITNET_OK;
  if (!Q || !K || !V || !Kc || !Vc) return BITNET_ERR_NULL;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(Kc) || !aligned16(Vc)) return BITNET_ERR_ALIGN;
  int d = check_device();
  if (d != BITNET_OK) return d;
  return cuda_status(bitnet::run_rope_append(Q, K, V, (int)B, (int)L, (int)t0, heads, head_dim, base, Kc, Vc,
                                             (int)T_cap, static_cast<cudaStream_t>(stream)));
}

int bitnet_attention(const float* Q, const float* Kc, const float* Vc, int64_t B, int64_t L, int64_t t0, int heads,
                     int head_dim, int64_t T_cap, float* A, void* stream) {
  const int sh = attention_shape(B, L, t0, heads, head_dim, T_cap);
  if (sh != BITNET_OK) return sh;
  if (heads > 65535) return BITNET_ERR_SHAPE;
  if (B == 0 || L == 0) return BITNET_OK;
  if (!Q || !Kc || !Vc || !A) return BITNET_ERR_NULL;
  if (!aligned16(Q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(A)) return BITNET_ERR_ALIGN;
  int d = check_device();
  if (d != BITNET_OK) return d;
  return cuda_status(bitnet::run_attention(Q, Kc, Vc, (int)B, (int)L, (int)t0, heads, head_dim, (int)T_cap, A,
                                           static_cast<cudaStream_t>(stream)));
}

int bitnet_device_error(int* code_out) {
  int code = 0, zero = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) { cudaGetLastError(); return BITNET_ERR_CUDA; }
  if (cudaMemcpyFromSymbol(&code, bitnet::g_device_error, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(bitnet::g_device_error, &zero, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return BITNET_ERR_CUDA;
  }
  if (code_out) *code_out = code;
  return BITNET_OK;
}

}  // extern "C"
