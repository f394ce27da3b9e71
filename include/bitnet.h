/*
 * bitnet.h - C ABI of the B200 (sm_100a) BitNet b1.58 BitLinear forward.
 *
 * The BitLinear layer replaces a linear layer by ternary weights {-1, 0, +1}
 * and 8-bit activations; BitNet v2's H-BitLinear adds a Hadamard transform
 * and 4-bit activations.  Sources, by page title and section:
 *   [P1] "초저용량 LLM의 진화: BitNet v2 파헤치기 (1비트 LLM을 위한 4비트 활성화)",
 *        section 방법론 (Hadamard before 4-bit activation quantisation).
 *   [P2] "AI 혁신의 선두: 마이크로소프트의 1비트 LLM, BitNet b1.58 2B4T",
 *        section 주요 아키텍처 혁신 (ternary weights by absmean; no bias terms).
 *   [P4] "LLM을 1.58비트로 파인튜닝: BitNet을 이용한 극단적인 양자화",
 *        sections 양자화 메커니즘 (absmean weight scale, per-token absmax int8,
 *        norm before activation quantisation), 계산 패러다임 (integer matmul),
 *        주요 결과 (four weights per int8), 추론 최적화 및 커스텀 커널 (unpack
 *        weights on the fly inside the matmul).
 *   [P5] "양자화(quantization) 1.58bit" (endplan.ai), absmax paragraph
 *        (factor 127/absmax; dequantise by dividing by it).
 *
 * Conventions for every entry point:
 *   - Pointers to tensors are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or keeps them.  `stream` is a cudaStream_t (NULL =
 *     the legacy default stream).  Calls are asynchronous: they only enqueue
 *     kernels (and, for bitnet_quantize_weights, one memset of the workspace).
 *   - Row-major layouts: X [M][K] (M tokens, K input features), W [N][K]
 *     (N output features), Y [M][N].
 *   - Every argument is validated on the host before anything is enqueued; on
 *     any error nothing is enqueued and a bitnet_status code is returned.
 *     Launch failures return BITNET_ERR_CUDA (cudaGetLastError is consumed).
 *   - Tensor pointers must be 16-byte aligned (BITNET_ERR_ALIGN).
 *   - The current CUDA device must be sm_100 (BITNET_ERR_UNSUPPORTED).
 *   - Fixed arithmetic: fp32 with IEEE round-to-nearest-even, no fused
 *     multiply-add where a result decides an integer code.  Codes, packed
 *     weights and int32 accumulators are deterministic and bit-exact.
 */
#ifndef BITNET_B200_H
#define BITNET_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BITNET_API __attribute__((visibility("default")))
#else
#define BITNET_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BITNET_OK = 0,
  BITNET_ERR_NULL = 1,         /* a required pointer is NULL */
  BITNET_ERR_SHAPE = 2,        /* a size breaks the documented limits */
  BITNET_ERR_ALIGN = 3,        /* a tensor pointer is not 16-byte aligned */
  BITNET_ERR_DTYPE = 4,        /* unknown dtype or act_bits value */
  BITNET_ERR_CUDA = 5,         /* a CUDA call or kernel launch failed */
  BITNET_ERR_UNSUPPORTED = 6,  /* no sm_100 device, or the TMA encoder is missing */
  BITNET_ERR_WORKSPACE = 7     /* workspace missing or too small */
} bitnet_status;

typedef enum { BITNET_F32 = 0, BITNET_BF16 = 1 } bitnet_dtype;

/* Static description of a status code; never NULL, thread-safe. */
BITNET_API const char* bitnet_status_string(int status);

/* Version of this ABI (increments on any signature change). */
BITNET_API int bitnet_abi_version(void);

/* Bytes of workspace bitnet_quantize_weights needs (a small constant). */
BITNET_API size_t bitnet_quantize_weights_workspace_size(int64_t N, int64_t K);

/*
 * Offline absmean ternarisation and packing of a weight matrix [P4 양자화
 * 메커니즘, 주요 결과; P2 주요 아키텍처 혁신].
 *   mean = (sum of |W| computed exactly, rounded once to fp64) / (N*K) in fp64,
 *          rounded to fp32;  s_w = 1 / max(mean, 1e-5) in fp32;
 *   q    = clamp(rint(W * s_w), -1, 1).
 * W        : [N][K] fp32 or bf16 (w_dtype), finite values.
 * pkW      : out, [N][K/4] bytes.  Codes are 2-bit two's complement (-1 = 0b11,
 *            0 = 0b00, +1 = 0b01); in each little-endian 32-bit word holding
 *            16 consecutive weights of a row, weight 4j+i sits at bits 8i+2j.
 * s_w      : out, one fp32 on the device (the dequantisation uses 1/s_w).
 * workspace: device scratch of at least bitnet_quantize_weights_workspace_size
 *            bytes, 16-byte aligned, caller-owned; it is overwritten.
 * Limits   : N >= 1, K >= 16, K % 16 == 0, N*K < 2^31.
 * Ordering : the linear kernels load pkW and s_w before they wait for the
 *            kernel ahead of them in the stream (programmatic dependent
 *            launch).  This call therefore ends with an empty kernel launched
 *            without that attribute, so a bitnet_linear enqueued right after
 *            it on the same stream starts only once the weights are complete.
 *            Weights written by other means (a copy, another library) must be
 *            complete before the bitnet_linear call is enqueued, or be
 *            separated from it by a stream synchronisation or an event wait.
 */
BITNET_API int bitnet_quantize_weights(const void* W, int w_dtype, int64_t N, int64_t K,
                            uint8_t* pkW, float* s_w,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * Variant of bitnet_quantize_weights for callers that cannot allocate device
 * memory (no counterpart on the pages; this is a deployment convenience).
 * Examples: a plugin inside an application that owns every device allocation,
 * a runtime that reserves all of its memory up front, code that must avoid the
 * implicit synchronisation of cudaMalloc/cudaFree.  Same arguments, result and
 * bit-exact output as bitnet_quantize_weights, minus the workspace: the scratch
 * is a fixed 256-byte array inside this library's device memory, held on every
 * device that uses it until the library is unloaded.  The caller still owns W,
 * pkW and s_w.  No cudaMalloc, cudaFree or allocating routine is called.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current).  The address is
 *     cached for the device's primary context: do not call this entry point
 *     after cudaDeviceReset or under a context the caller created itself
 *     (cuCtxCreate).
 *   - Every call shares the one array and clears it before use; calls whose
 *     kernels overlap on the GPU (e.g. on two streams) race on it.
 *   - Limit: N*K <= BITNET_NOALLOC_MAX_WEIGHTS (what the fixed 64-bit counters
 *     absorb without overflow); larger tensors return BITNET_ERR_SHAPE.
 */
#define BITNET_NOALLOC_MAX_WEIGHTS 2147483647LL
BITNET_API int bitnet_quantize_weights_noalloc(const void* W, int w_dtype, int64_t N, int64_t K,
                                               uint8_t* pkW, float* s_w, void* stream);

/*
 * BitLinear activation path: RMSNorm, then per-token absmax int8
 * [P4 양자화 메커니즘; P5 absmax].  Per token (row of K values x):
 *   ss = sum of x*x by the balanced pairwise tree over element indices
 *        (zero padded to a power of two), fp32;
 *   r  = 1 / sqrt(ss / K + eps);  y = (x * r) * gamma;
 *   s_x = 127 / max(max|y|, 1e-5);  Xq = clamp(rint(y * s_x), -128, 127).
 * X     : [M][K] fp32 or bf16 (x_dtype).
 * gamma : [K] fp32, or NULL for all ones.
 * Xq    : out, [M][K] int8.   s_x: out, [M] fp32 (the dequantisation uses 1/s_x).
 * Limits: M >= 0 (M == 0 is a no-op), 16 <= K <= 16384, K % 16 == 0.
 */
BITNET_API int bitnet_quant_act(const void* X, int x_dtype, int64_t M, int64_t K,
                     const float* gamma, float eps, int8_t* Xq, float* s_x, void* stream);

/*
 * H-BitLinear activation path: RMSNorm, Walsh-Hadamard transform, per-token
 * absmax int4 [P1 방법론].  y as in bitnet_quant_act; then per block of
 * b = 2^L consecutive features the Sylvester-order transform by radix-2 stages
 * of stride 1, 2, ..., b/2 (pair (a, c) -> (a + c, a - c)), times
 * fp32(1/sqrt(b)), giving t;  s_x = 7 / max(max|t|, 1e-5);
 * codes = clamp(rint(t * s_x), -8, 7).
 * had_block: b, a power of two in [32, 8192] dividing K, or 0 for the largest
 *            power of two dividing K.
 * Xq4  : out, [M][K/2] bytes; code 2j in the low nibble of byte j, code 2j+1
 *        in the high nibble, two's complement.
 * s_x  : out, [M] fp32.
 * T_dbg: out, [M][K] fp32 transformed values t, or NULL (diagnostics only).
 * Limits: M >= 0, 128 <= K <= 16384, K % 128 == 0.
 */
BITNET_API int bitnet_hadamard_quant_act(const void* X, int x_dtype, int64_t M, int64_t K,
                              const float* gamma, float eps, int had_block,
                              uint8_t* Xq4, float* s_x, float* T_dbg, void* stream);

/*
 * The quantisers with the stacked layer's element-wise producer folded in
 * (one kernel instead of two; results bit-identical to calling bitnet_add or
 * bitnet_relu2_glu first) [P2 주요 아키텍처 혁신: squared ReLU; residuals]:
 * bitnet_add_quant_act:          H = A + B (fp32, written out), then
 *                                bitnet_quant_act of H (fp32 input).
 * bitnet_glu_hadamard_quant_act: x = (r * r) * up with r = max(gate, 0),
 *                                then bitnet_hadamard_quant_act of x
 *                                (fp32 input; x is not written out).
 * A, B, H, gate, up: [M][K] fp32, 16-byte aligned.  Other arguments and
 * limits as for the plain quantisers.
 */
BITNET_API int bitnet_add_quant_act(const float* A, const float* B, int64_t M, int64_t K, const float* gamma,
                         float eps, float* H, int8_t* Xq, float* s_x, void* stream);
BITNET_API int bitnet_glu_hadamard_quant_act(const float* gate, const float* up, int64_t M, int64_t K,
                                  const float* gamma, float eps, int had_block, uint8_t* Xq4, float* s_x,
                                  void* stream);

/*
 * Ternary x int8 (act_bits = 8) or ternary x int4 (act_bits = 4) product with
 * int32 accumulation and dequantisation [P4 계산 패러다임, 추론 최적화 및
 * 커스텀 커널, 양자화 메커니즘 ("rescaled"); P5 (divide by the factor)]:
 *   acc[m][n] = sum_k code_x[m][k] * w[n][k]      (exact int32)
 *   Y[m][n]   = float(acc) * ((1 / s_x[m]) * (1 / s_w))   in fp32,
 *   rounded to bf16 (nearest even) when y_dtype is BITNET_BF16.  No bias.
 * Xq     : [M][K] int8 (act_bits 8) or [M][K/2] packed int4 (act_bits 4).
 * s_x    : [M] fp32 from the matching quantiser.   s_w: one fp32 (device).
 * pkW    : [N][K/4] packed ternary weights from bitnet_quantize_weights.
 * Y      : out, [M][N] fp32 or bf16 (y_dtype).
 * acc_dbg: out, [M][N] int32 accumulators, or NULL (diagnostics only).
 * Limits : M >= 0, N >= 1, 128 <= K <= 65536, K % 128 == 0.
 * Kernels: up to 32 tokens with K % 512 == 0 and K <= 16384, a one-pass
 *          kernel on warp-level int8 MMA (each CTA streams a slice of whole
 *          weight rows); otherwise the tcgen05 tensor-core kernel.
 */
BITNET_API int bitnet_linear(const void* Xq, int act_bits, const float* s_x, const uint8_t* pkW,
                  const float* s_w, int64_t M, int64_t N, int64_t K,
                  void* Y, int y_dtype, int32_t* acc_dbg, void* stream);

/*
 * Several ternary products that share one quantised activation tensor, in one
 * launch: the Q, K and V projections of an attention block, or the up and gate
 * projections of a gated FFN ("AI 혁신의 선두: 마이크로소프트의 1비트 LLM, BitNet
 * b1.58 2B4T", 주요 아키텍처 혁신: every linear layer of attention and FFN is a
 * BitLinear; P4 계산 패러다임 for the product itself).  For g < count,
 *   Y[g] = bitnet_linear(Xq, act_bits, s_x, pkW[g], s_w[g], M, N[g], K),
 * bit for bit.  One launch streams every matrix of the group, so its fixed
 * costs (the wait on the previous kernel, the pipeline fill) are paid once.
 * pkW, s_w, N, Y: HOST arrays of `count` entries holding device pointers and
 *                 sizes; they are read during the call only.
 * Limits: 1 <= count <= 4; M, K and each N[g] as for bitnet_linear; one
 *         y_dtype for all outputs; no accumulator output.
 */
BITNET_API int bitnet_linear_group(const void* Xq, int act_bits, const float* s_x, int64_t M, int64_t K,
                                   int count, const uint8_t* const* pkW, const float* const* s_w,
                                   const int64_t* N, void* const* Y, int y_dtype, void* stream);

/*
 * Denser weight storage: five ternary weights per byte as base-3 digits,
 * 1.6 bits per weight instead of 2 ("양자화(quantization) 1.58bit", section
 * "1.58비트는 어디서 나온거에요?": three states carry log2(3) = 1.58 bits).
 * Byte g of a row = sum_i (w[5g + i] + 1) * 3^i for i = 0..4; weights past K
 * count as 0; each row is padded to bitnet_trit5_row_bytes(K) bytes (a
 * multiple of 16) with the byte of five zero weights, 121.
 *
 * bitnet_trit5_row_bytes: bytes per row, ceil(K / 5) rounded up to 16.
 * bitnet_repack_trit5: pkW [N][K/4] (bitnet_quantize_weights' 2-bit format,
 *   read) -> pk5 [N][bitnet_trit5_row_bytes(K)] (written).  Limits: N >= 1,
 *   16 <= K, K % 16 == 0, N * row bytes < 2^31; pointers 16-byte aligned.
 *   Like bitnet_quantize_weights it ends with an empty kernel launched without
 *   the programmatic attribute, so a bitnet_linear_trit5 enqueued right after
 *   it (which loads pk5 before its dependency wait) sees complete weights.
 * bitnet_linear_trit5: bitnet_linear with the weights in this format, for the
 *   decode shapes only (1 <= M <= 32, K % 512 == 0, K <= 16384; otherwise
 *   BITNET_ERR_SHAPE).  Each CTA stages its rows and rewrites them into the
 *   2-bit layout in shared memory before it waits for the previous kernel;
 *   results are bit-identical to bitnet_linear.  Other arguments as there.
 */
BITNET_API size_t bitnet_trit5_row_bytes(int64_t K);
BITNET_API int bitnet_repack_trit5(const uint8_t* pkW, int64_t N, int64_t K, uint8_t* pk5, void* stream);
BITNET_API int bitnet_linear_trit5(const void* Xq, int act_bits, const float* s_x, const uint8_t* pk5,
                        const float* s_w, int64_t M, int64_t N, int64_t K,
                        void* Y, int y_dtype, int32_t* acc_dbg, void* stream);

/*
 * Fused BitLinear forward with int8 activations: bitnet_quant_act followed by
 * bitnet_linear (act_bits = 8) in one call, with bit-identical results
 * [P4 양자화 메커니즘, 계산 패러다임, 추론 최적화 및 커스텀 커널].
 * X      : [M][K] fp32 or bf16 (x_dtype).   gamma: [K] fp32 or NULL (= 1).
 * pkW    : [N][K/4] packed ternary weights.  s_w: one fp32 (device).
 * Y      : out, [M][N] fp32 or bf16 (y_dtype).
 * Xq, s_x: out, [M][K] int8 codes and [M] fp32 scales (always written).
 * Kernels: the two kernels of bitnet_quant_act and bitnet_linear (on B200
 *          the faster choice for every decode shape measured: the quantiser
 *          overlaps the linear kernel's weight stream).  bitnet_bitlinear_kernel
 *          with kernel 4 runs one fused kernel instead: thread-block clusters
 *          of 8 CTAs share the quantisation (each CTA quantises every eighth
 *          token and copies codes and scale into the shared memory of the
 *          other seven), then the one-pass decode product; it covers up to
 *          32 tokens with K % 512 == 0 and K <= 8192 (else BITNET_ERR_SHAPE).
 * Limits : M >= 0, N >= 1, 128 <= K <= 16384, K % 128 == 0; gamma, X, Xq,
 *          pkW and Y 16-byte aligned.
 */
BITNET_API int bitnet_bitlinear(const void* X, int x_dtype, int64_t M, int64_t K, const float* gamma, float eps,
                     const uint8_t* pkW, const float* s_w, int64_t N, void* Y, int y_dtype,
                     int8_t* Xq, float* s_x, void* stream);

/*
 * Element-wise glue of the stacked BitLinear chain (a transformer layer whose
 * linear layers are BitLinear; P2 주요 아키텍처 혁신: squared ReLU, no bias).
 * bitnet_add:        out[i] = a[i] + b[i]                      (fp32 residual)
 * bitnet_relu2_glu:  out[i] = (r * r) * up[i],  r = max(gate[i], 0)
 * fp32, round-to-nearest, no fused multiply-add; out may alias an input.
 * Limits: n >= 0, n % 4 == 0; all pointers 16-byte aligned device pointers.
 */
BITNET_API int bitnet_add(const float* a, const float* b, float* out, int64_t n, void* stream);
BITNET_API int bitnet_relu2_glu(const float* gate, const float* up, float* out, int64_t n, void* stream);

/*
 * Diagnostics: bitnet_linear and bitnet_bitlinear with the kernel family
 * chosen per call instead of automatically; every choice computes the same
 * bit-exact result.  Arguments as for the plain calls, plus `kernel`:
 *   bitnet_linear_kernel:    0 = automatic (as bitnet_linear), 1 = CUDA-core
 *                            dp4a kernel, 2 = tcgen05 tensor-core kernel
 *                            with 128 weight rows per CTA,
 *                            3 = warp-MMA decode kernel (BITNET_ERR_SHAPE for
 *                            shapes it does not cover: M > 32, K % 512 != 0 or
 *                            K > 16384), 4 = tcgen05 kernel with 256 weight
 *                            rows per CTA, 5 = persistent tcgen05 kernel (one
 *                            CTA per SM over 128 x 128 tiles; int8 codes,
 *                            M > 64 and an even K / 128, else
 *                            BITNET_ERR_SHAPE).
 *   bitnet_bitlinear_kernel: 0-3 = the int8 quantiser, then that linear
 *                            kernel; 4 = the fused single kernel described at
 *                            bitnet_bitlinear (BITNET_ERR_SHAPE outside its range).
 * Any other value returns BITNET_ERR_SHAPE.  No state is kept between calls.
 */
BITNET_API int bitnet_linear_kernel(const void* Xq, int act_bits, const float* s_x, const uint8_t* pkW,
                                    const float* s_w, int64_t M, int64_t N, int64_t K, void* Y, int y_dtype,
                                    int32_t* acc_dbg, int kernel, void* stream);
BITNET_API int bitnet_bitlinear_kernel(const void* X, int x_dtype, int64_t M, int64_t K, const float* gamma,
                                       float eps, const uint8_t* pkW, const float* s_w, int64_t N, void* Y,
                                       int y_dtype, int8_t* Xq, float* s_x, int kernel, void* stream);

/*
 * Attention core of a stacked layer: rotary position embedding, a key/value
 * cache, and causal softmax attention ("AI 혁신의 선두: 마이크로소프트의 1비트 LLM,
 * BitNet b1.58 2B4T", 주요 아키텍처 혁신: rotary position embedding; the Q/K/V/O
 * projections around it are BitLinear).  The pages give no formula; the
 * definitions are the methods' own:
 *   RoPE: in each head of width d, the pair (x[2i], x[2i+1]) of a token at
 *         position p turns by the angle p * theta_i, theta_i = base^(-2i/d)
 *         (computed in fp64, rounded once to fp32);
 *   attention: per head, softmax(q k^T / sqrt(d)) v over the keys at
 *         positions 0 .. the query's own (fp32 arithmetic).
 * Layout: token rows [B*L][heads*d] fp32, where sequence b's L tokens sit at
 * positions t0 .. t0+L-1; caches Kc, Vc [B][T_cap][heads*d] fp32 whose row t
 * holds position t (rotated key; value).
 * bitnet_rope_append: rotates Q in place; writes the rotated K rows and the V
 *   rows into the caches at positions t0 .. t0+L-1.
 * bitnet_attention: A [B*L][heads*d] = attention of every query row over its
 *   sequence's cached keys 0 .. t0+l (the caches must hold them already).
 * Limits: head_dim == 128; t0 + L <= T_cap; base > 1; B, L >= 0 (0 is a no-op).
 */
BITNET_API int bitnet_rope_append(float* Q, const float* K, const float* V, int64_t B, int64_t L, int64_t t0,
                                  int heads, int head_dim, double base, float* Kc, float* Vc, int64_t T_cap,
                                  void* stream);
BITNET_API int bitnet_attention(const float* Q, const float* Kc, const float* Vc, int64_t B, int64_t L, int64_t t0,
                                int heads, int head_dim, int64_t T_cap, float* A, void* stream);

/*
 * Reads and clears the library's device-side error flag on the current
 * device (synchronises the device).  A kernel that waited more than ~2 s on
 * a pipeline barrier gives up, records a nonzero code here and returns; 0
 * means no such event.  Returns BITNET_OK or BITNET_ERR_CUDA.
 */
BITNET_API int bitnet_device_error(int* code_out);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_B200_H */
