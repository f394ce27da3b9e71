// Fused BitLinear forward with int8 activations for a few tokens: RMSNorm,
// per-token absmax int8 ("LLM을 1.58비트로 파인튜닝: BitNet을 이용한 극단적인
// 양자화", section 양자화 메커니즘) and the ternary product with its
// dequantisation (sections 계산 패러다임, 추론 최적화 및 커스텀 커널), in one
// kernel.  Codes, scales, accumulators and outputs are bit-identical to
// bitnet_quant_act followed by bitnet_linear.
//
// Every CTA needs the codes of all tokens over the whole K range.  CTAs work
// in thread-block clusters of FUSE_CLUSTER: CTA r of a cluster quantises the
// tokens m = r, r + FUSE_CLUSTER, ... (one warp per token) into a staging row
// of its shared memory (codes, then the scale), and one bulk copy per cluster
// CTA delivers that row into the same place of every CTA's activation buffer,
// completing on the receiver's mbarrier.  The GEMV then reads its fragments
// from shared memory; weights are staged and multiplied exactly as in the
// decode kernel (decode_common.cuh).
//
// Quantisation of one token by one warp, fixed fp32 arithmetic:
//   ss: squares summed by the balanced pairwise tree over element indices,
//       zero padded to a power of two: E elements of a 16-byte chunk, the 32
//       consecutive chunks of the lanes (xor shuffles), then the iterations
//       through a binary-counter cascade (pairs, then quads, ... in order);
//   r = 1 / sqrt(ss / K + eps);  y = (x * r) * gamma;
//   s = 127 / max(max|y|, 1e-5);  q = clamp(rint(y * s), -128, 127).
#include "decode_common.cuh"
#include "quant_common.cuh"

namespace bitnet {

constexpr int FUSE_CLUSTER = 8;
constexpr size_t FUSE_SMEM_MAX = 200 * 1024;

// Quantises one token row (K elements) with the calling warp; codes go to
// `qrow` (this CTA's shared memory) and, if `gq` is not null, to global
// memory.  Returns the scale s on every lane.
template <typename TIn>
BN_DEV float warp_quant_row_i8(const TIn* __restrict__ xrow, int K, const float* __restrict__ gamma, float eps,
                               int8_t* qrow, int8_t* gq, int lane) {
  constexpr int E = InVec<TIn>::E;
  constexpr int B = 4;                         // chunks per lane in flight
  const int C = K / E;
  int PC = 32;
  while (PC < C) PC <<= 1;
  const int ITW = PC / 32;                     // iterations (power of two)

  // ---- pass 1: sum of squares ----
  float stk[8];
#pragma unroll
  for (int l = 0; l < 8; ++l) stk[l] = 0.f;
  int cnt = 0;
  for (int it0 = 0; it0 < ITW; it0 += B) {
    float v[B][E];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int j = (it0 + b) * 32 + lane;
      if (it0 + b < ITW && j < C) {
        InVec<TIn>::load(xrow + (size_t)j * E, v[b]);
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) v[b][e] = 0.f;
      }
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
      if (it0 + b < ITW) {
        float sq[E];
#pragma unroll
        for (int e = 0; e < E; ++e) sq[e] = __fmul_rn(v[b][e], v[b][e]);
        float p = warp_tree_sum(tree_sum<E>(sq));
        // push p: combine with the completed subtrees of equal size (bit l of
        // the count set: a subtree of 2^l iterations waits in stk[l]), in order
        bool placed = false;
#pragma unroll
        for (int l = 0; l < 8; ++l) {
          if (!placed) {
            if ((cnt >> l) & 1) {
              p = __fadd_rn(stk[l], p);
            } else {
              stk[l] = p;
              placed = true;
            }
          }
        }
        ++cnt;
      }
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int l = 0; l < 8; ++l)
    if ((1 << l) == ITW) ss = stk[l];

  const float ms = __fdiv_rn(ss, (float)K);
  const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));

  // ---- pass 2: normalise, absmax (the chunks are reread from L1) ----
  auto norm_chunk = [&](int j, float (&v)[E]) {
    InVec<TIn>::load(xrow + (size_t)j * E, v);
    if (gamma != nullptr) {
#pragma unroll
      for (int q = 0; q < E / 4; ++q) {
        const uint4 u = ldg_nc_v4(gamma + (size_t)j * E + 4 * q);
        v[4 * q] = __fmul_rn(__fmul_rn(v[4 * q], r), __uint_as_float(u.x));
        v[4 * q + 1] = __fmul_rn(__fmul_rn(v[4 * q + 1], r), __uint_as_float(u.y));
        v[4 * q + 2] = __fmul_rn(__fmul_rn(v[4 * q + 2], r), __uint_as_float(u.z));
        v[4 * q + 3] = __fmul_rn(__fmul_rn(v[4 * q + 3], r), __uint_as_float(u.w));
      }
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = __fmul_rn(v[e], r);
    }
  };
  float amax = 0.f;
  for (int j0 = 0; j0 < C; j0 += 32 * B) {
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int j = j0 + 32 * b + lane;
      if (j < C) {
        float v[E];
        norm_chunk(j, v);
#pragma unroll
        for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(v[e]));
      }
    }
  }
  amax = warp_max(amax);
  const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));

  // ---- pass 3: codes ----
  for (int j0 = 0; j0 < C; j0 += 32 * B) {
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int j = j0 + 32 * b + lane;
      if (j < C) {
        float v[E];
        norm_chunk(j, v);
        uint32_t packed[E / 4];
#pragma unroll
        for (int q = 0; q < E / 4; ++q) {
          uint32_t w = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            int c = __float2int_rn(__fmul_rn(v[4 * q + e], s));
            c = max(-128, min(127, c));
            w |= (uint32_t)(c & 0xFF) << (8 * e);
          }
          packed[q] = w;
        }
        if constexpr (E == 8) {
          *reinterpret_cast<uint2*>(qrow + (size_t)j * E) = make_uint2(packed[0], packed[1]);
          if (gq) *reinterpret_cast<uint2*>(gq + (size_t)j * E) = make_uint2(packed[0], packed[1]);
        } else {
          *reinterpret_cast<uint32_t*>(qrow + (size_t)j * E) = packed[0];
          if (gq) *reinterpret_cast<uint32_t*>(gq + (size_t)j * E) = packed[0];
        }
      }
    }
  }
  return s;
}

// Shared memory: weight slice (later the epilogue's partial tiles), the
// activation buffer [M][K + 64] (codes, the scale at byte K; the pitch makes
// the fragment loads conflict-free), staging rows [tokens per CTA][K + 16].
template <int TG, int RG>
inline size_t fused_smem_bytes(int M, int K) {
  const size_t wbytes = (size_t)16 * RG * K / 4, rbytes = dec_red_bytes<TG, RG>();
  const int ml = (M + FUSE_CLUSTER - 1) / FUSE_CLUSTER;
  return (wbytes > rbytes ? wbytes : rbytes) + (size_t)M * (K + 64) + (size_t)ml * (K + 16) + 1024;
}

template <typename TIn, int TG, int RG, typename TOut>
__global__ void __launch_bounds__(DEC_THREADS, 2)
bitlinear_fused_kernel(const TIn* __restrict__ X, int M, int K, const float* __restrict__ gamma, float eps,
                       const uint8_t* __restrict__ pkW, const float* __restrict__ s_w_ptr, int N,
                       TOut* __restrict__ Y, int8_t* __restrict__ Xq, float* __restrict__ s_x) {
  using C = DecCfg<TG>;
  constexpr int TOK = C::TOK, ROWS = 16 * RG, NACC = C::NACC;
  static_assert(RG >= 1 && RG <= C::RG_MAX, "row groups");
  extern __shared__ uint8_t fuse_smem_raw[];
  __shared__ __align__(8) uint64_t bar_x;
  __shared__ float sdq[TOK];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int nseg = K / 512;
  const int n0 = blockIdx.x * ROWS;
  const int rank = blockIdx.x % FUSE_CLUSTER;          // cluster = FUSE_CLUSTER x 1 x 1
  const bool first_cluster = blockIdx.x < FUSE_CLUSTER;
  const int xpitch = K + 64, spitch = K + 16;
  const uint32_t row_bytes = (uint32_t)K + 16u;        // codes and the scale

  uint8_t* wsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fuse_smem_raw) + 1023) & ~uintptr_t(1023));
  const size_t wbytes = (size_t)ROWS * K / 4, rbytes = dec_red_bytes<TG, RG>();
  uint8_t* xbuf = wsm + (wbytes > rbytes ? wbytes : rbytes);
  uint8_t* stage = xbuf + (size_t)M * xpitch;

  // No tensor memory here: the next kernel in the stream may be scheduled at once.
  pdl_launch_dependents();
  dec_copy_weights<ROWS>(pkW, N, K, n0, wsm);
  if (threadIdx.x == 0) {
    mbar_init(&bar_x, 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(&bar_x, (uint32_t)M * row_bytes);   // every token's row, from its owner
  }
  cluster_arrive();                            // (release) this CTA's barrier is initialised
  const float sw = threadIdx.x < TOK ? ldg_nc_f32(s_w_ptr) : 0.0f;
  pdl_wait();                                  // X comes from the previous kernel

  // ---- this CTA's tokens: one warp each ----
  const int m = rank + FUSE_CLUSTER * warp;
  const bool quantiser = m < M;
  if (quantiser) {
    int8_t* qrow = reinterpret_cast<int8_t*>(stage + (size_t)warp * spitch);
    const float s = warp_quant_row_i8<TIn>(X + (size_t)m * K, K, gamma, eps, qrow,
                                           first_cluster ? Xq + (size_t)m * K : nullptr, lane);
    if (lane == 0) {
      *reinterpret_cast<float*>(qrow + K) = s;
      if (first_cluster) s_x[m] = s;
    }
    fence_proxy_async_smem();                  // the row is read by the bulk copies
    __syncwarp();
  }
  cluster_wait();                              // every CTA of the cluster has initialised its barrier
  if (quantiser && lane == 0) {
    const uint32_t src_row = (uint32_t)m * (uint32_t)xpitch;
    for (int dst = 0; dst < FUSE_CLUSTER; ++dst)
      bulk_copy_to_cluster(cluster_map(smem_u32(xbuf) + src_row, dst), stage + (size_t)warp * spitch, row_bytes,
                           cluster_map(smem_u32(&bar_x), dst));
  }

  // ---- weights landed, activations of all tokens landed ----
  cp_async_wait_all();
  const bool ok = __syncthreads_and(mbar_wait_cluster(&bar_x, 0, DEV_ERR_TIMEOUT_CLUSTER));
  if (threadIdx.x < M && threadIdx.x < TOK) {
    const float sx = *reinterpret_cast<const float*>(xbuf + (size_t)threadIdx.x * xpitch + K);
    sdq[threadIdx.x] = __fmul_rn(__fdiv_rn(1.0f, sx), __fdiv_rn(1.0f, sw));
  }

  int d[NACC][RG][TG][4];
#pragma unroll
  for (int h = 0; h < NACC; ++h)
#pragma unroll
    for (int rg = 0; rg < RG; ++rg)
#pragma unroll
      for (int tg = 0; tg < TG; ++tg)
#pragma unroll
        for (int j = 0; j < 4; ++j) d[h][rg][tg][j] = 0;

  if (ok) {
    // activation fragments of segment sg: 16 bytes of token 8 tg + g at K offset 512 sg + 64 warp + 16 t
    auto load_x = [&](int sg, uint4 (&xv)[TG]) {
#pragma unroll
      for (int tg = 0; tg < TG; ++tg) {
        const int mm = 8 * tg + g;
        xv[tg] = mm < M ? *reinterpret_cast<const uint4*>(xbuf + (size_t)mm * xpitch + 512 * sg + 64 * warp + 16 * t)
                        : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    uint32_t wcur[RG][2];
    uint4 xcur[TG];
    dec_load_w<RG>(wsm, 0, warp, g, t, wcur);
    load_x(0, xcur);
    for (int sg = 0; sg < nseg; ++sg) {
      const int nx = sg + 1 < nseg ? sg + 1 : sg;
      uint32_t wnxt[RG][2];
      uint4 xnxt[TG];
      dec_load_w<RG>(wsm, nx, warp, g, t, wnxt);
      load_x(nx, xnxt);
      dec_segment_mma<TG, RG, NACC>(d, wcur, xcur);
#pragma unroll
      for (int rg = 0; rg < RG; ++rg) { wcur[rg][0] = wnxt[rg][0]; wcur[rg][1] = wnxt[rg][1]; }
#pragma unroll
      for (int tg = 0; tg < TG; ++tg) xcur[tg] = xnxt[tg];
    }
  }

  // partial tiles reuse the weight slice's memory (after the epilogue's barrier)
  dec_epilogue<TG, RG, NACC, 6>(d, reinterpret_cast<int32_t*>(wsm), sdq, ok ? M : 0, N, n0, Y,
                                static_cast<int32_t*>(nullptr));
  // the staging row must stay in place until the copies have read it
  if (quantiser && lane == 0) bulk_wait_read();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <typename TIn, int TG, int RG, typename TOut>
static cudaError_t launch_fused_rg(const void* X, int M, int K, const float* gamma, float eps, const uint8_t* pkW,
                                   const float* s_w, int N, void* Y, int8_t* Xq, float* s_x, size_t smem,
                                   cudaStream_t st) {
  constexpr int ROWS = 16 * RG;
  auto kern = bitlinear_fused_kernel<TIn, TG, RG, TOut>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  const int ctas = (N + ROWS - 1) / ROWS;
  const dim3 grid((unsigned)(((ctas + FUSE_CLUSTER - 1) / FUSE_CLUSTER) * FUSE_CLUSTER));
  return launch_pdl(kern, grid, dim3(DEC_THREADS), smem, st, dim3(FUSE_CLUSTER, 1, 1), static_cast<const TIn*>(X), M,
                    K, gamma, eps, pkW, s_w, N, static_cast<TOut*>(Y), Xq, s_x);
}

template <typename TIn, int TG, typename TOut>
static cudaError_t launch_fused_t(const void* X, int M, int K, const float* gamma, float eps, const uint8_t* pkW,
                                  const float* s_w, int N, void* Y, int8_t* Xq, float* s_x, int rg, cudaStream_t st) {
#define BN_FRG(R)                                                                                       \
  launch_fused_rg<TIn, TG, (R <= DecCfg<TG>::RG_MAX ? R : 1), TOut>(X, M, K, gamma, eps, pkW, s_w, N, Y, \
                                                                    Xq, s_x,                            \
                                                                    fused_smem_bytes<TG, (R <= DecCfg<TG>::RG_MAX ? R : 1)>(M, K), st)
  switch (rg) {
    case 1: return BN_FRG(1);
    case 2: return BN_FRG(2);
    case 3: return BN_FRG(3);
    default: return BN_FRG(4);
  }
#undef BN_FRG
}

static int fused_rg(int M, int N, int K) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int max_rows = M <= 16 ? DecCfg<2>::MAX_ROWS : DecCfg<4>::MAX_ROWS;
  return decode_rows(N, K, sms, max_rows) / 16;
}

// True when one fused kernel covers the shape (else two kernels run).
// (largest row-group count of each token-group count: an upper bound of the
// shared memory any of its kernels takes)
bool fused_path_applies(int M, int K) {
  if (M < 1 || M > DEC_MAX_TOKENS || K % 512 != 0 || K > 8192) return false;
  const size_t smem = M <= 8 ? fused_smem_bytes<1, 4>(M, K) : M <= 16 ? fused_smem_bytes<2, 4>(M, K)
                                                                       : fused_smem_bytes<4, 2>(M, K);
  return smem <= FUSE_SMEM_MAX;
}

cudaError_t run_quant_act_i8(const void* X, int bf16, int M, int K, const float* gamma, float eps, int8_t* Xq,
                             float* s_x, cudaStream_t st);
cudaError_t run_linear(const void* Xq, int act_bits, const float* s_x, const uint8_t* pkW, const float* s_w,
                       int M, int N, int K, void* Y, int y_bf16, int32_t* acc_dbg, int path, cudaStream_t st);

cudaError_t run_bitlinear(const void* X, int x_bf16, int M, int K, const float* gamma, float eps, const uint8_t* pkW,
                          const float* s_w, int N, void* Y, int y_bf16, int8_t* Xq, float* s_x, int path,
                          cudaStream_t st) {
  if (path == 0 && fused_path_applies(M, K)) {
    const int rg = fused_rg(M, N, K);
#define BN_FT(TIN, TOUT)                                                                                    \
  return M <= 8    ? launch_fused_t<TIN, 1, TOUT>(X, M, K, gamma, eps, pkW, s_w, N, Y, Xq, s_x, rg, st)       \
         : M <= 16 ? launch_fused_t<TIN, 2, TOUT>(X, M, K, gamma, eps, pkW, s_w, N, Y, Xq, s_x, rg, st)       \
                   : launch_fused_t<TIN, 4, TOUT>(X, M, K, gamma, eps, pkW, s_w, N, Y, Xq, s_x, rg, st)
    if (x_bf16) {
      if (y_bf16) { BN_FT(uint16_t, __nv_bfloat16); } else { BN_FT(uint16_t, float); }
    } else {
      if (y_bf16) { BN_FT(float, __nv_bfloat16); } else { BN_FT(float, float); }
    }
#undef BN_FT
  }
  // two kernels: the quantiser, then the linear layer (any kernel family)
  cudaError_t e = run_quant_act_i8(X, x_bf16, M, K, gamma, eps, Xq, s_x, st);
  if (e != cudaSuccess) return e;
  return run_linear(Xq, 8, s_x, pkW, s_w, M, N, K, Y, y_bf16, nullptr, path, st);
}

}  // namespace bitnet
