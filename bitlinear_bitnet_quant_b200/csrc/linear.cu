// Ternary x int8 (or int4) product with int32 accumulation, dequantised by the
// activation and weight scales.
//
// "LLM을 1.58비트로 파인튜닝: BitNet을 이용한 극단적인 양자화": section 계산
// 패러다임 (the matmul uses integer additions), section 추론 최적화 및 커스텀
// 커널 (weights are unpacked on the fly inside the matmul) and section 타일링
// 매트릭스 곱셈 (tiles staged through on-chip memory).
//
// Unpacking trick used by both kernels: a 2-bit two's complement code placed
// in the top two bits of a byte is the int8 value 64*w, so one shift and one
// mask turn a packed word into four int8 weights; the int32 result is 64x the
// true sum and an arithmetic shift by 6 restores it exactly.  int4
// activations placed in the top nibble are 16*x, hence a shift by 10.
//
// Dequantisation: y = float(acc) * ((1/s_x) * (1/s_w)), fp32 round-to-nearest;
// |acc| < 2^24 so float(acc) is exact.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace bitnet {

template <typename T> BN_DEV void store_out(T* p, float v);
template <> BN_DEV void store_out<float>(float* p, float v) { *p = v; }
template <> BN_DEV void store_out<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

BN_DEV float dequant_scale(float sx, float sw) {
  return __fmul_rn(__fdiv_rn(1.0f, sx), __fdiv_rn(1.0f, sw));
}

// Four int8 weights (64*w) for k = 16g + 4j + 0..3 from packed word g.
BN_DEV uint32_t unpack4(uint32_t word, int j) {
  return (word << (6 - 2 * j)) & 0xC0C0C0C0u;
}

// Eight int4 codes of one packed word -> two words of four int8 (16*x), k order.
BN_DEV void widen8(uint32_t p, uint32_t& lo4, uint32_t& hi4) {
  const uint32_t ev = (p << 4) & 0xF0F0F0F0u;      // codes 0, 2, 4, 6
  const uint32_t od = p & 0xF0F0F0F0u;             // codes 1, 3, 5, 7
  lo4 = __byte_perm(ev, od, 0x5140);
  hi4 = __byte_perm(ev, od, 0x7362);
}

// ===========================================================================
// SIMT kernel: one warp per output row n and block of 16 tokens; lanes split
// K; dp4a accumulation.  Used for very small M and as a second GPU path.
// ===========================================================================
template <int ACT_BITS, typename TOut>
__global__ void __launch_bounds__(256)
linear_simt_kernel(const uint8_t* __restrict__ Xq, const float* __restrict__ s_x,
                   const uint32_t* __restrict__ pkW, const float* __restrict__ s_w_ptr,
                   int M, int N, int K, TOut* __restrict__ Y, int32_t* __restrict__ acc_dbg) {
  constexpr int MT = 16;
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int m0 = blockIdx.y * MT;
  if (n >= N) return;
  const int G = K / 16;
  const uint32_t* wrow = pkW + (size_t)n * G;
  int acc[MT];
#pragma unroll
  for (int t = 0; t < MT; ++t) acc[t] = 0;
  const int mcount = min(MT, M - m0);
  for (int g = lane; g < G; g += 32) {
    const uint32_t word = __ldg(wrow + g);
    uint32_t w4[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) w4[j] = unpack4(word, j);
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if (t < mcount) {
        uint32_t x4[4];
        if constexpr (ACT_BITS == 8) {
          const uint4 u = ldg_nc_v4(Xq + (size_t)(m0 + t) * K + 16 * g);
          x4[0] = u.x; x4[1] = u.y; x4[2] = u.z; x4[3] = u.w;
        } else {
          const uint2 u = __ldg(reinterpret_cast<const uint2*>(Xq + (size_t)(m0 + t) * (K / 2) + 8 * g));
          widen8(u.x, x4[0], x4[1]);
          widen8(u.y, x4[2], x4[3]);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[t] = __dp4a((int)x4[j], (int)w4[j], acc[t]);
      }
    }
  }
  const float sw = __ldg(s_w_ptr);
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    int a = acc[t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0 && t < mcount) {
      const int m = m0 + t;
      const int v = a >> (ACT_BITS == 8 ? 6 : 10);
      if (acc_dbg) acc_dbg[(size_t)m * N + n] = v;
      store_out(Y + (size_t)m * N + n, __fmul_rn((float)v, dequant_scale(__ldg(s_x + m), sw)));
    }
  }
}

// ===========================================================================
// tcgen05 kernel.  CTA tile: 128 output features (MMA M) x BN tokens (MMA N),
// K in steps of 128.  Operand A = the unpacked weights, written into tensor
// memory by the converter warps (no shared-memory round trip for them);
// operand B = the activation tile, brought by TMA into shared memory with the
// 128-byte swizzle (int4 tiles are widened there by the converter warps);
// D = int32 accumulators in tensor memory.
//   warp 0   : TMA producer
//   warp 1   : tensor-memory allocator and MMA issuer (one thread)
//   warps 2-5: converters, then the epilogue (tensor-memory lanes 32*(w%4)..)
// ===========================================================================
constexpr int TC_THREADS = 192;
constexpr int TC_BK = 128;
constexpr int TC_WBYTES = 128 * TC_BK / 4;       // packed W tile: 128 rows x 32 B

template <int BN, int ACT_BITS>
struct TcCfg {
  static constexpr int XBYTES = BN * 128;                      // int8 operand tile
  static constexpr int XRAW = ACT_BITS == 4 ? BN * 64 : 0;     // packed int4 tile
  static constexpr int STAGE = XBYTES + XRAW + TC_WBYTES;
  static constexpr int S_SMEM = (200 * 1024) / STAGE;
  static constexpr int S_TMEM = (512 - BN) / 32;
  static constexpr int S0 = S_SMEM < S_TMEM ? S_SMEM : S_TMEM;
  static constexpr int S = S0 > 6 ? 6 : S0;
  static constexpr int COLS_NEEDED = BN + 32 * S;
  static constexpr int TMEM_COLS = COLS_NEEDED <= 32 ? 32 : COLS_NEEDED <= 64 ? 64 :
                                   COLS_NEEDED <= 128 ? 128 : COLS_NEEDED <= 256 ? 256 : 512;
  static constexpr size_t SMEM = (size_t)S * STAGE + 1024;
  static_assert(S >= 2, "pipeline needs two stages");
};

template <int BN, int ACT_BITS, typename TOut>
__global__ void __launch_bounds__(TC_THREADS, 1)
linear_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                 const float* __restrict__ s_x, const float* __restrict__ s_w_ptr,
                 int M, int N, int K, TOut* __restrict__ Y, int32_t* __restrict__ acc_dbg) {
  using C = TcCfg<BN, ACT_BITS>;
  constexpr int S = C::S;
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ __align__(8) uint64_t bar_full[S], bar_empty[S], bar_conv[S], bar_acc;
  __shared__ uint32_t tmem_base_sh;
  __shared__ float sdq[BN];

  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
  auto xs = [&](int s) { return base + (size_t)s * C::XBYTES; };                          // 1024-aligned
  auto xraw = [&](int s) { return base + (size_t)S * C::XBYTES + (size_t)s * C::XRAW; };
  auto ws = [&](int s) { return base + (size_t)S * (C::XBYTES + C::XRAW) + (size_t)s * TC_WBYTES; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * 128;
  const int m0 = blockIdx.y * BN;
  const int nk = K / TC_BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1 + 4);
      mbar_init(&bar_conv[s], 4);
    }
    mbar_init(&bar_acc, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      constexpr uint32_t XTX = ACT_BITS == 8 ? BN * 128 : BN * 64;
      int issued = 0;
      for (int i = 0; i < nk; ++i) {
        const int s = i % S, r = i / S;
        if (r > 0 && !mbar_wait(&bar_empty[s], (r - 1) & 1, DEV_ERR_TIMEOUT_EMPTY)) break;
        mbar_arrive_expect_tx(&bar_full[s], TC_WBYTES + XTX);
        tma_load_2d(ws(s), &tmW, &bar_full[s], i * (TC_BK / 4), n0);
        if constexpr (ACT_BITS == 8) tma_load_2d(xs(s), &tmX, &bar_full[s], i * TC_BK, m0);
        else tma_load_2d(xraw(s), &tmX, &bar_full[s], i * (TC_BK / 2), m0);
        issued = i + 1;
      }
      // every copy issued has landed before the CTA may exit (returns at once
      // on the normal path, where the consumers have already waited for them)
      for (int i = issued - S < 0 ? 0 : issued - S; i < issued; ++i)
        mbar_wait(&bar_full[i % S], (i / S) & 1, DEV_ERR_TIMEOUT_FULL, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_i8(128, BN);
      for (int i = 0; i < nk; ++i) {
        const int s = i % S, r = i / S;
        if (!mbar_wait(&bar_full[s], r & 1, DEV_ERR_TIMEOUT_FULL)) break;
        if (!mbar_wait(&bar_conv[s], r & 1, DEV_ERR_TIMEOUT_A)) break;
        tc_fence_after();
        const uint32_t xaddr = smem_u32(xs(s));
#pragma unroll
        for (int kk = 0; kk < TC_BK / 32; ++kk) {
          const uint64_t bdesc = smem_desc_k_sw128(xaddr + kk * 32);
          const uint32_t aaddr = tmem + (uint32_t)(BN + 32 * s + 8 * kk);
          mma_i8_ts(tmem, aaddr, bdesc, IDESC, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bar_empty[s]);
      }
      mma_commit(&bar_acc);
      mbar_wait(&bar_acc, 0, DEV_ERR_TIMEOUT_ACC, false);   // no MMA in flight at teardown
    }
  } else {
    // ------------------------------------------------------------ converters
    const int q = warp & 3;                      // tensor-memory lane quarter
    const int row = 32 * q + lane;               // output feature inside the tile
    const int ct = threadIdx.x - 64;             // 0..127
    const float sw = __ldg(s_w_ptr);
    for (int j = ct; j < BN; j += 128) {
      const int m = m0 + j;
      sdq[j] = m < M ? dequant_scale(__ldg(s_x + m), sw) : 0.f;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);

    for (int i = 0; i < nk; ++i) {
      const int s = i % S, r = i / S;
      if (!mbar_wait_warp(&bar_full[s], r & 1, DEV_ERR_TIMEOUT_FULL)) break;
      tc_fence_after();
      // weights: 128 values of this row -> 32 tensor-memory columns
      const uint4* wp = reinterpret_cast<const uint4*>(ws(s) + 32 * row);
      const uint4 w0 = wp[0], w1 = wp[1];
      const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      uint32_t a[32];
#pragma unroll
      for (int g = 0; g < 8; ++g) {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) a[4 * g + jj] = unpack4(wv[g], jj);
      }
      tmem_st32(lane_base + (uint32_t)(BN + 32 * s), a);
      if constexpr (ACT_BITS == 4) {
        // int4 activation tile: widen to int8 (16*x) in the 128-byte-swizzled layout
        uint8_t* dst = xs(s);
        const uint8_t* src = xraw(s);
        for (int idx = ct; idx < BN * 8; idx += 128) {
          const int rr = idx >> 3, c = idx & 7;
          const uint2 p = *reinterpret_cast<const uint2*>(src + 64 * rr + 8 * c);
          uint32_t o0, o1, o2, o3;
          widen8(p.x, o0, o1);
          widen8(p.y, o2, o3);
          *reinterpret_cast<uint4*>(dst + 128 * rr + 16 * (c ^ (rr & 7))) = make_uint4(o0, o1, o2, o3);
        }
        fence_proxy_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar_conv[s]);
        mbar_arrive(&bar_empty[s]);
      }
    }

    // ------------------------------------------------------------ epilogue
    if (mbar_wait_warp(&bar_acc, 0, DEV_ERR_TIMEOUT_ACC)) {
      tc_fence_after();
      const int n = n0 + row;
      constexpr int SHIFT = ACT_BITS == 8 ? 6 : 10;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(lane_base + (uint32_t)c0, v);
        tmem_wait_ld();
        if (n < N) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int m = m0 + c0 + jj;
            if (m < M) {
              const int acc = (int)v[jj] >> SHIFT;
              if (acc_dbg) acc_dbg[(size_t)m * N + n] = acc;
              store_out(Y + (size_t)m * N + n, __fmul_rn((float)acc, sdq[c0 + jj]));
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ===========================================================================
// host side
// ===========================================================================
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeFn get_encode() {
  static EncodeFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  }
  return fn;
}

static bool make_map_2d(CUtensorMap* map, const void* ptr, uint64_t inner_bytes, uint64_t rows,
                        uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner_bytes, rows};
  cuuint64_t strides[1] = {inner_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int ACT_BITS, typename TOut>
static cudaError_t launch_tc(const void* Xq, const float* s_x, const uint8_t* pkW, const float* s_w,
                             int M, int N, int K, void* Y, int32_t* acc_dbg, cudaStream_t st) {
  using C = TcCfg<BN, ACT_BITS>;
  CUtensorMap tmW, tmX;
  if (!make_map_2d(&tmW, pkW, (uint64_t)K / 4, (uint64_t)N, TC_BK / 4, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const bool ok = ACT_BITS == 8
      ? make_map_2d(&tmX, Xq, (uint64_t)K, (uint64_t)M, TC_BK, BN, CU_TENSOR_MAP_SWIZZLE_128B)
      : make_map_2d(&tmX, Xq, (uint64_t)K / 2, (uint64_t)M, TC_BK / 2, BN, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
  auto kern = linear_tc_kernel<BN, ACT_BITS, TOut>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((N + 127) / 128, (M + BN - 1) / BN);
  kern<<<grid, TC_THREADS, C::SMEM, st>>>(tmW, tmX, s_x, s_w, M, N, K, static_cast<TOut*>(Y), acc_dbg);
  return cudaGetLastError();
}

template <int ACT_BITS, typename TOut>
static cudaError_t dispatch_tc(const void* Xq, const float* s_x, const uint8_t* pkW, const float* s_w,
                               int M, int N, int K, void* Y, int32_t* acc_dbg, cudaStream_t st) {
  if (M <= 16) return launch_tc<16, ACT_BITS, TOut>(Xq, s_x, pkW, s_w, M, N, K, Y, acc_dbg, st);
  if (M <= 32) return launch_tc<32, ACT_BITS, TOut>(Xq, s_x, pkW, s_w, M, N, K, Y, acc_dbg, st);
  if (M <= 64) return launch_tc<64, ACT_BITS, TOut>(Xq, s_x, pkW, s_w, M, N, K, Y, acc_dbg, st);
  if (M <= 128) return launch_tc<128, ACT_BITS, TOut>(Xq, s_x, pkW, s_w, M, N, K, Y, acc_dbg, st);
  return launch_tc<256, ACT_BITS, TOut>(Xq, s_x, pkW, s_w, M, N, K, Y, acc_dbg, st);
}

template <int ACT_BITS, typename TOut>
static cudaError_t launch_simt(const void* Xq, const float* s_x, const uint8_t* pkW, const float* s_w,
                               int M, int N, int K, void* Y, int32_t* acc_dbg, cudaStream_t st) {
  dim3 grid((N + 7) / 8, (M + 15) / 16);
  linear_simt_kernel<ACT_BITS, TOut><<<grid, 256, 0, st>>>(
      static_cast<const uint8_t*>(Xq), s_x, reinterpret_cast<const uint32_t*>(pkW), s_w, M, N, K,
      static_cast<TOut*>(Y), acc_dbg);
  return cudaGetLastError();
}

bool tensor_map_encoder_available() { return get_encode() != nullptr; }

// path: 0 = automatic, 1 = SIMT, 2 = tcgen05
cudaError_t run_linear(const void* Xq, int act_bits, const float* s_x, const uint8_t* pkW, const float* s_w,
                       int M, int N, int K, void* Y, int y_bf16, int32_t* acc_dbg, int path, cudaStream_t st) {
  const bool tc = path == 2 || (path == 0 && M > 2);
#define BN_LIN(BITS, T)                                                                  \
  return tc ? dispatch_tc<BITS, T>(Xq, s_x, pkW, s_w, M, N, K, Y, acc_dbg, st)           \
            : launch_simt<BITS, T>(Xq, s_x, pkW, s_w, M, N, K, Y, acc_dbg, st)
  if (act_bits == 8) {
    if (y_bf16) { BN_LIN(8, __nv_bfloat16); } else { BN_LIN(8, float); }
  } else {
    if (y_bf16) { BN_LIN(4, __nv_bfloat16); } else { BN_LIN(4, float); }
  }
#undef BN_LIN
}

}  // namespace bitnet
