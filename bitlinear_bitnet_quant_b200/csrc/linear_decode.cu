// Decode path of the ternary linear layer: up to 32 tokens per call.
//
// Same arithmetic as the tensor-memory kernel ("LLM을 1.58비트로 파인튜닝:
// BitNet을 이용한 극단적인 양자화", sections 계산 패러다임 and 추론 최적화 및
// 커스텀 커널: integer products of ternary weights unpacked on the fly, int32
// sums, one dequantisation per output), organised for a handful of tokens,
// where the work is one pass over the packed weights:
//
// * Each CTA owns `rows` consecutive output features (16 to 64) and the whole
//   K range.  Its packed weights (rows x K/4 bytes) arrive by 16-byte
//   asynchronous copies issued before the wait on the previous kernel, so the
//   weight stream of this launch overlaps the tail of the one before.  (On
//   B200, tensor-memory-access bulk loads issued before that wait were seen
//   to complete only after it; per-thread copies are not held back.)  The
//   slice is stored as 128-byte lines, one per weight row and 512-wide K
//   segment, with the 16-byte chunks of line r rotated by XOR with (r & 7),
//   which makes every fragment load below conflict-free.
// * Warp-level int8 MMA, m16n8k32: the 16 MMA rows are weight rows, the 8
//   MMA columns are tokens (further column groups cover tokens 8-31), so a
//   single token wastes nothing on the weight side.  Thread (g, t) of a warp
//   takes packed word t of a 16-byte unit and feeds its four 2-bit quarters
//   (shifted into the top bits of each byte: int8 64*w) as the A fragments of
//   two MMAs; the matching activation bytes are one 16-byte load per token.
//   The K order inside an MMA is permuted identically on both sides, which
//   leaves the sum unchanged.
// * Warp w takes the 64-wide K slice w of every segment; the eight partial
//   tiles meet in shared memory and one pass sums, shifts (>> 6, or >> 10 for
//   int4 activations held as 16*x) and dequantises:
//   y = float(acc) * ((1/s_x) * (1/s_w)) in fp32 round-to-nearest.
#include <cuda_bf16.h>

#include "common.cuh"

namespace bitnet {

constexpr int DEC_WARPS = 8;
constexpr int DEC_THREADS = 32 * DEC_WARPS;
constexpr int DEC_MAX_TOKENS = 32;
constexpr int DEC_MAX_SEGS = 32;                 // K <= 16384
constexpr size_t DEC_W_SMEM_MAX = 96 * 1024;

// Per token-group count TG (groups of 8 tokens): weight rows per CTA and K
// segments whose activations are held in registers at once (the register
// budget is 128 per thread for two CTAs per SM).
template <int TG> struct DecCfg {
  static constexpr int TOK = 8 * TG;
  static constexpr int RG_MAX = TG == 4 ? 2 : 4;            // groups of 16 weight rows
  static constexpr int MAX_ROWS = 16 * RG_MAX;
  static constexpr int PASS_BATCH = TG == 4 ? 4 : 8;
};

template <typename T> BN_DEV void dec_store(T* p, float v);
template <> BN_DEV void dec_store<float>(float* p, float v) { *p = v; }
template <> BN_DEV void dec_store<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// D[16 x 8] += A[16 x 32] * B[32 x 8], s8 inputs, s32 accumulators.
BN_DEV void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16 int4 codes (8 bytes, code 2j in the low nibble of byte j) -> 16 int8
// values 16*x in K order.
BN_DEV uint4 widen16(uint2 p) {
  uint4 r;
  const uint32_t e0 = (p.x << 4) & 0xF0F0F0F0u, o0 = p.x & 0xF0F0F0F0u;
  const uint32_t e1 = (p.y << 4) & 0xF0F0F0F0u, o1 = p.y & 0xF0F0F0F0u;
  r.x = __byte_perm(e0, o0, 0x5140);
  r.y = __byte_perm(e0, o0, 0x7362);
  r.z = __byte_perm(e1, o1, 0x5140);
  r.w = __byte_perm(e1, o1, 0x7362);
  return r;
}

// TG = token groups of 8 (1: M <= 8, 2: M <= 16, 4: M <= 32); RG = groups of
// 16 weight rows per CTA (rows = 16 * RG).  Both are compile-time so that one
// K segment is a single straight-line block: the next segment's weight words
// are loaded while this one's MMAs issue, and consecutive MMAs never depend on
// each other (with one token group, the two MMAs of a 64-wide slice go to two
// accumulator sets, summed at the end).
template <int ACT_BITS, int TG, int RG, typename TOut>
__global__ void __launch_bounds__(DEC_THREADS, 2)
linear_decode_kernel(const uint8_t* __restrict__ pkW, const uint8_t* __restrict__ Xq,
                     const float* __restrict__ s_x, const float* __restrict__ s_w_ptr, int M, int N, int K,
                     TOut* __restrict__ Y, int32_t* __restrict__ acc_dbg) {
  using C = DecCfg<TG>;
  constexpr int TOK = C::TOK, PB = C::PASS_BATCH;
  constexpr int ROWS = 16 * RG;
  constexpr int NACC = TG == 1 ? 2 : 1;                      // accumulator sets
  constexpr int SHIFT = ACT_BITS == 8 ? 6 : 10;
  constexpr uint32_t SEG_BYTES = ROWS * 128u;
  static_assert(RG >= 1 && RG <= C::RG_MAX, "row groups");
  extern __shared__ uint8_t dec_smem_raw[];
  __shared__ float sdq[TOK];

  uint8_t* wsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dec_smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int nseg = K / 512;
  const int n0 = blockIdx.x * ROWS;

  // This kernel holds no tensor memory, so the next kernel in the stream may
  // be scheduled at once (it only waits for this grid to finish).
  pdl_launch_dependents();
  {
    // The weights do not depend on the previous kernel: stream them now.
    // Chunk c (16 bytes): segment (c / 8) / ROWS, row (c / 8) % ROWS, chunk c % 8.
    const size_t wrow = (size_t)K / 4;
    const int nchunks = nseg * ROWS * 8;
    const uint32_t sbase = smem_u32(wsm);
    for (int c = threadIdx.x; c < nchunks; c += DEC_THREADS) {
      const int q = c & 7, line = c >> 3;
      const int sg = line / ROWS, r = line - sg * ROWS;
      const bool in = n0 + r < N;                         // rows past N read as zeros
      const uint8_t* src = pkW + (in ? (size_t)(n0 + r) * wrow + 128 * (size_t)sg + 16 * q : 0);
      cp_async_16(sbase + sg * SEG_BYTES + (uint32_t)r * 128u + 16u * (uint32_t)(q ^ (r & 7)), src, in ? 16u : 0u);
    }
    cp_async_commit();
  }
  // s_w belongs to the weights: read it before the wait as well
  const float sw = threadIdx.x < TOK ? ldg_nc_f32(s_w_ptr) : 0.0f;
  pdl_wait();                                  // activations and s_x come from the previous kernel
  // issued now, consumed only in the epilogue
  const float sx = threadIdx.x < M && threadIdx.x < TOK ? ldg_f32(s_x + threadIdx.x) : 1.0f;

  int d[NACC][RG][TG][4];
#pragma unroll
  for (int h = 0; h < NACC; ++h)
#pragma unroll
    for (int rg = 0; rg < RG; ++rg)
#pragma unroll
      for (int tg = 0; tg < TG; ++tg)
#pragma unroll
        for (int j = 0; j < 4; ++j) d[h][rg][tg][j] = 0;

  // this thread's packed words of one segment: rows 16 rg + g and + 8, word t
  // of 16-byte chunk `warp` (stored at chunk warp ^ (row & 7); (row & 7) = g)
  const uint32_t woff = (uint32_t)g * 128u + 16u * (uint32_t)(warp ^ g) + 4u * (uint32_t)t;
  auto load_w = [&](int sg, uint32_t (&w)[RG][2]) {
    const uint8_t* base = wsm + (size_t)sg * SEG_BYTES + woff;
#pragma unroll
    for (int rg = 0; rg < RG; ++rg) {
      w[rg][0] = *reinterpret_cast<const uint32_t*>(base + rg * 2048);
      w[rg][1] = *reinterpret_cast<const uint32_t*>(base + rg * 2048 + 1024);
    }
  };

  const size_t xrow = ACT_BITS == 8 ? (size_t)K : (size_t)K / 2;
  uint32_t wcur[RG][2];
  for (int u0 = 0; u0 < nseg; u0 += PB) {
    // activation bytes of this warp's K slices: 16 consecutive K per token and segment
    uint4 xv[PB][TG];
#pragma unroll
    for (int u = 0; u < PB; ++u) {
      const int k0 = 512 * (u0 + u) + 64 * warp + 16 * t;
#pragma unroll
      for (int tg = 0; tg < TG; ++tg) {
        const int m = 8 * tg + g;
        xv[u][tg] = make_uint4(0u, 0u, 0u, 0u);
        if (u0 + u < nseg && m < M) {
          if constexpr (ACT_BITS == 8) {
            xv[u][tg] = ldg_v4(Xq + (size_t)m * xrow + k0);
          } else {
            const uint2 p = ldg_v2(Xq + (size_t)m * xrow + k0 / 2);
            xv[u][tg] = make_uint4(p.x, p.y, 0u, 0u);     // widened below, after every load is issued
          }
        }
      }
    }
    if constexpr (ACT_BITS == 4) {
#pragma unroll
      for (int u = 0; u < PB; ++u)
#pragma unroll
        for (int tg = 0; tg < TG; ++tg) xv[u][tg] = widen16(make_uint2(xv[u][tg].x, xv[u][tg].y));
    }
    if (u0 == 0) {
      cp_async_wait_all();                     // this thread's weight copies
      __syncthreads();                         // and everyone else's
      load_w(0, wcur);
    }
#pragma unroll
    for (int u = 0; u < PB; ++u) {
      const int s = u0 + u;
      if (s < nseg) {
        uint32_t wnxt[RG][2];
        load_w(s + 1 < nseg ? s + 1 : s, wnxt);            // next segment's words, ahead of use
        // quarters 0,1 (first MMA) and 2,3 (second MMA) of each packed word,
        // moved into the top two bits of every byte: int8 64 * w
        uint32_t a[RG][2][4];
#pragma unroll
        for (int rg = 0; rg < RG; ++rg) {
          const uint32_t wl = wcur[rg][0], wh = wcur[rg][1];
          a[rg][0][0] = (wl << 6) & 0xC0C0C0C0u;  a[rg][0][1] = (wh << 6) & 0xC0C0C0C0u;
          a[rg][0][2] = (wl << 4) & 0xC0C0C0C0u;  a[rg][0][3] = (wh << 4) & 0xC0C0C0C0u;
          a[rg][1][0] = (wl << 2) & 0xC0C0C0C0u;  a[rg][1][1] = (wh << 2) & 0xC0C0C0C0u;
          a[rg][1][2] = wl & 0xC0C0C0C0u;         a[rg][1][3] = wh & 0xC0C0C0C0u;
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int h = NACC == 2 ? q : 0;
#pragma unroll
          for (int rg = 0; rg < RG; ++rg)
#pragma unroll
            for (int tg = 0; tg < TG; ++tg)
              mma_s8_16832(d[h][rg][tg], a[rg][q][0], a[rg][q][1], a[rg][q][2], a[rg][q][3],
                           q == 0 ? xv[u][tg].x : xv[u][tg].z, q == 0 ? xv[u][tg].y : xv[u][tg].w);
        }
#pragma unroll
        for (int rg = 0; rg < RG; ++rg) { wcur[rg][0] = wnxt[rg][0]; wcur[rg][1] = wnxt[rg][1]; }
      }
    }
  }

  if (threadIdx.x < M && threadIdx.x < TOK) sdq[threadIdx.x] = __fmul_rn(__fdiv_rn(1.0f, sx), __fdiv_rn(1.0f, sw));
  __syncthreads();                             // all warps are done with the weight slice

  // partial tiles [warp][token][row], row pitch ROWS + 4 (conflict-free stores)
  constexpr int RP = ROWS + 4;
  int32_t* red = reinterpret_cast<int32_t*>(wsm);
  int32_t* mine = red + (size_t)warp * TOK * RP;
#pragma unroll
  for (int rg = 0; rg < RG; ++rg) {
#pragma unroll
    for (int tg = 0; tg < TG; ++tg) {
      int v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = NACC == 2 ? d[0][rg][tg][j] + d[NACC - 1][rg][tg][j] : d[0][rg][tg][j];
      const int tok = 8 * tg + 2 * t, r = 16 * rg + g;
      mine[tok * RP + r] = v[0];
      mine[(tok + 1) * RP + r] = v[1];
      mine[tok * RP + r + 8] = v[2];
      mine[(tok + 1) * RP + r + 8] = v[3];
    }
  }
  __syncthreads();
  const int mcount = M < TOK ? M : TOK;
  for (int idx = threadIdx.x; idx < mcount * ROWS; idx += DEC_THREADS) {
    const int m = idx / ROWS, nn = idx - m * ROWS;
    const int n = n0 + nn;
    if (n < N) {
      int acc = 0;
#pragma unroll
      for (int w = 0; w < DEC_WARPS; ++w) acc += red[((size_t)w * TOK + m) * RP + nn];
      acc >>= SHIFT;
      if (acc_dbg) acc_dbg[(size_t)m * N + n] = acc;
      dec_store(Y + (size_t)m * N + n, __fmul_rn((float)acc, sdq[m]));
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
bool decode_path_applies(int M, int K) {
  return M >= 1 && M <= DEC_MAX_TOKENS && K % 512 == 0 && K / 512 <= DEC_MAX_SEGS;
}

// Weight rows per CTA: spread N over the SMs in multiples of 16, at most
// max_rows, with the weight slice within the shared-memory budget.
static int decode_rows(int N, int K, int sms, int max_rows) {
  int rows = 16 * ((N + 16 * sms - 1) / (16 * sms));
  if (rows > max_rows) rows = max_rows;
  while (rows > 16 && (size_t)rows * (size_t)K / 4 > DEC_W_SMEM_MAX) rows -= 16;
  return rows;
}

template <int ACT_BITS, int TG, int RG, typename TOut>
static cudaError_t launch_decode_rg(const void* Xq, const float* s_x, const uint8_t* pkW, const float* s_w, int M,
                                    int N, int K, void* Y, int32_t* acc_dbg, cudaStream_t st) {
  constexpr int ROWS = 16 * RG;
  const size_t wbytes = (size_t)ROWS * (size_t)K / 4;
  const size_t rbytes = (size_t)DEC_WARPS * DecCfg<TG>::TOK * (size_t)(ROWS + 4) * sizeof(int32_t);
  const size_t smem = (wbytes > rbytes ? wbytes : rbytes) + 1024;
  auto kern = linear_decode_kernel<ACT_BITS, TG, RG, TOut>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((N + ROWS - 1) / ROWS));
  return launch_pdl(kern, grid, dim3(DEC_THREADS), smem, st, 1u, pkW, static_cast<const uint8_t*>(Xq), s_x, s_w, M, N,
                    K, static_cast<TOut*>(Y), acc_dbg);
}

template <int ACT_BITS, int TG, typename TOut>
static cudaError_t launch_decode_t(const void* Xq, const float* s_x, const uint8_t* pkW, const float* s_w, int M,
                                   int N, int K, void* Y, int32_t* acc_dbg, cudaStream_t st) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int rg = decode_rows(N, K, sms, DecCfg<TG>::MAX_ROWS) / 16;
#define BN_RG(R) launch_decode_rg<ACT_BITS, TG, (R <= DecCfg<TG>::RG_MAX ? R : 1), TOut>(Xq, s_x, pkW, s_w, M, N, K, Y, acc_dbg, st)
  switch (rg) {
    case 1: return BN_RG(1);
    case 2: return BN_RG(2);
    case 3: return BN_RG(3);
    default: return BN_RG(4);
  }
#undef BN_RG
}

cudaError_t run_linear_decode(const void* Xq, int act_bits, const float* s_x, const uint8_t* pkW, const float* s_w,
                              int M, int N, int K, void* Y, int y_bf16, int32_t* acc_dbg, cudaStream_t st) {
#define BN_DEC(BITS, T)                                                                           \
  return M <= 8    ? launch_decode_t<BITS, 1, T>(Xq, s_x, pkW, s_w, M, N, K, Y, acc_dbg, st)       \
         : M <= 16 ? launch_decode_t<BITS, 2, T>(Xq, s_x, pkW, s_w, M, N, K, Y, acc_dbg, st)       \
                   : launch_decode_t<BITS, 4, T>(Xq, s_x, pkW, s_w, M, N, K, Y, acc_dbg, st)
  if (act_bits == 8) {
    if (y_bf16) { BN_DEC(8, __nv_bfloat16); } else { BN_DEC(8, float); }
  } else {
    if (y_bf16) { BN_DEC(4, __nv_bfloat16); } else { BN_DEC(4, float); }
  }
#undef BN_DEC
}

}  // namespace bitnet
