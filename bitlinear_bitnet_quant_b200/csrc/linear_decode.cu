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
// * More than 8 tokens: the token groups can also be spread over adjacent
//   CTAs that share a weight slice (the second read of the slice hits L2), so
//   twice the warps issue MMAs on each SM and every CTA loads fewer
//   activation bytes after the wait.
// * Warp w takes the 64-wide K slice w of every segment; the eight partial
//   tiles meet in shared memory and one pass sums, shifts (>> 6, or >> 10 for
//   int4 activations held as 16*x) and dequantises:
//   y = float(acc) * ((1/s_x) * (1/s_w)) in fp32 round-to-nearest.
#include "decode_common.cuh"

namespace bitnet {

// TG = token groups of 8 (1: M <= 8, 2: M <= 16, 4: M <= 32); RG = groups of
// 16 weight rows per CTA (rows = 16 * RG).  Both are compile-time so that one
// K segment is a single straight-line block: the next segment's weight words
// are loaded while this one's MMAs issue, and consecutive MMAs never depend on
// each other (with one token group, the two MMAs of a 64-wide slice go to two
// accumulator sets, summed at the end).
//
// `tsplit` CTAs share each weight slice: CTA b takes rows (b / tsplit) * ROWS
// onwards and tokens 8 * TG * (b % tsplit) onwards.  W5: pkW holds the weights
// five per byte (trit5_row_bytes(K) bytes per row), rewritten into the 2-bit
// slice layout in shared memory before the dependency wait.
// A group of weight matrices sharing the activations runs in one launch: CTAs
// grp.first[g] .. grp.first[g+1]-1 stream matrix g (see LinGroup).
template <int ACT_BITS, int TG, int RG, typename TOut, bool W5>
__global__ void __launch_bounds__(DEC_THREADS, 2)
linear_decode_kernel(const __grid_constant__ LinGroup grp, const uint8_t* __restrict__ Xq,
                     const float* __restrict__ s_x, int M, int K, int tsplit) {
  using C = DecCfg<TG>;
  constexpr int TOK = C::TOK, PB = C::PASS_BATCH;
  constexpr int ROWS = 16 * RG;
  constexpr int NACC = C::NACC;
  constexpr int SHIFT = ACT_BITS == 8 ? 6 : 10;
  static_assert(RG >= 1 && RG <= C::RG_MAX, "row groups");
  extern __shared__ uint8_t dec_smem_raw[];
  __shared__ float sdq[TOK];
  __shared__ uint16_t lut5[W5 ? 243 : 1];

  uint8_t* wsm = smem_align(dec_smem_raw, 1024u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int nseg = K / 512;
  const int gi = group_of(grp, blockIdx.x);
  const int blk = blockIdx.x - grp.first[gi];
  const uint8_t* __restrict__ pkW = grp.pkW[gi];
  const float* __restrict__ s_w_ptr = grp.s_w[gi];
  TOut* __restrict__ Y = static_cast<TOut*>(grp.Y[gi]);
  int32_t* __restrict__ acc_dbg = grp.acc_dbg[gi];
  const int N = grp.N[gi];
  const int n0 = (blk / tsplit) * ROWS;
  const size_t xrow = ACT_BITS == 8 ? (size_t)K : (size_t)K / 2;
  {
    const int m0 = (blk % tsplit) * TOK;            // this CTA's first token
    M = M - m0 < TOK ? M - m0 : TOK;
    Xq += (size_t)m0 * xrow;
    s_x += m0;
    Y += (size_t)m0 * N;
    if (acc_dbg) acc_dbg += (size_t)m0 * N;
  }

  // This kernel holds no tensor memory, so the next kernel in the stream may
  // be scheduled at once (it only waits for this grid to finish).
  pdl_launch_dependents();
  // the weights do not depend on the previous kernel: stream them now
  const int r5 = trit5_row_bytes(K);
  uint8_t* stage = wsm + dec_stage_offset<TG, RG>(K);
  if constexpr (W5) {
    dec_copy_trit5<ROWS>(pkW, N, r5, n0, stage);
    for (int b = threadIdx.x; b < 243; b += DEC_THREADS) lut5[b] = (uint16_t)trit5_codes(b);
  } else {
    dec_copy_weights<ROWS>(pkW, N, K, n0, wsm);
  }
  // s_w belongs to the weights: read it before the wait as well
  const float sw = threadIdx.x < TOK ? ldg_nc_f32(s_w_ptr) : 0.0f;
  if constexpr (W5) {
    cp_async_wait_all();
    __syncthreads();                           // staged bytes and the digit table
    dec_trit5_to_2bit<ROWS>(stage, r5, K, lut5, wsm);   // made visible by the loop's first barrier
  }
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
      dec_load_w<RG>(wsm, 0, warp, g, t, wcur);
    }
#pragma unroll
    for (int u = 0; u < PB; ++u) {
      const int s = u0 + u;
      if (s < nseg) {
        uint32_t wnxt[RG][2];
        dec_load_w<RG>(wsm, s + 1 < nseg ? s + 1 : s, warp, g, t, wnxt);   // next segment, ahead of use
        dec_segment_mma<TG, RG, NACC>(d, wcur, xv[u]);
#pragma unroll
        for (int rg = 0; rg < RG; ++rg) { wcur[rg][0] = wnxt[rg][0]; wcur[rg][1] = wnxt[rg][1]; }
      }
    }
  }

  if (threadIdx.x < M && threadIdx.x < TOK) sdq[threadIdx.x] = __fmul_rn(__fdiv_rn(1.0f, sx), __fdiv_rn(1.0f, sw));
  // the partial tiles reuse the weight slice's memory (after the epilogue's barrier)
  dec_epilogue<TG, RG, NACC, SHIFT>(d, reinterpret_cast<int32_t*>(wsm), sdq, M, N, n0, Y, acc_dbg);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
bool decode_path_applies(int M, int K) {
  return M >= 1 && M <= DEC_MAX_TOKENS && K % 512 == 0 && K / 512 <= DEC_MAX_SEGS;
}

// Shared memory of one CTA: the 2-bit slice (reused by the epilogue's partial
// tiles), then, for five-per-byte weights, the staged rows.
template <int TG, int RG>
static size_t dec_smem_bytes(int K, bool w5) {
  return dec_stage_offset<TG, RG>(K) + (w5 ? (size_t)16 * RG * trit5_row_bytes(K) : 0) + 1024;
}

template <int ACT_BITS, int TG, int RG, typename TOut, bool W5>
static cudaError_t launch_decode_rg(LinGroup grp, const void* Xq, const float* s_x, int M, int K, int tsplit,
                                    cudaStream_t st) {
  constexpr int ROWS = 16 * RG;
  const size_t smem = dec_smem_bytes<TG, RG>(K, W5);
  auto kern = linear_decode_kernel<ACT_BITS, TG, RG, TOut, W5>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  grp.first[0] = 0;
  for (int g = 0; g < grp.count; ++g) grp.first[g + 1] = grp.first[g] + (grp.N[g] + ROWS - 1) / ROWS * tsplit;
  for (int g = grp.count + 1; g <= GROUP_MAX; ++g) grp.first[g] = grp.first[grp.count];
  const dim3 grid((unsigned)grp.first[grp.count]);
  return launch_pdl(kern, grid, dim3(DEC_THREADS), smem, st, 1u, grp, static_cast<const uint8_t*>(Xq), s_x, M, K,
                    tsplit);
}

template <int ACT_BITS, int TG, typename TOut, bool W5>
static cudaError_t launch_decode_t(const LinGroup& grp, const void* Xq, const float* s_x, int M, int K, int tsplit,
                                   cudaStream_t st) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int n_all = 0;
  for (int g = 0; g < grp.count; ++g) n_all += grp.N[g];
  // one CTA per weight slice (up to 8 tokens): slices sized for two CTAs per
  // SM, which halves each warp's MMA chain (measured on B200: 8 tokens
  // 3.5 -> 2.9 us at N = 6912, K = 2560); with the token groups spread over
  // CTAs the grid already holds two per SM
  const int rg = decode_rows(n_all, K, sms * (tsplit == 1 ? 2 : 1), DecCfg<TG>::MAX_ROWS) / 16;
#define BN_RG(R) launch_decode_rg<ACT_BITS, TG, (R <= DecCfg<TG>::RG_MAX ? R : 1), TOut, W5>(grp, Xq, s_x, M, K, tsplit, st)
  switch (rg) {
    case 1: return BN_RG(1);
    case 2: return BN_RG(2);
    case 3: return BN_RG(3);
    default: return BN_RG(4);
  }
#undef BN_RG
}

template <bool W5>
static cudaError_t dispatch_decode(const LinGroup& grp, const void* Xq, int act_bits, const float* s_x, int M, int K,
                                   int y_bf16, cudaStream_t st) {
  // up to 16 tokens: one token group per CTA (two CTAs per weight slice past
  // 8 tokens); up to 32: two token groups per CTA, two CTAs per slice, except
  // for long rows (K > 4096), where four CTAs of one token group share a slice
  // (measured on B200 at 32 tokens: the 5632-wide down projection 7.2 -> 6.6 us;
  // the 2048-wide products are faster with two groups per CTA)
#define BN_DEC(BITS, T)                                                                     \
  return M <= 8    ? launch_decode_t<BITS, 1, T, W5>(grp, Xq, s_x, M, K, 1, st)            \
         : M <= 16 ? launch_decode_t<BITS, 1, T, W5>(grp, Xq, s_x, M, K, 2, st)            \
         : K > 4096 ? launch_decode_t<BITS, 1, T, W5>(grp, Xq, s_x, M, K, (M + 7) / 8, st) \
                   : launch_decode_t<BITS, 2, T, W5>(grp, Xq, s_x, M, K, (M + 15) / 16, st)
  if (act_bits == 8) {
    if (y_bf16) { BN_DEC(8, __nv_bfloat16); } else { BN_DEC(8, float); }
  } else {
    if (y_bf16) { BN_DEC(4, __nv_bfloat16); } else { BN_DEC(4, float); }
  }
#undef BN_DEC
}

static LinGroup single_group(const uint8_t* pkW, const float* s_w, int N, void* Y, int32_t* acc_dbg) {
  LinGroup g = {};
  g.pkW[0] = pkW;
  g.s_w[0] = s_w;
  g.Y[0] = Y;
  g.acc_dbg[0] = acc_dbg;
  g.N[0] = N;
  g.count = 1;
  return g;
}

cudaError_t run_linear_decode(const void* Xq, int act_bits, const float* s_x, const uint8_t* pkW, const float* s_w,
                              int M, int N, int K, void* Y, int y_bf16, int32_t* acc_dbg, cudaStream_t st) {
  return dispatch_decode<false>(single_group(pkW, s_w, N, Y, acc_dbg), Xq, act_bits, s_x, M, K, y_bf16, st);
}

// Several weight matrices that share the activations, in one launch.
cudaError_t run_linear_decode_group(const LinGroup& grp, const void* Xq, int act_bits, const float* s_x, int M, int K,
                                    int y_bf16, cudaStream_t st) {
  return dispatch_decode<false>(grp, Xq, act_bits, s_x, M, K, y_bf16, st);
}

// Weights five per byte (trit5_row_bytes(K) bytes per row); same shapes as the
// 2-bit decode path, results bit-identical to it.
cudaError_t run_linear_decode_trit5(const void* Xq, int act_bits, const float* s_x, const uint8_t* pk5,
                                    const float* s_w, int M, int N, int K, void* Y, int y_bf16, int32_t* acc_dbg,
                                    cudaStream_t st) {
  return dispatch_decode<true>(single_group(pk5, s_w, N, Y, acc_dbg), Xq, act_bits, s_x, M, K, y_bf16, st);
}

}  // namespace bitnet
