// Pieces shared by the one-pass decode kernels (linear_decode.cu and
// bitlinear_fused.cu): the weight slice staged in shared memory, warp-level
// int8 MMA on unpacked ternary fragments, and the split-K-over-warps epilogue.
//
// Arithmetic ("LLM을 1.58비트로 파인튜닝: BitNet을 이용한 극단적인 양자화",
// sections 계산 패러다임 and 추론 최적화 및 커스텀 커널): integer products of
// ternary weights unpacked on the fly, exact int32 sums, then
// y = float(acc) * ((1/s_x) * (1/s_w)) in fp32 round-to-nearest.
//
// Weight slice: a CTA owns ROWS = 16 * RG consecutive weight rows and the
// whole K range, stored as 128-byte lines, one per (row, 512-wide K segment),
// segment-major; the 16-byte chunk c of line r sits at chunk c ^ (r & 7).
// MMA: m16n8k32, the 16 rows are weight rows and the 8 columns tokens.
// Thread (g, t) of warp w takes packed word t of chunk w (16 weights of K
// slice 64 w + 16 t) for rows g and g + 8; its four 2-bit quarters, moved to
// the top of each byte (int8 64 * w), are the A fragments of two MMAs whose
// B fragments are the 16 matching activation bytes of token g.  The K order
// inside an MMA is permuted identically on both sides.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace bitnet {

constexpr int DEC_WARPS = 8;
constexpr int DEC_THREADS = 32 * DEC_WARPS;
constexpr int DEC_MAX_TOKENS = 32;
constexpr int DEC_MAX_SEGS = 32;                 // K <= 16384
constexpr size_t DEC_W_SMEM_MAX = 96 * 1024;

// Per token-group count TG (groups of 8 tokens): row groups per CTA and K
// segments whose activations are held in registers at once (the register
// budget is 128 per thread for two CTAs per SM).
template <int TG> struct DecCfg {
  static constexpr int TOK = 8 * TG;
  static constexpr int RG_MAX = TG == 4 ? 2 : 4;            // groups of 16 weight rows
  static constexpr int MAX_ROWS = 16 * RG_MAX;
  static constexpr int PASS_BATCH = TG == 4 ? 4 : 8;
  static constexpr int NACC = TG == 1 ? 2 : 1;              // accumulator sets
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

// Issues the 16-byte copies of this CTA's weight slice (rows n0 .. n0+ROWS-1,
// rows past N read as zeros) into `wsm`; every thread commits one group.
template <int ROWS>
BN_DEV void dec_copy_weights(const uint8_t* __restrict__ pkW, int N, int K, int n0, uint8_t* wsm) {
  constexpr uint32_t SEG_BYTES = ROWS * 128u;
  const size_t wrow = (size_t)K / 4;
  const int nchunks = (K / 512) * ROWS * 8;
  const uint32_t sbase = smem_u32(wsm);
  // chunk c (16 bytes): segment (c / 8) / ROWS, row (c / 8) % ROWS, chunk c % 8
  for (int c = threadIdx.x; c < nchunks; c += DEC_THREADS) {
    const int q = c & 7, line = c >> 3;
    const int sg = line / ROWS, r = line - sg * ROWS;
    const bool in = n0 + r < N;
    const uint8_t* src = pkW + (in ? (size_t)(n0 + r) * wrow + 128 * (size_t)sg + 16 * q : 0);
    cp_async_16(sbase + sg * SEG_BYTES + (uint32_t)r * 128u + 16u * (uint32_t)(q ^ (r & 7)), src, in ? 16u : 0u);
  }
  cp_async_commit();
}

// ---------------------------------------------------------------------------
// Weights stored five per byte ("양자화(quantization) 1.58bit", section
// "1.58비트는 어디서 나온거에요?": three states carry log2(3) = 1.58 bits):
// byte g of a row holds w[5g .. 5g+4] as base-3 digits w + 1, least
// significant first, so 3^5 = 243 <= 256 and a weight costs 1.6 bits.  Rows
// are padded to 16 bytes.  The decode kernel stages a slice of these rows and
// rewrites it into the 2-bit slice layout above before the dependency wait.
// ---------------------------------------------------------------------------
__host__ __device__ inline int trit5_row_bytes(int K) { return ((K + 4) / 5 + 15) / 16 * 16; }

// The five weights of byte b as 2-bit two's complement codes, weight i at bits 2i.
BN_DEV uint32_t trit5_codes(int b) {
  uint32_t c = 0;
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    const int d = b % 3;
    b /= 3;
    c |= (uint32_t)((d - 1) & 3) << (2 * i);
  }
  return c;
}

// 16-byte asynchronous copies of rows n0 .. n0+ROWS-1 of the five-per-byte
// weights (row stride r5 bytes) into `stage`; rows past N read as zeros.
template <int ROWS>
BN_DEV void dec_copy_trit5(const uint8_t* __restrict__ pk5, int N, int r5, int n0, uint8_t* stage) {
  const int cpr = r5 / 16;
  const uint32_t sbase = smem_u32(stage);
  for (int c = threadIdx.x; c < ROWS * cpr; c += DEC_THREADS) {
    const int r = c / cpr, q = c - r * cpr;
    const bool in = n0 + r < N;
    const uint8_t* src = pk5 + (in ? (size_t)(n0 + r) * r5 + 16 * (size_t)q : 0);
    cp_async_16(sbase + (uint32_t)(r * r5 + 16 * q), src, in ? 16u : 0u);
  }
  cp_async_commit();
}

// Rewrites the staged slice into the 2-bit slice layout.  Packed word wi of a
// row (weights 16 wi .. 16 wi + 15) always draws on four consecutive bytes:
// their codes are laid end to end (weight m at bits 2m), then the 4 x 4 grid
// of 2-bit cells is transposed by two bit-field swaps, which puts weight
// 4j + i at bits 8i + 2j.
template <int ROWS>
BN_DEV void dec_trit5_to_2bit(const uint8_t* stage, int r5, int K, const uint16_t* lut5, uint8_t* wsm) {
  const int wpr = K / 16;
  for (int idx = threadIdx.x; idx < ROWS * wpr; idx += DEC_THREADS) {
    const int r = idx / wpr, wi = idx - r * wpr;
    const int k0 = 16 * wi, g0 = k0 / 5, o = k0 - 5 * g0;
    const uint8_t* src = stage + r * r5 + g0;
    uint32_t v = (uint32_t)lut5[src[0]] >> (2 * o);
#pragma unroll
    for (int n = 1; n < 4; ++n) v |= (uint32_t)lut5[src[n]] << (10 * n - 2 * o);
    uint32_t t = ((v >> 12) ^ v) & 0x0000F0F0u;     // swap the 2 x 2 blocks of cells
    v ^= t ^ (t << 12);
    t = ((v >> 6) ^ v) & 0x00CC00CCu;               // swap the cells inside each block
    v ^= t ^ (t << 6);
    const int sg = k0 >> 9, q = (k0 >> 6) & 7, tt = (k0 >> 4) & 3;
    *reinterpret_cast<uint32_t*>(wsm + (size_t)sg * (ROWS * 128) + r * 128 + 16 * (q ^ (r & 7)) + 4 * tt) = v;
  }
}

// This thread's packed words of segment sg: rows 16 rg + g and + 8, word t of
// chunk `warp` (stored at chunk warp ^ g).
template <int RG>
BN_DEV void dec_load_w(const uint8_t* wsm, int sg, int warp, int g, int t, uint32_t (&w)[RG][2]) {
  const uint8_t* base = wsm + (size_t)sg * (RG * 2048) + g * 128 + 16 * (warp ^ g) + 4 * t;
#pragma unroll
  for (int rg = 0; rg < RG; ++rg) {
    w[rg][0] = *reinterpret_cast<const uint32_t*>(base + rg * 2048);
    w[rg][1] = *reinterpret_cast<const uint32_t*>(base + rg * 2048 + 1024);
  }
}

// One K segment: 2 * RG * TG independent MMAs.  With one token group the two
// MMAs of a slice go to two accumulator sets.
template <int TG, int RG, int NACC>
BN_DEV void dec_segment_mma(int (&d)[NACC][RG][TG][4], const uint32_t (&w)[RG][2], const uint4 (&xv)[TG]) {
  // quarters 0,1 (first MMA) and 2,3 (second MMA) of each packed word, moved
  // into the top two bits of every byte: int8 64 * w
  uint32_t a[RG][2][4];
#pragma unroll
  for (int rg = 0; rg < RG; ++rg) {
    const uint32_t wl = w[rg][0], wh = w[rg][1];
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
                     q == 0 ? xv[tg].x : xv[tg].z, q == 0 ? xv[tg].y : xv[tg].w);
  }
}

// Shared-memory bytes of the epilogue's partial tiles.
template <int TG, int RG>
constexpr size_t dec_red_bytes() {
  return (size_t)DEC_WARPS * DecCfg<TG>::TOK * (16 * RG + 4) * sizeof(int32_t);
}

// Epilogue: the warps' partial tiles [warp][token][row] (row pitch ROWS + 4:
// conflict-free stores) meet in `red`; one pass sums, shifts and dequantises.
// Starts with a CTA barrier (the caller's last use of `red`'s memory is
// before it); sdq[m] = (1/s_x[m]) * (1/s_w) must be visible by then.
template <int TG, int RG, int NACC, int SHIFT, typename TOut>
BN_DEV void dec_epilogue(const int (&d)[NACC][RG][TG][4], int32_t* red, const float* sdq, int M, int N, int n0,
                         TOut* __restrict__ Y, int32_t* __restrict__ acc_dbg) {
  constexpr int TOK = DecCfg<TG>::TOK, ROWS = 16 * RG, RP = ROWS + 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  __syncthreads();
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

// Offset of the five-per-byte staging rows: after the 2-bit slice, which the
// epilogue's partial tiles reuse.
template <int TG, int RG>
__host__ __device__ inline size_t dec_stage_offset(int K) {
  const size_t wbytes = (size_t)16 * RG * (size_t)K / 4, rbytes = dec_red_bytes<TG, RG>();
  return wbytes > rbytes ? wbytes : rbytes;
}

// Weight rows per CTA: spread N over the SMs in multiples of 16, at most
// max_rows, with the weight slice within the shared-memory budget.
inline int decode_rows(int N, int K, int sms, int max_rows) {
  int rows = 16 * ((N + 16 * sms - 1) / (16 * sms));
  if (rows > max_rows) rows = max_rows;
  while (rows > 16 && (size_t)rows * (size_t)K / 4 > DEC_W_SMEM_MAX) rows -= 16;
  return rows;
}

}  // namespace bitnet
