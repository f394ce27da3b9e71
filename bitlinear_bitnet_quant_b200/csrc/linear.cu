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

// The epilogue's store of one output into the staged tile.  bf16: round to
// nearest even on the bit pattern with integer operations (the conversion
// instruction issues at a quarter of the rate); equal to __float2bfloat16_rn
// for every non-NaN input, and the dequantised outputs are never NaN.
template <typename T> BN_DEV void stage_out(T* p, float v);
template <> BN_DEV void stage_out<float>(float* p, float v) { *p = v; }
template <> BN_DEV void stage_out<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  const uint32_t u = __float_as_uint(v);
  *reinterpret_cast<uint16_t*>(p) = (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

// float(a) for |a| < 2^22 without the (quarter-rate) conversion instruction:
// a + 0x4B400000 is the bit pattern of 1.5 * 2^23 + a (consecutive fp32
// values are 1 apart there), and the subtraction is exact.
BN_DEV float small_int_to_float(int a) { return __fsub_rn(__int_as_float(a + 0x4B400000), 12582912.0f); }

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
// K; dp4a accumulation.  A second, independent GPU implementation, selected
// only through bitnet_linear_kernel (the tcgen05 kernel is faster at every M).
// ===========================================================================
template <int ACT_BITS, typename TOut>
__global__ void __launch_bounds__(256)
linear_simt_kernel(const uint8_t* __restrict__ Xq, const float* __restrict__ s_x,
                   const uint32_t* __restrict__ pkW, const float* __restrict__ s_w_ptr,
                   int M, int N, int K, TOut* __restrict__ Y, int32_t* __restrict__ acc_dbg) {
  constexpr int MT = 16;
  pdl_launch_dependents();
  pdl_wait();                                // Xq and s_x come from the previous kernel
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
          const uint4 u = ldg_v4(Xq + (size_t)(m0 + t) * K + 16 * g);
          x4[0] = u.x; x4[1] = u.y; x4[2] = u.z; x4[3] = u.w;
        } else {
          const uint2 u = ldg_v2(Xq + (size_t)(m0 + t) * (K / 2) + 8 * g);
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
      store_out(Y + (size_t)m * N + n, __fmul_rn((float)v, dequant_scale(ldg_f32(s_x + m), sw)));
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
//   warp 0    : TMA producer of the weight tiles (and the per-token
//               dequantisation scales)
//   warp 1    : tensor-memory allocator and MMA issuer (one thread)
//   warps 2-9 : converters, then the epilogue.  Warp w serves tensor-memory
//               lanes 32*(w%4).. and half (w-2)/4 of the K bytes of a step
//               (and of the token columns in the epilogue).
//   warp 10   : TMA producer of the activation tiles.  Measured on B200, the
//               tiles one warp issues land one after another (about 0.36 us
//               each, whatever their size); two issuing warps halve the wait.
// When the tiles alone leave SMs idle, K is split over a cluster of ksplit
// CTAs (grid z); partial sums travel to the leader by one bulk copy each.
// ===========================================================================
constexpr int TC_THREADS = 352;
constexpr int TC_XWARP = 10;                       // activation-tile producer
constexpr int TC_CONV_THREADS = 256;
constexpr int TC_BK = 128;

// MB = 128 or 256 weight rows per CTA.  With 256, two M = 128 MMAs (two
// accumulators, two A slices in tensor memory) share every activation tile:
// half the activation bytes per MMA, at one CTA per SM (all 512 columns).
// Measured on B200 (clock64 stamps per K step): in the steady state the
// 128 x 128 tile at two CTAs per SM issues a K step every ~850-900 cycles per
// CTA against 256 of MMA work, with each activation tile landing ~2500 cycles
// after its copy is issued; the SM then takes in ~45 bytes per clock of the
// 80 that the MMA rate needs, while the shared memory also serves the MMA's
// reads of the same tiles.  A CTA spends another ~2000 cycles before its
// first MMA and ~6000 in the epilogue, which the CTA sharing its SM overlaps
// only in part.
template <int BN, int ACT_BITS, int MB = 128>
struct TcCfg {
  static constexpr int RB = MB / 128;                          // row blocks = accumulators
  static constexpr int XBYTES = BN * 128;                      // int8 operand tile
  static constexpr int XRAW = ACT_BITS == 4 ? BN * 64 : 0;     // packed int4 tile
  static constexpr int WBYTES = MB * TC_BK / 4;                // packed W tile: MB rows x 32 B
  static constexpr int STAGE = XBYTES + XRAW + WBYTES;
  // One accumulator per row block: measured on B200, rotating tcgen05.mma over
  // several accumulators costs ~3x more per instruction than chaining into one.
  static constexpr int DCOLS = BN * RB;                        // accumulator columns
  static constexpr int ACOLS = 32 * RB;                        // A columns per stage
  // 256 columns: two CTAs share an SM, so one CTA's prologue and epilogue
  // overlap the other's MMAs (a 256-token or 256-row tile needs all 512 columns)
  static constexpr int TMEM_BUDGET = (BN <= 128 && RB == 1) ? 256 : 512;
  static constexpr int SMEM_BUDGET = TMEM_BUDGET == 256 ? 108 * 1024 : 200 * 1024;
  static constexpr int S_SMEM = SMEM_BUDGET / STAGE;
  static constexpr int S_TMEM = (TMEM_BUDGET - DCOLS) / ACOLS;
  // 128-row tile: one ring of stages (shared-memory stage s and tensor-memory
  // A slot s go together; two CTAs per SM keep enough steps in flight).
  // 256-row tile: one CTA per SM, so the shared-memory ring runs deeper than
  // the four A slots tensor memory has room for; each A slot is released by
  // its own MMA commit.
  static constexpr int S0 = S_SMEM < S_TMEM ? S_SMEM : S_TMEM;
  static constexpr int S = RB == 1 ? (S0 > 6 ? 6 : S0) : (S_SMEM > 8 ? 8 : S_SMEM);   // shared-memory stages
  static constexpr int ST = RB == 1 ? S : S_TMEM;                                      // tensor-memory A slots
  // K steps per copy: consecutive stages are filled in pairs by one 3-D box
  // each (measured on B200, the boxes one warp issues land one after another
  // at about 0.36 us each whatever their size, so fewer, larger boxes feed an
  // SM faster); a pair shares its full / empty barriers.
  static constexpr int P = (S % 2 == 0 && S >= 4) ? 2 : 1;
  static constexpr int SP = S / P;                                                     // pair stages
  static constexpr int COLS_NEEDED = DCOLS + ACOLS * ST;
  static constexpr int TMEM_COLS = COLS_NEEDED <= 32 ? 32 : COLS_NEEDED <= 64 ? 64 :
                                   COLS_NEEDED <= 128 ? 128 : COLS_NEEDED <= 256 ? 256 : 512;
  static constexpr size_t SMEM = (size_t)S * STAGE + 1024;
  static constexpr int HALF = BN / 2;                          // token columns per epilogue warp
  static_assert(S >= 2 && ST >= 2 && ST <= S, "pipeline needs two stages");
  static_assert((size_t)BN * 128 * 4 <= (size_t)S * STAGE, "output staging fits in the operand stages");
};

// G chunks of NC (8 or 16) consecutive columns of this thread's TMEM lane,
// starting at taddr, with a single wait for all of them.
template <int NC, int G>
BN_DEV void load_cols(uint32_t taddr, uint32_t (&v)[G][16]) {
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if constexpr (NC == 8) {
      uint32_t t[8];
      tmem_ld8(taddr + (uint32_t)(g * NC), t);
#pragma unroll
      for (int q = 0; q < 8; ++q) v[g][q] = t[q];
    } else {
      tmem_ld16(taddr + (uint32_t)(g * NC), v[g]);
    }
  }
  tmem_wait_ld();
}

// Tensor maps of a group's weight matrices and outputs (see LinGroup).
struct TcMaps {
  CUtensorMap w[GROUP_MAX];
  CUtensorMap y[GROUP_MAX];
};

template <int BN, int ACT_BITS, typename TOut, int MB>
__global__ void __launch_bounds__(TC_THREADS, (BN <= 128 && MB == 128) ? 2 : 1)
linear_tc_kernel(const __grid_constant__ TcMaps maps, const __grid_constant__ CUtensorMap tmX,
                 const __grid_constant__ LinGroup grp, int use_tma_store, const float* __restrict__ s_x,
                 int M, int K, int ksplit) {
  using C = TcCfg<BN, ACT_BITS, MB>;
  constexpr int RB = C::RB;
  constexpr int S = C::S, ST = C::ST;
  constexpr uint32_t XTX = ACT_BITS == 8 ? BN * 128 : BN * 64;      // activation bytes per stage
  constexpr uint32_t PART_BYTES = 128u * BN * 4u;                    // one split-K partial tile
  constexpr int NC = C::HALF < 16 ? C::HALF : 16;                    // epilogue column chunk
  constexpr int NCH = C::HALF / NC;                                  // chunks per epilogue warp
  constexpr int G = NCH < 2 ? NCH : 2;                               // chunks per TMEM-load wait
  extern __shared__ uint8_t dsmem_raw[];
  // wfull: weight tile landed; xfull: activation tile landed; conv: weights in TMEM (and, for
  // int4, activations widened); empty: stage free; acc: all MMAs done; sdq: scales ready;
  // red: split-K partials of the other ranks landed (leader only)
  // afree: the A slot's MMAs are done (used only when the A ring is shorter than the stage ring)
  constexpr int P = C::P, SP = C::SP;
  __shared__ __align__(8) uint64_t bar_wfull[SP], bar_xfull[SP], bar_empty[SP], bar_conv[ST], bar_afree[ST];
  __shared__ __align__(8) uint64_t bar_acc, bar_sdq, bar_red;
  __shared__ uint32_t tmem_base_sh;
  __shared__ __align__(16) float sdq[BN];

  uint8_t* base = smem_align(dsmem_raw, 1024u);
  auto xs = [&](int s) { return base + (size_t)s * C::XBYTES; };                          // 1024-aligned
  auto xraw = [&](int s) { return base + (size_t)S * C::XBYTES + (size_t)s * C::XRAW; };
  // packed weights of pair stage p: [row block][step of the pair][128 rows][32 B]
  auto wsp = [&](int p) { return base + (size_t)S * (C::XBYTES + C::XRAW) + (size_t)p * P * C::WBYTES; };
  // split-K partial sums, [slot][column][row] int32: in the leader, slot r-1 receives rank r;
  // in the other ranks, slot 0 stages the outgoing partial
  int32_t* red = reinterpret_cast<int32_t*>(base + (size_t)S * C::STAGE);
  // output staging for the TMA store, [token][128 features] (reuses the activation stages)
  TOut* ostage = reinterpret_cast<TOut*>(base);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the weight matrix of this tile (one of a group that shares the activations)
  const int gi = group_of(grp, blockIdx.x);
  const CUtensorMap* tmW = &maps.w[gi];
  const CUtensorMap* tmY = &maps.y[gi];
  const float* __restrict__ s_w_ptr = grp.s_w[gi];
  TOut* __restrict__ Y = static_cast<TOut*>(grp.Y[gi]);
  int32_t* __restrict__ acc_dbg = grp.acc_dbg[gi];
  const int N = grp.N[gi];
  const int n0 = (blockIdx.x - grp.first[gi]) * MB;
  const int m0 = blockIdx.y * BN;
  const int kr = blockIdx.z;                    // rank inside the cluster (cluster = 1 x 1 x ksplit)
  const int nk_all = K / TC_BK;
  const int kb = (int)((int64_t)nk_all * kr / ksplit);
  const int nk = (int)((int64_t)nk_all * (kr + 1) / ksplit) - kb;

  if (threadIdx.x == 0) {
    for (int p = 0; p < SP; ++p) {
      mbar_init(&bar_wfull[p], 1);
      mbar_init(&bar_xfull[p], 1);
      mbar_init(&bar_empty[p], 1 + 8);
    }
    for (int a = 0; a < ST; ++a) {
      mbar_init(&bar_conv[a], 8);
      mbar_init(&bar_afree[a], 1);
    }
    mbar_init(&bar_acc, 1);
    mbar_init(&bar_sdq, 1);
    mbar_init(&bar_red, 1);
    fence_barrier_init();
    if (kr == 0 && ksplit > 1) mbar_arrive_expect_tx(&bar_red, (uint32_t)(ksplit - 1) * PART_BYTES);
    tma_prefetch_desc(tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if (ksplit > 1) cluster_arrive();            // matched by a cluster_wait before any remote access
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  // Only now, with this CTA's tensor memory held, may the next kernel in the
  // stream be scheduled: a dependent CTA never takes tensor memory that a CTA
  // of this grid still has to allocate (later grids only wait on earlier ones).
  pdl_launch_dependents();

  // pair j covers K steps jP .. jP+P-1 and uses pair stage j % SP in round j / SP
  const int npairs = (nk + P - 1) / P;
  if (warp == 0) {
    // ------------------------------------------------------------ weight producer
    const int pre = npairs < SP ? npairs : SP;
    auto load_w = [&](int j) {
      const int p = j % SP;
      mbar_arrive_expect_tx(&bar_wfull[p], (uint32_t)(P * C::WBYTES));
#pragma unroll
      for (int rb = 0; rb < RB; ++rb)
        tma_load_3d(wsp(p) + rb * P * (C::WBYTES / RB), tmW, &bar_wfull[p], 0, n0 + 128 * rb, kb + j * P);
    };
    if (lane == 0)
      for (int j = 0; j < pre; ++j) load_w(j);   // weights do not depend on the previous kernel
    __syncwarp();
    pdl_wait();                                    // s_x comes from the previous kernel
    if (kr == 0) {
      if (lane == 0 && use_tma_store) tma_prefetch_desc(tmY);
      const float sw = ldg_nc_f32(s_w_ptr);
      for (int j = lane; j < BN; j += 32) {
        const int m = m0 + j;
        sdq[j] = m < M ? dequant_scale(ldg_f32(s_x + m), sw) : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_sdq);
    }
    if (lane == 0) {
      int issued = pre;
      for (int j = pre; j < npairs; ++j) {
        if (!mbar_wait(&bar_empty[j % SP], ((j / SP) - 1) & 1, DEV_ERR_TIMEOUT_EMPTY)) break;
        load_w(j);
        issued = j + 1;
      }
      // every copy issued has landed before the CTA may exit (returns at once
      // on the normal path, where the consumers have already waited for them)
      for (int j = issued - SP < 0 ? 0 : issued - SP; j < issued; ++j)
        mbar_wait(&bar_wfull[j % SP], (j / SP) & 1, DEV_ERR_TIMEOUT_FULL, false);
    }
  } else if (warp == TC_XWARP) {
    // ------------------------------------------------------------ activation producer
    if (lane == 0) {
      pdl_wait();                                  // the activations come from the previous kernel
      int issued = 0;
      for (int j = 0; j < npairs; ++j) {
        const int p = j % SP;
        if (j >= SP && !mbar_wait(&bar_empty[p], ((j / SP) - 1) & 1, DEV_ERR_TIMEOUT_EMPTY)) break;
        mbar_arrive_expect_tx(&bar_xfull[p], (uint32_t)P * XTX);
        // the pair's steps land in consecutive stages p P and p P + 1
        if constexpr (ACT_BITS == 8) tma_load_3d(xs(p * P), &tmX, &bar_xfull[p], 0, m0, kb + j * P);
        else tma_load_3d(xraw(p * P), &tmX, &bar_xfull[p], 0, m0, kb + j * P);
        issued = j + 1;
      }
      for (int j = issued - SP < 0 ? 0 : issued - SP; j < issued; ++j)
        mbar_wait(&bar_xfull[j % SP], (j / SP) & 1, DEV_ERR_TIMEOUT_FULL, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_i8(128, BN);
      for (int i = 0; i < nk; ++i) {
        const int s = i % S, r = i / S;
        const int a = i % ST, ra = i / ST;
        if (!mbar_wait(&bar_xfull[s / P], r & 1, DEV_ERR_TIMEOUT_FULL)) break;
        if (!mbar_wait(&bar_conv[a], ra & 1, DEV_ERR_TIMEOUT_A)) break;
        tc_fence_after();
        const uint32_t xaddr = smem_u32(xs(s));
        // all of one accumulator's MMAs of the step, then the other's: switching the
        // accumulator between consecutive MMAs costs about three times the MMA
#pragma unroll
        for (int rb = 0; rb < RB; ++rb) {
#pragma unroll
          for (int kk = 0; kk < TC_BK / 32; ++kk) {
            const uint64_t bdesc = smem_desc_k_sw128(xaddr + kk * 32);
            const uint32_t aaddr = tmem + (uint32_t)(C::DCOLS + C::ACOLS * a + 32 * rb + 8 * kk);
            mma_i8_ts(tmem + (uint32_t)(BN * rb), aaddr, bdesc, IDESC, (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        // a pair stage is released after its last step's MMAs (the commit
        // tracks every earlier MMA), and only if it is refilled
        if (s % P == P - 1 && i - (P - 1) + S < nk) mma_commit(&bar_empty[s / P]);
        if (ST < S && i + ST < nk) mma_commit(&bar_afree[a]);
      }
      mma_commit(&bar_acc);
      mbar_wait(&bar_acc, 0, DEV_ERR_TIMEOUT_ACC, false);   // no MMA in flight at teardown
    }
  } else {
    // ------------------------------------------------------------ converters
    const int q = warp & 3;                      // tensor-memory lane quarter
    const int h = (warp - 2) >> 2;               // which half of the K bytes / token columns
    const int row = 32 * q + lane;               // output feature inside the tile
    const int ct = threadIdx.x - 64;             // 0..255
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);

    for (int i = 0; i < nk; ++i) {
      const int s = i % S, r = i / S;
      const int a = i % ST, ra = i / ST;
      const int c = s % P;                         // step inside the pair
      if (!mbar_wait_warp(&bar_wfull[s / P], r & 1, DEV_ERR_TIMEOUT_FULL)) break;
      tc_fence_after();
      // 64 weights of this row (of each row block) -> 16 tensor-memory columns
      // the tile arrives with the 32-byte swizzle: the two 16-byte halves of
      // row r are swapped when bit 2 of r is set, so the eight rows a
      // quarter-warp reads fall on distinct banks
      uint4 w[RB];
#pragma unroll
      for (int rb = 0; rb < RB; ++rb)
        w[rb] = *reinterpret_cast<const uint4*>(wsp(s / P) + (rb * P + c) * (C::WBYTES / RB) + 32 * row +
                                                16 * (h ^ ((row >> 2) & 1)));
      if constexpr (ACT_BITS == 8) {
        __syncwarp();
        if (lane == 0 && c == P - 1) mbar_arrive(&bar_empty[s / P]);   // the pair's packed tiles consumed
      }
      if constexpr (ST < S) {
        // the A slot is free once the MMAs of step i - ST are done
        if (i >= ST && !mbar_wait_warp(&bar_afree[a], (ra - 1) & 1, DEV_ERR_TIMEOUT_A)) break;
        tc_fence_after();
      }
#pragma unroll
      for (int rb = 0; rb < RB; ++rb) {
        const uint32_t wv[4] = {w[rb].x, w[rb].y, w[rb].z, w[rb].w};
        uint32_t av[16];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) av[4 * g + jj] = unpack4(wv[g], jj);
        }
        tmem_st16(lane_base + (uint32_t)(C::DCOLS + C::ACOLS * a + 32 * rb + 16 * h), av);
      }
      if constexpr (ACT_BITS == 4) {
        // int4 activation tile: widen to int8 (16*x) in the 128-byte-swizzled layout
        if (!mbar_wait_warp(&bar_xfull[s / P], r & 1, DEV_ERR_TIMEOUT_FULL)) break;
        // all of a thread's 8-byte chunks are read before any is widened, so
        // their shared-memory latencies overlap
        constexpr int WI = (BN * 8 + TC_CONV_THREADS - 1) / TC_CONV_THREADS;
        uint8_t* dst = xs(s);
        const uint8_t* src = xraw(s);
        uint2 pk[WI];
#pragma unroll
        for (int u = 0; u < WI; ++u) {
          const int idx = ct + u * TC_CONV_THREADS;
          if (idx < BN * 8) pk[u] = *reinterpret_cast<const uint2*>(src + 64 * (idx >> 3) + 8 * (idx & 7));
        }
#pragma unroll
        for (int u = 0; u < WI; ++u) {
          const int idx = ct + u * TC_CONV_THREADS;
          if (idx < BN * 8) {
            const int rr = idx >> 3, c = idx & 7;
            uint32_t o0, o1, o2, o3;
            widen8(pk[u].x, o0, o1);
            widen8(pk[u].y, o2, o3);
            *reinterpret_cast<uint4*>(dst + 128 * rr + 16 * (c ^ (rr & 7))) = make_uint4(o0, o1, o2, o3);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && c == P - 1) mbar_arrive(&bar_empty[s / P]);
      }
      // Hand every step to the MMA issuer as soon as its operands are in place
      // (measured on B200: holding steps back to batch the tensor-memory store
      // waits cost 7 % on the int8 and 20 % on the int4 GEMM).
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_conv[a]);
    }

    // ------------------------------------------------------------ epilogue
    constexpr int SHIFT = ACT_BITS == 8 ? 6 : 10;
    // |acc| <= qmax * K: below 2^22 the cheap exact conversion applies
    const bool small_acc = (int64_t)(ACT_BITS == 8 ? 127 : 8) * K < (int64_t)(1 << 22);
    const int cbeg = h * C::HALF;                // this warp's token columns
    const bool acc_ok = mbar_wait_warp(&bar_acc, 0, DEV_ERR_TIMEOUT_ACC);
    tc_fence_after();
    if (kr > 0) {
      // split-K partner: stage the raw partial sums, then one bulk copy to the leader
#pragma unroll 1
      for (int g0 = 0; g0 < NCH; g0 += G) {
        uint32_t v[G][16];
        load_cols<NC, G>(lane_base + (uint32_t)(cbeg + g0 * NC), v);
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int jj = 0; jj < NC; ++jj)
            red[(cbeg + (g0 + g) * NC + jj) * 128 + row] = acc_ok ? (int32_t)v[g][jj] : 0;
      }
      fence_proxy_async_smem();
      cluster_wait();                              // the leader's barrier is initialised
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (ct == 0) {
        const uint32_t dst = cluster_map(smem_u32(red), 0) + (uint32_t)(kr - 1) * PART_BYTES;
        bulk_copy_to_cluster(dst, red, PART_BYTES, cluster_map(smem_u32(&bar_red), 0));
        bulk_wait_read();                          // the source may be released after this
      }
    } else {
      if (ksplit > 1) cluster_wait();
      const bool sdq_ok = mbar_wait_warp(&bar_sdq, 0, DEV_ERR_TIMEOUT_ACC);
      const bool red_ok = ksplit == 1 || mbar_wait_cluster(&bar_red, 0, DEV_ERR_TIMEOUT_CLUSTER);
      const bool ok = acc_ok && red_ok && sdq_ok;
#pragma unroll 1
      for (int rb = 0; rb < RB; ++rb) {
      const int n = n0 + 128 * rb + row;
      if (rb > 0 && use_tma_store) {
        // the thread that stored the previous row block waited for its copy
        asm volatile("bar.sync 1, 256;" ::: "memory");
      }
#pragma unroll 1
      for (int g0 = 0; g0 < NCH; g0 += G) {
        uint32_t v[G][16];
        load_cols<NC, G>(lane_base + (uint32_t)(BN * rb + cbeg + g0 * NC), v);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const int c0 = cbeg + (g0 + g) * NC;
          for (int pr = 1; pr < ksplit; ++pr) {
#pragma unroll
            for (int jj = 0; jj < NC; ++jj) v[g][jj] += (uint32_t)red[((pr - 1) * BN + c0 + jj) * 128 + row];
          }
          if (use_tma_store) {
            // the chunk's scales in registers (c0 is a multiple of 16), and the
            // conversion chosen once per chunk: measured on B200, the per-value
            // scale reads, conversion instructions and select made this loop
            // ~2/3 of the epilogue
            float sq[NC];
#pragma unroll
            for (int q4 = 0; q4 < NC / 4; ++q4) {
              const float4 f = *reinterpret_cast<const float4*>(sdq + c0 + 4 * q4);
              sq[4 * q4] = f.x; sq[4 * q4 + 1] = f.y; sq[4 * q4 + 2] = f.z; sq[4 * q4 + 3] = f.w;
            }
            if (!ok) {
#pragma unroll
              for (int jj = 0; jj < NC; ++jj) sq[jj] = 0.f;
            }
            TOut* dst = ostage + (size_t)c0 * 128 + row;
            if (small_acc) {
#pragma unroll
              for (int jj = 0; jj < NC; ++jj)
                stage_out(dst + jj * 128, __fmul_rn(small_int_to_float((int)v[g][jj] >> SHIFT), sq[jj]));
            } else {
#pragma unroll
              for (int jj = 0; jj < NC; ++jj)
                stage_out(dst + jj * 128, __fmul_rn((float)((int)v[g][jj] >> SHIFT), sq[jj]));
            }
          } else if (ok && n < N) {
#pragma unroll
            for (int jj = 0; jj < NC; ++jj) {
              const int m = m0 + c0 + jj;
              if (m < M) {
                const int acc = (int)v[g][jj] >> SHIFT;
                if (acc_dbg) acc_dbg[(size_t)m * N + n] = acc;
                store_out(Y + (size_t)m * N + n, __fmul_rn((float)acc, sdq[c0 + jj]));
              }
            }
          }
        }
      }
      if (use_tma_store) {
        // the staged tile leaves as one bulk tensor store (rows past M and
        // columns past N are dropped by the copy engine)
        fence_proxy_async_smem();
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (ct == 0 && ok) {
          tma_store_2d(tmY, ostage, n0 + 128 * rb, m0);
          bulk_wait_read();                        // the staging may be reused / released once read
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
  if (ksplit > 1 && (warp < 2 || warp == TC_XWARP)) cluster_wait();     // pairs this warp's cluster_arrive
}

// ===========================================================================
// Persistent variant of the int8 tcgen05 kernel (selectable per call, kernel
// 5): one CTA per SM loops over the 128 x 128 tiles (static round robin), with
// two accumulators in tensor memory and four epilogue warps of its own, so a
// tile's epilogue and the next tile's start overlap the K loop instead of
// adding to it.  Measured on B200 its K steps come no faster than those of one
// CTA of the two-per-SM kernel (~800 cycles), so it is slower overall.
//   warp 0     : weight-tile producer (two K steps per 3-D copy)
//   warp 1     : tensor-memory allocator (all 512 columns) and MMA issuer
//   warps 2-9  : converters (packed weights -> int8 in tensor memory)
//   warp 10    : activation-tile producer
//   warps 11-14: epilogue (tensor-memory lane quarter = warp % 4)
// Tensor memory: accumulators at columns 0 and 128, eight A slots of 32 from
// 256 (all 512 columns).  Shared memory: eight activation stages (16 KB), four
// weight pair stages (8 KB), the output staging tile (128 x 128 outputs): as
// many bytes in flight per SM as two CTAs of the non-persistent kernel hold.
// ===========================================================================
constexpr int PT_THREADS = 480;
constexpr int PT_S = 8;                          // K-step stages (pairs of two)
constexpr int PT_SP = PT_S / 2;
constexpr int PT_ST = 8;                         // tensor-memory A slots
constexpr int PT_XBYTES = 128 * 128;
constexpr int PT_WBYTES = 128 * 32;
constexpr int PT_EPI_WARP0 = 11;

template <typename TOut>
constexpr size_t pt_smem_bytes() {
  return (size_t)PT_S * PT_XBYTES + (size_t)PT_S * PT_WBYTES + (size_t)128 * 128 * sizeof(TOut) + 1024;
}

template <typename TOut>
__global__ void __launch_bounds__(PT_THREADS, 1)
linear_tc_persistent_kernel(const __grid_constant__ TcMaps maps, const __grid_constant__ CUtensorMap tmX,
                            const __grid_constant__ LinGroup grp, int use_tma_store, const float* __restrict__ s_x,
                            int M, int K) {
  constexpr int S = PT_S, SP = PT_SP, ST = PT_ST;
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ __align__(8) uint64_t bar_wfull[SP], bar_xfull[SP], bar_empty[SP], bar_conv[ST];
  __shared__ __align__(8) uint64_t bar_accf[2], bar_acce[2], bar_fin;
  __shared__ uint32_t tmem_base_sh;
  __shared__ __align__(16) float sdq[128];

  uint8_t* base = smem_align(dsmem_raw, 1024u);
  auto xs = [&](int st) { return base + (size_t)st * PT_XBYTES; };
  auto wsp = [&](int pp) { return base + (size_t)S * PT_XBYTES + (size_t)pp * 2 * PT_WBYTES; };
  TOut* ostage = reinterpret_cast<TOut*>(base + (size_t)S * (PT_XBYTES + PT_WBYTES));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntn = grp.first[grp.count];                    // weight-row tiles over the group
  const int ntm = (M + 127) / 128;                         // token tiles
  const int total = ntn * ntm;
  const int ntl = blockIdx.x < total ? (total - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;   // tiles of this CTA
  const int nk = K / TC_BK, npt = nk / 2;                  // K steps and pairs per tile (nk even)
  const int npairs = ntl * npt;
  auto tile_of = [&](int lt, int& gi, int& n0, int& m0) {
    const int tt = (int)blockIdx.x + lt * (int)gridDim.x;
    const int ni = tt % ntn;
    gi = group_of(grp, ni);
    n0 = (ni - grp.first[gi]) * 128;
    m0 = (tt / ntn) * 128;
  };

  if (threadIdx.x == 0) {
    for (int q = 0; q < SP; ++q) {
      mbar_init(&bar_wfull[q], 1);
      mbar_init(&bar_xfull[q], 1);
      mbar_init(&bar_empty[q], 1 + 8);
    }
    for (int a = 0; a < ST; ++a) mbar_init(&bar_conv[a], 8);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar_accf[b], 1);
      mbar_init(&bar_acce[b], 4);
    }
    mbar_init(&bar_fin, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ weight producer
    if (lane == 0) {
      int issued = 0;
      for (int gj = 0; gj < npairs; ++gj) {
        const int lt = gj / npt, j = gj - lt * npt, q = gj % SP;
        int gi, n0, m0;
        tile_of(lt, gi, n0, m0);
        if (gj >= SP && !mbar_wait(&bar_empty[q], ((gj / SP) - 1) & 1, DEV_ERR_TIMEOUT_EMPTY)) break;
        mbar_arrive_expect_tx(&bar_wfull[q], 2u * PT_WBYTES);
        tma_load_3d(wsp(q), &maps.w[gi], &bar_wfull[q], 0, n0, 2 * j);
        issued = gj + 1;
      }
      for (int gj = issued - SP < 0 ? 0 : issued - SP; gj < issued; ++gj)
        mbar_wait(&bar_wfull[gj % SP], (gj / SP) & 1, DEV_ERR_TIMEOUT_FULL, false);
    }
  } else if (warp == TC_XWARP) {
    // ------------------------------------------------------------ activation producer
    if (lane == 0) {
      pdl_wait();                                  // the activations come from the previous kernel
      int issued = 0;
      for (int gj = 0; gj < npairs; ++gj) {
        const int lt = gj / npt, j = gj - lt * npt, q = gj % SP;
        int gi, n0, m0;
        tile_of(lt, gi, n0, m0);
        if (gj >= SP && !mbar_wait(&bar_empty[q], ((gj / SP) - 1) & 1, DEV_ERR_TIMEOUT_EMPTY)) break;
        mbar_arrive_expect_tx(&bar_xfull[q], 2u * PT_XBYTES);
        tma_load_3d(xs(2 * q), &tmX, &bar_xfull[q], 0, m0, 2 * j);
        issued = gj + 1;
      }
      for (int gj = issued - SP < 0 ? 0 : issued - SP; gj < issued; ++gj)
        mbar_wait(&bar_xfull[gj % SP], (gj / SP) & 1, DEV_ERR_TIMEOUT_FULL, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_i8(128, 128);
      bool ok = true;
      for (int lt = 0; lt < ntl && ok; ++lt) {
        const int b = lt & 1;
        // the epilogue has read this accumulator's previous tile
        if (lt >= 2 && !mbar_wait(&bar_acce[b], ((lt >> 1) - 1) & 1, DEV_ERR_TIMEOUT_ACC)) break;
        tc_fence_after();
        for (int i = 0; i < nk; ++i) {
          const int gs = lt * nk + i, st = gs % S, gj = gs >> 1, a = gs % ST;
          if (!mbar_wait(&bar_xfull[st >> 1], (gj / SP) & 1, DEV_ERR_TIMEOUT_FULL) ||
              !mbar_wait(&bar_conv[a], (gs / ST) & 1, DEV_ERR_TIMEOUT_A)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xaddr = smem_u32(xs(st));
#pragma unroll
          for (int kk = 0; kk < TC_BK / 32; ++kk)
            mma_i8_ts(tmem + 128u * b, tmem + 256u + 32u * a + 8u * kk, smem_desc_k_sw128(xaddr + kk * 32), IDESC,
                      (i > 0 || kk > 0) ? 1u : 0u);
          // a pair stage is released after its second step's MMAs, if it is refilled
          if ((st & 1) && gj + SP < npairs) mma_commit(&bar_empty[st >> 1]);
        }
        if (ok) mma_commit(&bar_accf[b]);
      }
      mma_commit(&bar_fin);
      mbar_wait(&bar_fin, 0, DEV_ERR_TIMEOUT_ACC, false);   // no MMA in flight at teardown
    }
  } else if (warp < PT_EPI_WARP0) {
    // ------------------------------------------------------------ converters
    const int q4 = warp & 3;                      // tensor-memory lane quarter
    const int h = (warp - 2) >> 2;                // which half of the K bytes of a step
    const int row = 32 * q4 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    for (int gs = 0; gs < ntl * nk; ++gs) {
      const int st = gs % S, gj = gs >> 1, a = gs % ST, c = st & 1;
      if (!mbar_wait_warp(&bar_wfull[st >> 1], (gj / SP) & 1, DEV_ERR_TIMEOUT_FULL)) break;
      tc_fence_after();
      const uint4 w = *reinterpret_cast<const uint4*>(wsp(st >> 1) + c * PT_WBYTES + 32 * row +
                                                      16 * (h ^ ((row >> 2) & 1)));
      __syncwarp();
      if (lane == 0 && c == 1) mbar_arrive(&bar_empty[st >> 1]);   // the pair's packed tiles consumed
      const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
      uint32_t av[16];
#pragma unroll
      for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) av[4 * g + jj] = unpack4(wv[g], jj);
      tmem_st16(lane_base + (uint32_t)(256 + 32 * a + 16 * h), av);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_conv[a]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;
    const int row = 32 * q4 + lane;               // output feature inside the tile
    const int et = threadIdx.x - 32 * PT_EPI_WARP0;   // 0..127
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    const bool small_acc = (int64_t)127 * K < (int64_t)(1 << 22);
    pdl_wait();                                   // s_x comes from the previous kernel
    for (int lt = 0; lt < ntl; ++lt) {
      int gi, n0, m0;
      tile_of(lt, gi, n0, m0);
      const int N = grp.N[gi];
      TOut* __restrict__ Y = static_cast<TOut*>(grp.Y[gi]);
      int32_t* __restrict__ acc_dbg = grp.acc_dbg[gi];
      // the previous tile's staged outputs have been read by its store, and its scales are no longer used
      asm volatile("bar.sync 3, 128;" ::: "memory");
      {
        const int m = m0 + et;
        sdq[et] = m < M ? dequant_scale(ldg_f32(s_x + m), ldg_nc_f32(grp.s_w[gi])) : 0.f;
      }
      const int b = lt & 1;
      const bool ok = mbar_wait_warp(&bar_accf[b], (lt >> 1) & 1, DEV_ERR_TIMEOUT_ACC);
      tc_fence_after();
      asm volatile("bar.sync 3, 128;" ::: "memory");     // the tile's scales are in place
      const int n = n0 + row;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[2][16];
        load_cols<16, 2>(lane_base + (uint32_t)(128 * b + c0), v);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const int cc = c0 + 16 * g;
          float sq[16];
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const float4 f = *reinterpret_cast<const float4*>(sdq + cc + 4 * k4);
            sq[4 * k4] = f.x; sq[4 * k4 + 1] = f.y; sq[4 * k4 + 2] = f.z; sq[4 * k4 + 3] = f.w;
          }
          if (use_tma_store) {
            TOut* dst = ostage + (size_t)cc * 128 + row;
            if (small_acc) {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj)
                stage_out(dst + jj * 128, __fmul_rn(small_int_to_float((int)v[g][jj] >> 6), sq[jj]));
            } else {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) stage_out(dst + jj * 128, __fmul_rn((float)((int)v[g][jj] >> 6), sq[jj]));
            }
          } else if (ok && n < N) {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int m = m0 + cc + jj;
              if (m < M) {
                const int acc = (int)v[g][jj] >> 6;
                if (acc_dbg) acc_dbg[(size_t)m * N + n] = acc;
                store_out(Y + (size_t)m * N + n, __fmul_rn((float)acc, sq[jj]));
              }
            }
          }
        }
      }
      // every read of this accumulator is done: the MMAs of tile lt + 2 may use it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_acce[b]);
      if (use_tma_store) {
        fence_proxy_async_smem();
        asm volatile("bar.sync 3, 128;" ::: "memory");
        if (et == 0 && ok) {
          tma_store_2d(&maps.y[gi], ostage, n0, m0);
          bulk_wait_read();                        // the staging is reused by the next tile
        }
      }
      // no early exit: the four warps take the same barriers whatever their waits returned
      // (after a give-up every later wait returns at once)
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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

static bool make_map_2d(CUtensorMap* map, const void* ptr, CUtensorMapDataType dt, uint64_t inner, uint64_t rows,
                        uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Bytes [K steps][rows][step bytes] of a row-major [rows][row_bytes] matrix:
// dimension 0 = the step_bytes of one K step, 1 = rows (stride row_bytes),
// 2 = K steps (stride step_bytes); a box of `steps` K steps lands as
// consecutive [box_rows][step_bytes] tiles.
static bool make_map_steps(CUtensorMap* map, const void* ptr, uint64_t row_bytes, uint64_t rows, uint32_t step_bytes,
                           uint32_t box_rows, uint32_t steps, CUtensorMapSwizzle sw) {
  EncodeFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {step_bytes, rows, row_bytes / step_bytes};
  cuuint64_t strides[2] = {row_bytes, step_bytes};
  cuuint32_t box[3] = {step_bytes, box_rows, steps};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T> struct MapType;
template <> struct MapType<float> { static constexpr CUtensorMapDataType v = CU_TENSOR_MAP_DATA_TYPE_FLOAT32; };
template <> struct MapType<__nv_bfloat16> { static constexpr CUtensorMapDataType v = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16; };

template <int BN, int ACT_BITS, typename TOut, int MB>
static cudaError_t launch_tc(LinGroup grp, const void* Xq, const float* s_x, int M, int K, cudaStream_t st) {
  using C = TcCfg<BN, ACT_BITS, MB>;
  TcMaps maps;                                     // copied into the launch's parameters
  CUtensorMap tmX;
  const bool ok = ACT_BITS == 8
      ? make_map_steps(&tmX, Xq, (uint64_t)K, (uint64_t)M, TC_BK, BN, C::P, CU_TENSOR_MAP_SWIZZLE_128B)
      : make_map_steps(&tmX, Xq, (uint64_t)K / 2, (uint64_t)M, TC_BK / 2, BN, C::P, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
  // The output leaves through one TMA store per tile when rows are 16-byte
  // multiples; the diagnostics accumulators take the per-element path.
  int use_tma_store = 1;
  for (int g = 0; g < grp.count; ++g)
    if (grp.acc_dbg[g] != nullptr || ((uint64_t)grp.N[g] * sizeof(TOut)) % 16 != 0) use_tma_store = 0;
  grp.first[0] = 0;
  for (int g = 0; g < grp.count; ++g) {
    if (!make_map_steps(&maps.w[g], grp.pkW[g], (uint64_t)K / 4, (uint64_t)grp.N[g], TC_BK / 4, 128, C::P,
                        CU_TENSOR_MAP_SWIZZLE_32B))
      return cudaErrorInvalidValue;
    if (use_tma_store && !make_map_2d(&maps.y[g], grp.Y[g], MapType<TOut>::v, (uint64_t)grp.N[g], (uint64_t)M,
                                      (uint64_t)grp.N[g] * sizeof(TOut), 128, BN, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    if (!use_tma_store) maps.y[g] = tmX;           // unused
    grp.first[g + 1] = grp.first[g] + (grp.N[g] + MB - 1) / MB;
  }
  for (int g = grp.count; g < GROUP_MAX; ++g) {
    maps.w[g] = maps.w[0];
    maps.y[g] = maps.y[0];
    grp.first[g + 1] = grp.first[grp.count];
  }
  // Split K across a cluster when the output tiles alone leave most SMs idle
  // (decode): each rank streams a K range, partial sums meet in the leader.
  const int ntiles = grp.first[grp.count];
  const int tiles = ntiles * ((M + BN - 1) / BN);
  const int nk = K / TC_BK;
  // With 64 or 128 tokens per tile the partial tiles (32 or 64 KB) take shared
  // memory, so a split tile holds an SM alone; it pays when the tiles would
  // otherwise leave SMs idle (the N = 2048 layers of a 512-token batch), and a
  // CTA alone on its SM also gets the SM's whole load bandwidth.
  int ksplit = 1;
  if (MB == 128) {
    int sms = 148, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int kmax = BN <= 32 ? 8 : BN == 64 ? 4 : 2;
    const int per_sm = BN <= 32 ? 2 : 1;
    while (ksplit < kmax && tiles * ksplit * 2 <= per_sm * sms && ksplit * 2 <= nk) ksplit *= 2;
  }
  size_t smem = C::SMEM + (size_t)(ksplit - 1) * 128 * BN * sizeof(int32_t);
  // Never more CTAs per SM than tensor memory can serve at once (512 columns):
  // a CTA blocked in tcgen05.alloc behind cluster peers waiting at the cluster
  // barrier would never run.  Shared memory (228 KB per SM) enforces the bound.
  const size_t min_smem = (size_t)(228 * 1024) / (512 / C::TMEM_COLS + 1) + 1024;
  if (smem < min_smem) smem = min_smem;
  auto kern = linear_tc_kernel<BN, ACT_BITS, TOut, MB>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  dim3 grid(ntiles, (M + BN - 1) / BN, ksplit);
  return launch_pdl(kern, grid, dim3(TC_THREADS), smem, st, dim3(1, 1, ksplit), maps, tmX, grp, use_tma_store,
                    s_x, M, K, ksplit);
}

// The persistent int8 kernel (128 x 128 tiles, one CTA per SM over all tiles).
template <typename TOut>
static cudaError_t launch_tc_persistent(LinGroup grp, const void* Xq, const float* s_x, int M, int K,
                                        cudaStream_t st) {
  TcMaps maps;
  CUtensorMap tmX;
  if (!make_map_steps(&tmX, Xq, (uint64_t)K, (uint64_t)M, TC_BK, 128, 2, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int use_tma_store = 1;
  for (int g = 0; g < grp.count; ++g)
    if (grp.acc_dbg[g] != nullptr || ((uint64_t)grp.N[g] * sizeof(TOut)) % 16 != 0) use_tma_store = 0;
  grp.first[0] = 0;
  for (int g = 0; g < grp.count; ++g) {
    if (!make_map_steps(&maps.w[g], grp.pkW[g], (uint64_t)K / 4, (uint64_t)grp.N[g], TC_BK / 4, 128, 2,
                        CU_TENSOR_MAP_SWIZZLE_32B))
      return cudaErrorInvalidValue;
    if (use_tma_store && !make_map_2d(&maps.y[g], grp.Y[g], MapType<TOut>::v, (uint64_t)grp.N[g], (uint64_t)M,
                                      (uint64_t)grp.N[g] * sizeof(TOut), 128, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    if (!use_tma_store) maps.y[g] = tmX;           // unused
    grp.first[g + 1] = grp.first[g] + (grp.N[g] + 127) / 128;
  }
  for (int g = grp.count; g < GROUP_MAX; ++g) {
    maps.w[g] = maps.w[0];
    maps.y[g] = maps.y[0];
    grp.first[g + 1] = grp.first[grp.count];
  }
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int total = grp.first[grp.count] * ((M + 127) / 128);
  const int grid = total < sms ? total : sms;
  if (grid == 0) return cudaSuccess;
  const size_t smem = pt_smem_bytes<TOut>();
  auto kern = linear_tc_persistent_kernel<TOut>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3((unsigned)grid), dim3(PT_THREADS), smem, st, 1u, maps, tmX, grp, use_tma_store, s_x,
                    M, K);
}

// rows: 0 = choose the weight rows per CTA, 128 or 256 = that tile.
template <int ACT_BITS, typename TOut>
static cudaError_t dispatch_tc(const LinGroup& grp, const void* Xq, const float* s_x, int M, int K, int rows,
                               cudaStream_t st) {
  if (rows == 256) return launch_tc<128, ACT_BITS, TOut, 256>(grp, Xq, s_x, M, K, st);
  if (rows == -1) {                   // the persistent kernel, asked for (int8, > 64 tokens, even K steps)
    if constexpr (ACT_BITS == 8) return launch_tc_persistent<TOut>(grp, Xq, s_x, M, K, st);
    return cudaErrorInvalidValue;
  }
  if (M <= 16) return launch_tc<16, ACT_BITS, TOut, 128>(grp, Xq, s_x, M, K, st);
  if (M <= 32) return launch_tc<32, ACT_BITS, TOut, 128>(grp, Xq, s_x, M, K, st);
  if (M <= 64) return launch_tc<64, ACT_BITS, TOut, 128>(grp, Xq, s_x, M, K, st);
  // 256 weight rows per CTA halve the activation bytes per MMA but hold a
  // whole SM.  Measured on B200 it runs the batched prefill product slower
  // than the 128-row tile at two CTAs per SM (about 1250 cycles per K step
  // against 512 of MMA work, with the activation tiles landing only every
  // ~1250 cycles), so it is used only when asked for (kernel 4).
  // The persistent kernel (kernel 5) hides each tile's start and epilogue
  // behind the next tile's K loop, but at one CTA per SM its K steps come no
  // faster than one CTA's of this kernel: measured on B200 it runs the batched
  // prefill product in 242 us (6 or 8 stages) against 205 us here, so it is
  // not chosen automatically.
  return launch_tc<128, ACT_BITS, TOut, 128>(grp, Xq, s_x, M, K, st);
}

template <int ACT_BITS, typename TOut>
static cudaError_t launch_simt(const void* Xq, const float* s_x, const uint8_t* pkW, const float* s_w,
                               int M, int N, int K, void* Y, int32_t* acc_dbg, cudaStream_t st) {
  dim3 grid((N + 7) / 8, (M + 15) / 16);
  return launch_pdl(linear_simt_kernel<ACT_BITS, TOut>, grid, dim3(256), 0, st, 1u,
                    static_cast<const uint8_t*>(Xq), s_x, reinterpret_cast<const uint32_t*>(pkW), s_w, M, N, K,
                    static_cast<TOut*>(Y), acc_dbg);
}

bool tensor_map_encoder_available() { return get_encode() != nullptr; }

bool decode_path_applies(int M, int K);
cudaError_t run_linear_decode(const void* Xq, int act_bits, const float* s_x, const uint8_t* pkW, const float* s_w,
                              int M, int N, int K, void* Y, int y_bf16, int32_t* acc_dbg, cudaStream_t st);
cudaError_t run_linear_decode_group(const LinGroup& grp, const void* Xq, int act_bits, const float* s_x, int M, int K,
                                    int y_bf16, cudaStream_t st);

cudaError_t run_linear_group(const LinGroup& grp, const void* Xq, int act_bits, const float* s_x, int M, int K,
                             int y_bf16, int path, cudaStream_t st);

// path: 0 = automatic, 1 = SIMT, 2 = tcgen05, 3 = warp-MMA decode kernel, 4 = tcgen05 with
// 256 weight rows per CTA, 5 = persistent tcgen05 (int8)
cudaError_t run_linear(const void* Xq, int act_bits, const float* s_x, const uint8_t* pkW, const float* s_w,
                       int M, int N, int K, void* Y, int y_bf16, int32_t* acc_dbg, int path, cudaStream_t st) {
  // up to 32 tokens: one pass over the weights with warp-level MMA
  if ((path == 0 || path == 3) && decode_path_applies(M, K))
    return run_linear_decode(Xq, act_bits, s_x, pkW, s_w, M, N, K, Y, y_bf16, acc_dbg, st);
  if (path == 3) return cudaErrorInvalidValue;
  if (path == 1) {                    // the dp4a kernel is a diagnostics path (slower at every M)
#define BN_LIN(BITS, T) return launch_simt<BITS, T>(Xq, s_x, pkW, s_w, M, N, K, Y, acc_dbg, st)
    if (act_bits == 8) {
      if (y_bf16) { BN_LIN(8, __nv_bfloat16); } else { BN_LIN(8, float); }
    } else {
      if (y_bf16) { BN_LIN(4, __nv_bfloat16); } else { BN_LIN(4, float); }
    }
#undef BN_LIN
  }
  LinGroup grp = {};
  grp.pkW[0] = pkW;
  grp.s_w[0] = s_w;
  grp.Y[0] = Y;
  grp.acc_dbg[0] = acc_dbg;
  grp.N[0] = N;
  grp.count = 1;
  return run_linear_group(grp, Xq, act_bits, s_x, M, K, y_bf16, path, st);
}

// Several weight matrices sharing Xq and s_x in one launch.  path: 0 = automatic,
// 2 = tcgen05 with 128 weight rows per CTA, 3 = warp-MMA decode kernel, 4 =
// tcgen05 with 256 weight rows per CTA.
cudaError_t run_linear_group(const LinGroup& grp, const void* Xq, int act_bits, const float* s_x, int M, int K,
                             int y_bf16, int path, cudaStream_t st) {
  if ((path == 0 || path == 3) && decode_path_applies(M, K))
    return run_linear_decode_group(grp, Xq, act_bits, s_x, M, K, y_bf16, st);
  if (path == 3) return cudaErrorInvalidValue;
  const int rows = path == 2 ? 128 : path == 4 ? 256 : path == 5 ? -1 : 0;
  if (act_bits == 8) {
    return y_bf16 ? dispatch_tc<8, __nv_bfloat16>(grp, Xq, s_x, M, K, rows, st)
                  : dispatch_tc<8, float>(grp, Xq, s_x, M, K, rows, st);
  }
  return y_bf16 ? dispatch_tc<4, __nv_bfloat16>(grp, Xq, s_x, M, K, rows, st)
                : dispatch_tc<4, float>(grp, Xq, s_x, M, K, rows, st);
}

}  // namespace bitnet
