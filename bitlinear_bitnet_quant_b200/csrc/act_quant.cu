// Activation quantisers of the BitLinear forward.
//
//  * quant_act_i8: RMSNorm, then per-token absmax int8 ("LLM을 1.58비트로
//    파인튜닝: BitNet을 이용한 극단적인 양자화", section 양자화 메커니즘:
//    absmax per token into [-128, 127], layer norm before the quantiser).
//  * hadamard_quant_i4: RMSNorm, Walsh-Hadamard transform, per-token absmax
//    int4 ("초저용량 LLM의 진화: BitNet v2 파헤치기", section 방법론: the
//    H-BitLinear layer applies a Hadamard transform before 4-bit quantisation).
//
// Fixed arithmetic (fp32, round-to-nearest-even, no contraction):
//   ss = sum of x*x by the balanced pairwise tree over element indices
//        (zero padded to a power of two)
//   r  = 1 / sqrt(ss / K + eps);  y = (x * r) * gamma
//   s  = qmax / max(max|y|, 1e-5);  q = clamp(rint(y * s), qmin, qmax)
// Hadamard: Sylvester order per block of b = 2^L elements, radix-2 stages of
// stride 1, 2, ..., b/2 (pair (a, c) -> (a + c, a - c)), then times
// c_b = fp32(1/sqrt(b)).  Codes are then taken from t with qmax = 7.
#include "quant_common.cuh"

namespace bitnet {

// Element-wise prologues of the stacked layer, applied to each fp32 input
// chunk before the quantiser sees it (bit-identical to running bitnet_add or
// bitnet_relu2_glu first):
//   PRE_ADD: x = a + b, and x is written out (the residual stream);
//   PRE_GLU: x = (r * r) * up with r = max(gate, 0).
enum Prologue : int { PRE_NONE = 0, PRE_ADD = 1, PRE_GLU = 2 };

template <int PRE, typename TIn, int E>
BN_DEV void load_chunk(const TIn* x, const float* b, float* h, float (&v)[E]) {
  InVec<TIn>::load(x, v);
  if constexpr (PRE == PRE_ADD || PRE == PRE_GLU) {
    static_assert(sizeof(TIn) == 4, "prologues take fp32 inputs");
    float u[E];
    InVec<float>::load(b, u);
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = PRE == PRE_ADD ? __fadd_rn(v[e], u[e]) : relu2_times(v[e], u[e]);
    if constexpr (PRE == PRE_ADD)
      *reinterpret_cast<float4*>(h) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

// ---------------------------------------------------------------------------
// RMSNorm + int8: one CTA of NT threads per token.  Chunk j (16 bytes of
// input: E elements) goes to thread j % NT in iteration j / NT, so the loads
// are coalesced; the pairwise tree is then: E elements inside a chunk, the
// NT threads (warp xor-shuffles, then warps in order), the IT iterations.
// ---------------------------------------------------------------------------
template <typename TIn, int NT, int IT, int PRE>
__global__ void __launch_bounds__(NT)
quant_act_i8_kernel(const TIn* __restrict__ X, const float* __restrict__ B, float* __restrict__ H, int K,
                    const float* __restrict__ gamma, float eps, int8_t* __restrict__ Xq, float* __restrict__ s_x) {
  constexpr int E = InVec<TIn>::E;
  constexpr int NW = NT / 32;
  __shared__ float red[IT][NW];
  __shared__ float wmax[NW];

  pdl_launch_dependents();
  pdl_wait();                                // X may come from, and Xq may still be read by, the previous kernel
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int m = blockIdx.x;
  const int C = K / E;                       // chunks in the row
  const TIn* xrow = X + (size_t)m * K;

  float v[IT][E];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int j = it * NT + tid;
    if (j < C) {
      const size_t off = (size_t)m * K + (size_t)j * E;
      load_chunk<PRE, TIn, E>(xrow + (size_t)j * E, B + off, H + off, v[it]);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) v[it][e] = 0.f;
    }
  }

  // ---- sum of squares, pairwise over element indices ----
  float cs[IT];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    float sq[E];
#pragma unroll
    for (int e = 0; e < E; ++e) sq[e] = __fmul_rn(v[it][e], v[it][e]);
    const float w = warp_tree_sum(tree_sum<E>(sq));
    if (lane == 0) red[it][warp] = w;
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    float p[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) p[w] = red[it][w];
    cs[it] = tree_sum<NW>(p);
  }
  const float ss = tree_sum<IT>(cs);

  const float ms = __fdiv_rn(ss, (float)K);
  const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));

  // ---- normalise, absmax ----
  float amax = 0.f;
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int j = it * NT + tid;
    if (gamma != nullptr && j < C) {
      float g[4 * ((E + 3) / 4)];
#pragma unroll
      for (int q = 0; q < E / 4; ++q) {
        uint4 u = ldg_nc_v4(gamma + (size_t)j * E + 4 * q);
        g[4 * q] = __uint_as_float(u.x); g[4 * q + 1] = __uint_as_float(u.y);
        g[4 * q + 2] = __uint_as_float(u.z); g[4 * q + 3] = __uint_as_float(u.w);
      }
#pragma unroll
      for (int e = 0; e < E; ++e) v[it][e] = __fmul_rn(__fmul_rn(v[it][e], r), g[e]);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) v[it][e] = __fmul_rn(v[it][e], r);
    }
#pragma unroll
    for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(v[it][e]));
  }
  amax = warp_max(amax);
  if (lane == 0) wmax[warp] = amax;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < NW; ++w) amax = fmaxf(amax, wmax[w]);

  const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));

  // ---- codes: rint(y * s), clamped to [-128, 127] ----
  // With s = 127 / max(amax, 1e-5) and |y| <= amax, |y * s| <= 127 (1 + 2^-23)
  // after both roundings, so every code lies in [-127, 127] and the clamp never
  // acts; the rounded products go through rint_low_bits.
  int8_t* qrow = Xq + (size_t)m * K;
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int j = it * NT + tid;
    if (j >= C) continue;
    uint32_t packed[E / 4];
#pragma unroll
    for (int q = 0; q < E / 4; ++q) {
      uint32_t b[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) b[e] = rint_low_bits(__fmul_rn(v[it][4 * q + e], s));
      packed[q] = pack_low_bytes(b[0], b[1], b[2], b[3]);
    }
    if constexpr (E == 8) {
      *reinterpret_cast<uint2*>(qrow + (size_t)j * E) = make_uint2(packed[0], packed[1]);
    } else {
      *reinterpret_cast<uint32_t*>(qrow + (size_t)j * E) = packed[0];
    }
  }
  if (tid == 0) s_x[m] = s;
}

// ---------------------------------------------------------------------------
// RMSNorm + Hadamard + int4.  Each thread owns 128 consecutive elements of a
// token (G = K/128 threads per token, rounded up to a power of two GP; TPB
// tokens per CTA).  Stages of stride < 128 run in registers; the stages of
// stride 128 .. b/2 run after one transpose through shared memory, in which
// a thread holds the elements whose index bits [a, 7) and the block index are
// fixed (a = 14 - L), i.e. in-thread bits [0, a) and [7, L).  Bit 0 stays in
// the thread, so codes are packed two per byte there; the packed bytes (not
// the fp32 values) go back through shared memory for coalesced stores.
// ---------------------------------------------------------------------------
constexpr int HT_R = 128;                          // elements per thread

// fp32 slot of element e: two pad words per 128 keep 8-byte accesses of both
// the transpose's writers and readers free of bank conflicts
BN_DEV int hpidx(int e) { return e + 2 * (e >> 7); }

// In-register radix-2 stages s = S0 .. S1-1 over v[c], where in-thread index
// bit (s - SHIFT) is the element-index bit s.
template <int S0, int S1, int SHIFT>
BN_DEV void fwht_reg(float (&v)[HT_R]) {
#pragma unroll
  for (int s = S0; s < S1; ++s) {
    const int h = 1 << (s - SHIFT);
#pragma unroll
    for (int c = 0; c < HT_R; ++c) {
      if ((c & h) == 0) {
        const float a = v[c], b = v[c + h];
        v[c] = __fadd_rn(a, b);
        v[c + h] = __fsub_rn(a, b);
      }
    }
  }
}

// Phase-2 in-thread index c -> element index inside the token row.
template <int L>
BN_DEV int phase2_elem(int tprime, int c) {
  constexpr int A = 14 - L;                        // low in-thread bits
  constexpr int MIDB = L - 7;                      // thread bits inside a block
  const int blk = tprime >> MIDB;
  const int mid = tprime & ((1 << MIDB) - 1);
  const int within = ((c >> A) << 7) | (mid << A) | (c & ((1 << A) - 1));
  return (blk << L) | within;
}

// Code of t: rint(t * s) clamped to [-8, 7], in the low nibble.  With
// s = 7 / max(amax, 1e-5) and |t| <= amax, |t * s| <= 7 (1 + 2^-23) after both
// roundings, so the code lies in [-7, 7] and the clamp never acts.
BN_DEV uint32_t nib(float t, float s) { return rint_low_bits(__fmul_rn(t, s)); }

// Eight codes (element 0 in the low nibble) as one word.
BN_DEV uint32_t pack_nibbles8(const float* t, float s) {
  return pack_low_bytes(pair_nibbles(nib(t[0], s), nib(t[1], s)), pair_nibbles(nib(t[2], s), nib(t[3], s)),
                        pair_nibbles(nib(t[4], s), nib(t[5], s)), pair_nibbles(nib(t[6], s), nib(t[7], s)));
}

template <typename TIn, int L, int PRE>
__global__ void __launch_bounds__(128, 3)
hadamard_quant_i4_kernel(const TIn* __restrict__ X, const float* __restrict__ B, int M, int K, int GP,
                         const float* __restrict__ gamma, float eps, float cb,
                         uint8_t* __restrict__ Xq4, float* __restrict__ s_x,
                         float* __restrict__ T_dbg) {
  extern __shared__ float hsm[];
  pdl_launch_dependents();
  pdl_wait();                                // X may come from, and Xq4 may still be read by, the previous kernel
  const int G = K / HT_R;
  const int TPB = blockDim.x / GP;
  const int g = threadIdx.x / GP;                  // token slot in the CTA
  const int t = threadIdx.x % GP;                  // thread inside the token
  const int lane = threadIdx.x & 31;
  const int m = blockIdx.x * TPB + g;
  const bool active = (m < M) && (t < G);
  const int rowpad = (K + 2 * (K >> 7) + 3) & ~3;   // 16-byte aligned token rows
  float* tok = hsm + (size_t)g * rowpad;
  float* red = hsm + (size_t)TPB * rowpad;         // [TPB][4] partials
  uint8_t* bytes = reinterpret_cast<uint8_t*>(tok);  // packed codes, K/2 bytes (after the transpose)

  float v[HT_R];
  if (active) {
    const size_t off = (size_t)m * K + (size_t)t * HT_R;
    const TIn* src = X + off;
    constexpr int E = InVec<TIn>::E;
#pragma unroll
    for (int q = 0; q < HT_R / E; ++q) {
      float tmp[E];
      load_chunk<PRE, TIn, E>(src + q * E, B + off + q * E, nullptr, tmp);
#pragma unroll
      for (int e = 0; e < E; ++e) v[q * E + e] = tmp[e];
    }
  } else {
#pragma unroll
    for (int c = 0; c < HT_R; ++c) v[c] = 0.f;
  }

  // ---- sum of squares: in-thread subtree of 128 (first level fused), then threads in order ----
  float part;
  {
    float sq[HT_R / 2];
#pragma unroll
    for (int c = 0; c < HT_R / 2; ++c)
      sq[c] = __fadd_rn(__fmul_rn(v[2 * c], v[2 * c]), __fmul_rn(v[2 * c + 1], v[2 * c + 1]));
    part = tree_sum<HT_R / 2>(sq);
  }
  const int wl = GP < 32 ? GP : 32;                // lanes of one token inside a warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1)
    if (o < wl) part = __fadd_rn(part, __shfl_xor_sync(0xffffffffu, part, o));
  float ss = part;
  if (GP > 32) {                                   // 2 or 4 warps per token
    if (lane == 0) red[g * 4 + (t >> 5)] = part;
    __syncthreads();
    float p[4] = {red[g * 4], red[g * 4 + 1], 0.f, 0.f};
    if (GP == 64) {
      ss = __fadd_rn(p[0], p[1]);
    } else {
      p[2] = red[g * 4 + 2]; p[3] = red[g * 4 + 3];
      ss = __fadd_rn(__fadd_rn(p[0], p[1]), __fadd_rn(p[2], p[3]));
    }
  }
  const float ms = __fdiv_rn(ss, (float)K);
  const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
  if (active) {
    if (gamma != nullptr) {
      const float* gp = gamma + (size_t)t * HT_R;
#pragma unroll
      for (int c = 0; c < HT_R; ++c) v[c] = __fmul_rn(__fmul_rn(v[c], r), __ldg(gp + c));
    } else {
#pragma unroll
      for (int c = 0; c < HT_R; ++c) v[c] = __fmul_rn(v[c], r);
    }
  }

  // ---- Hadamard stages of stride 1 .. min(b, 128)/2 in registers ----
  constexpr int P1 = L < 7 ? L : 7;
  fwht_reg<0, P1, 0>(v);

  if constexpr (L > 7) {
    __syncthreads();                                // red[] reads above are done
    if (active) {
#pragma unroll
      for (int c = 0; c < HT_R; c += 2)
        *reinterpret_cast<float2*>(tok + hpidx(t * HT_R + c)) = make_float2(v[c], v[c + 1]);
    }
    __syncthreads();
    if (active) {
#pragma unroll
      for (int c = 0; c < HT_R; c += 2) {          // bit 0 of c is bit 0 of the element: pairs are adjacent
        const float2 p = *reinterpret_cast<const float2*>(tok + hpidx(phase2_elem<L>(t, c)));
        v[c] = p.x;
        v[c + 1] = p.y;
      }
    }
    fwht_reg<7, L, 7 - (14 - L)>(v);
  }

  // ---- normalise, absmax over the token ----
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < HT_R; ++c) {
    v[c] = __fmul_rn(v[c], cb);
    amax = fmaxf(amax, fabsf(v[c]));
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1)
    if (o < wl) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (GP > 32) {
    __syncthreads();
    if (lane == 0) red[g * 4 + (t >> 5)] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(red[g * 4], red[g * 4 + 1]),
                 GP == 128 ? fmaxf(red[g * 4 + 2], red[g * 4 + 3]) : 0.f);
  }
  const float s = __fdiv_rn(7.0f, fmaxf(amax, 1e-5f));

  if constexpr (L <= 7) {
    // the thread's 128 elements are consecutive: 64 bytes straight out
    if (!active) return;
    if (T_dbg != nullptr) {
      float* dst = T_dbg + (size_t)m * K + (size_t)t * HT_R;
#pragma unroll
      for (int c = 0; c < HT_R; c += 4)
        *reinterpret_cast<float4*>(dst + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
    }
    uint32_t w[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) w[q] = pack_nibbles8(v + 8 * q, s);
    uint4* dst = reinterpret_cast<uint4*>(Xq4 + (size_t)m * (K / 2) + (size_t)t * (HT_R / 2));
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
    if (t == 0) s_x[m] = s;
  } else {
    // codes two per byte in the phase-2 mapping, staged as bytes, then coalesced stores
    __syncthreads();                                // every thread has read its transposed values
    if (active) {
      if (T_dbg != nullptr) {
        float* dst = T_dbg + (size_t)m * K;
#pragma unroll
        for (int c = 0; c < HT_R; ++c) dst[phase2_elem<L>(t, c)] = v[c];
      }
#pragma unroll
      for (int c = 0; c < HT_R; c += 2)
        bytes[phase2_elem<L>(t, c) >> 1] = (uint8_t)pair_nibbles(nib(v[c], s), nib(v[c + 1], s));
    }
    __syncthreads();
    if (m < M) {
      const uint4* src = reinterpret_cast<const uint4*>(bytes);
      uint4* dst = reinterpret_cast<uint4*>(Xq4 + (size_t)m * (K / 2));
      for (int q = t; q < K / 32; q += GP) dst[q] = src[q];
      if (t == 0) s_x[m] = s;
    }
  }
}

// ---------------------------------------------------------------------------
// RMSNorm + Hadamard + int4 for a few tokens: one CTA of 256 threads per token.
// The sum of squares uses the fixed tree (E elements of a chunk, 32 lanes, the
// 8 warps in order, then the iterations, padded with zero subtrees).  The row
// is kept in shared memory; the radix-2 stages (stride 1, 2, ..., b/2, pairs
// (a, c) -> (a + c, a - c)) run three at a time: a thread takes 8 elements at
// stride 2^st, applies stages st, st+1, st+2 in registers in that order and
// writes them back, one barrier per pass.  Every value is the one the register
// kernel produces.  The first pass also applies the norm, the last one c_b
// and the absmax.
// ---------------------------------------------------------------------------
constexpr int HR_THREADS = 256;
constexpr int HR_MAX_IT = 16;                        // K <= 16384 (fp32: 4 elements per chunk)

// Shared-memory slot of element i: one pad word per 8 keeps every pass's
// accesses (8 elements at stride 1, 8, 64, ...) free of bank conflicts.
BN_DEV int hr_pidx(int i) { return i + (i >> 3); }

// Stages st .. st+P-1 over groups of 2^P elements; returns this thread's absmax
// of the results when LAST (after the factor cb).
template <int P, bool FIRST, bool LAST>
BN_DEV float hr_pass(float* hrow, int K, int st, float r, const float* __restrict__ gamma, float cb) {
  constexpr int G = 1 << P;
  const int h = 1 << st;
  float amax = 0.f;
  for (int q = threadIdx.x; q < K / G; q += HR_THREADS) {
    const int i0 = ((q >> st) << (st + P)) | (q & (h - 1));
    float v[G];
#pragma unroll
    for (int k = 0; k < G; ++k) v[k] = hrow[hr_pidx(i0 + k * h)];
    if constexpr (FIRST) {
#pragma unroll
      for (int k = 0; k < G; ++k)
        v[k] = gamma != nullptr ? __fmul_rn(__fmul_rn(v[k], r), __ldg(gamma + i0 + k * h)) : __fmul_rn(v[k], r);
    }
#pragma unroll
    for (int sg = 0; sg < P; ++sg) {
      const int d = 1 << sg;
#pragma unroll
      for (int k = 0; k < G; ++k) {
        if ((k & d) == 0) {
          const float a = v[k], c = v[k + d];
          v[k] = __fadd_rn(a, c);
          v[k + d] = __fsub_rn(a, c);
        }
      }
    }
    if constexpr (LAST) {
#pragma unroll
      for (int k = 0; k < G; ++k) {
        v[k] = __fmul_rn(v[k], cb);
        amax = fmaxf(amax, fabsf(v[k]));
      }
    }
#pragma unroll
    for (int k = 0; k < G; ++k) hrow[hr_pidx(i0 + k * h)] = v[k];
  }
  return amax;
}

template <typename TIn, int L, int PRE>
__global__ void __launch_bounds__(HR_THREADS)
hadamard_quant_i4_row_kernel(const TIn* __restrict__ X, const float* __restrict__ B, int K,
                             const float* __restrict__ gamma, float eps, float cb, uint8_t* __restrict__ Xq4,
                             float* __restrict__ s_x, float* __restrict__ T_dbg) {
  static_assert(L >= 4, "the first pass takes three stages, the last at least one");
  constexpr int E = InVec<TIn>::E, NW = HR_THREADS / 32;
  extern __shared__ float hrow[];                    // K + K/8 floats (hr_pidx)
  __shared__ float red[HR_MAX_IT][NW];
  pdl_launch_dependents();
  pdl_wait();                                        // X may come from, and Xq4 may still be read by, the previous kernel
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int m = blockIdx.x;
  const int C = K / E;
  int P = 1;
  while (P < C) P <<= 1;
  const int IT = P > HR_THREADS ? P / HR_THREADS : 1;  // iterations covering the padded row

  // ---- load (with the prologue), squares by the fixed tree ----
  for (int it = 0; it < IT; ++it) {
    const int j = it * HR_THREADS + tid;
    float v[E];
    if (j < C) {
      const size_t off = (size_t)m * K + (size_t)j * E;
      load_chunk<PRE, TIn, E>(X + off, B + off, nullptr, v);
#pragma unroll
      for (int e = 0; e < E; ++e) hrow[hr_pidx(j * E + e)] = v[e];
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = 0.f;
    }
    float sq[E];
#pragma unroll
    for (int e = 0; e < E; ++e) sq[e] = __fmul_rn(v[e], v[e]);
    const float w = warp_tree_sum(tree_sum<E>(sq));
    if (lane == 0) red[it][warp] = w;
  }
  __syncthreads();
  // every thread forms the same tree from the partials
  float cs[HR_MAX_IT];
#pragma unroll
  for (int it = 0; it < HR_MAX_IT; ++it) {
    cs[it] = 0.f;                                    // past the padded row: zero subtrees, exact
    if (it < IT) {
      float p[NW];
#pragma unroll
      for (int w = 0; w < NW; ++w) p[w] = red[it][w];
      cs[it] = tree_sum<NW>(p);
    }
  }
  const float ss = tree_sum<HR_MAX_IT>(cs);
  const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)K), eps)));

  // ---- norm and stages 0-2, then three stages per pass (blocks of 2^L; groups never cross a block) ----
  hr_pass<3, true, false>(hrow, K, 0, r, gamma, cb);
  __syncthreads();
  int st = 3;
#pragma unroll 1
  for (; st + 3 < L; st += 3) {
    hr_pass<3, false, false>(hrow, K, st, r, gamma, cb);
    __syncthreads();
  }
  float amax = L - st == 3 ? hr_pass<3, false, true>(hrow, K, st, r, gamma, cb)
             : L - st == 2 ? hr_pass<2, false, true>(hrow, K, st, r, gamma, cb)
                           : hr_pass<1, false, true>(hrow, K, st, r, gamma, cb);
  amax = warp_max(amax);
  if (lane == 0) red[0][warp] = amax;                // red's partial sums were read before the first pass's barrier
  __syncthreads();
  float a = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) a = fmaxf(a, red[0][w]);
  const float s = __fdiv_rn(7.0f, fmaxf(a, 1e-5f));

  // ---- codes: 32 elements (16 bytes) per step, two per byte ----
  for (int c32 = tid; c32 < K / 32; c32 += HR_THREADS) {
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = pack_nibbles8(hrow + hr_pidx(32 * c32 + 8 * q), s);   // 8 adjacent slots
    *reinterpret_cast<uint4*>(Xq4 + (size_t)m * (K / 2) + 16 * (size_t)c32) = make_uint4(w[0], w[1], w[2], w[3]);
    if (T_dbg != nullptr) {
#pragma unroll
      for (int q = 0; q < 32; q += 4) {
        const float* src = hrow + hr_pidx(32 * c32 + q);
        *reinterpret_cast<float4*>(T_dbg + (size_t)m * K + 32 * (size_t)c32 + q) =
            make_float4(src[0], src[1], src[2], src[3]);
      }
    }
  }
  if (tid == 0) s_x[m] = s;
}

// ---------------------------------------------------------------------------
// host launchers (called from abi.cu after validation)
// ---------------------------------------------------------------------------
// ---------------------------------------------------------------------------
// RMSNorm + Hadamard + int4, one token per CTA of T = K / 32 threads (K =
// 2048, 4096, 8192 or 16384: W = log2(T / 32) = 1 .. 4 warp bits), 32 elements
// per thread, for blocks of b = 2^L >= 1024.  The element index bits are handled in
// three groups, each while a thread holds all 32 elements the group's stages
// pair up (stages always in the order stride 1, 2, ..., b/2):
//   mapping A: thread t holds elements 32t .. 32t+31 (bits 0-4 in-thread):
//              coalesced loads, the sum of squares (in-thread tree, lanes,
//              warps in order), the norm, stages 0-4;
//   mapping B: in-thread bits 5-9, thread = (bits 10.. << 5) | bits 0-4:
//              stages 5-9;
//   mapping C: in-thread bits 10..10+W-1 and 0..4-W, thread = bits 5-W .. 9:
//              stages 10 .. L-1, the normalisation c_b, the absmax and the
//              codes (bit 0 is in-thread, so codes pair into bytes there).
// The row goes through shared memory between mappings with one pad word per
// 32 (every access pattern is conflict-free).  Fewer registers per thread
// than the 128-element kernel, so more warps keep the SM busy; every value is
// the one the other Hadamard kernels produce.
// ---------------------------------------------------------------------------
BN_DEV int hsidx(int e) { return e + (e >> 5); }

template <int W>
BN_DEV int map_b(int t, int c) { return ((t >> 5) << 10) | (c << 5) | (t & 31); }

template <int W>
BN_DEV int map_c(int t, int c) {
  constexpr int LOW = 5 - W;                       // low in-thread bits
  return ((c >> LOW) << 10) | (t << LOW) | (c & ((1 << LOW) - 1));
}

// Radix-2 stages s = S0 .. S1-1 (stride 2^s) on 32 in-thread values whose
// in-thread index bit (s - SHIFT) is element bit s.
template <int S0, int S1, int SHIFT>
BN_DEV void fwht32(float (&v)[32]) {
#pragma unroll
  for (int st = S0; st < S1; ++st) {
    const int h = 1 << (st - SHIFT);
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      if ((c & h) == 0) {
        const float a = v[c], b = v[c + h];
        v[c] = __fadd_rn(a, b);
        v[c + h] = __fsub_rn(a, b);
      }
    }
  }
}

template <typename TIn, int L, int W, int PRE>
__global__ void __launch_bounds__(32 << W, (32 << W) == 512 ? 2 : (32 << W) == 256 ? 4 : (32 << W) == 128 ? 8 : 16)
hadamard_quant_i4_split_kernel(const TIn* __restrict__ X, const float* __restrict__ B, int K,
                               const float* __restrict__ gamma, float eps, float cb, uint8_t* __restrict__ Xq4,
                               float* __restrict__ s_x, float* __restrict__ T_dbg) {
  constexpr int T = 32 << W, NW = 1 << W, LOW = 5 - W;
  static_assert(L >= 10 && L <= 10 + W, "block of 2^10 .. K");
  extern __shared__ float hs[];
  uint8_t* bytes = reinterpret_cast<uint8_t*>(hs + (K + K / 32));
  __shared__ float red[NW];
  pdl_launch_dependents();
  pdl_wait();                                // X may come from, and Xq4 may still be read by, the previous kernel
  const int m = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  float v[32];
  {
    const size_t off = (size_t)m * K + (size_t)t * 32;
    constexpr int E = InVec<TIn>::E;
#pragma unroll
    for (int q = 0; q < 32 / E; ++q) {
      float tmp[E];
      load_chunk<PRE, TIn, E>(X + off + q * E, B + off + q * E, nullptr, tmp);
#pragma unroll
      for (int e = 0; e < E; ++e) v[q * E + e] = tmp[e];
    }
  }
  // ---- sum of squares: in-thread tree (first level fused), lanes, warps in order ----
  float part;
  {
    float sq[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) sq[c] = __fadd_rn(__fmul_rn(v[2 * c], v[2 * c]), __fmul_rn(v[2 * c + 1], v[2 * c + 1]));
    part = warp_tree_sum(tree_sum<16>(sq));
  }
  if (lane == 0) red[warp] = part;
  __syncthreads();
  float w[NW];
#pragma unroll
  for (int i = 0; i < NW; ++i) w[i] = red[i];
  const float ss = tree_sum<NW>(w);
  const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)K), eps)));
  if (gamma != nullptr) {
    const float* gp = gamma + (size_t)t * 32;
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = __fmul_rn(__fmul_rn(v[c], r), __ldg(gp + c));
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = __fmul_rn(v[c], r);
  }
  // ---- stages 0-4 (mapping A) ----
  fwht32<0, 5, 0>(v);
#pragma unroll
  for (int c = 0; c < 32; ++c) hs[hsidx(32 * t + c)] = v[c];
  __syncthreads();
  // ---- stages 5-9 (mapping B) ----
#pragma unroll
  for (int c = 0; c < 32; ++c) v[c] = hs[hsidx(map_b<W>(t, c))];
  fwht32<5, 10, 5>(v);
#pragma unroll
  for (int c = 0; c < 32; ++c) hs[hsidx(map_b<W>(t, c))] = v[c];
  __syncthreads();
  // ---- stages 10 .. L-1 (mapping C), normalisation, absmax ----
#pragma unroll
  for (int c = 0; c < 32; ++c) v[c] = hs[hsidx(map_c<W>(t, c))];
  fwht32<10, L, 10 - LOW>(v);
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    v[c] = __fmul_rn(v[c], cb);
    amax = fmaxf(amax, fabsf(v[c]));
  }
  amax = warp_max(amax);
  __syncthreads();                           // every thread has read red[] (the sum of squares)
  if (lane == 0) red[warp] = amax;
  __syncthreads();
#pragma unroll
  for (int i = 0; i < NW; ++i) amax = fmaxf(amax, red[i]);
  const float sc = __fdiv_rn(7.0f, fmaxf(amax, 1e-5f));
  if (T_dbg != nullptr) {
    float* dst = T_dbg + (size_t)m * K;
#pragma unroll
    for (int c = 0; c < 32; ++c) dst[map_c<W>(t, c)] = v[c];
  }
  // ---- codes, two per byte (element pairs differ in bit 0, held in-thread) ----
#pragma unroll
  for (int hh = 0; hh < NW; ++hh) {
    const int e0 = map_c<W>(t, hh << LOW);           // first element of this run of 2^LOW
#pragma unroll
    for (int j = 0; j < (1 << LOW); j += 2) {
      const int c = (hh << LOW) + j;
      bytes[(e0 + j) >> 1] = (uint8_t)pair_nibbles(nib(v[c], sc), nib(v[c + 1], sc));
    }
  }
  __syncthreads();
  const uint4* src = reinterpret_cast<const uint4*>(bytes);
  uint4* dst = reinterpret_cast<uint4*>(Xq4 + (size_t)m * (K / 2));
  for (int q = t; q < K / 32; q += T) dst[q] = src[q];
  if (t == 0) s_x[m] = sc;
}

// ---------------------------------------------------------------------------
// RMSNorm + Hadamard + int4 for K = 8192 in one block of b = 8192 (the H-
// BitLinear input of the 2048 x 8192 workload), one token per CTA of 256
// threads, on packed fp32 pairs (add / sub / mul .f32x2: half the arithmetic
// instructions of the scalar stages, the same roundings).  Every mapping keeps
// element bit 0 inside a thread's 64-bit register pair, so a pair is the unit
// of the stages that do not touch bit 0 and of the shared-memory traffic:
//   mapping A: thread t holds elements 32t .. 32t+31 (bits 0-4 in-thread):
//              the loads, the sum of squares, the norm, stage 0 (the one stage
//              inside a pair, scalar) and stages 1-4 (packed);
//   mapping B: in-thread bits 0 and 5-8, thread = bits 1-4 and 9-12: stages 5-8;
//   mapping C: in-thread bits 0 and 9-12, thread = bits 1-8: stages 9-12, the
//              normalisation c_b, the absmax and the codes (a pair is a byte).
// The row sits in shared memory as 32-element lines whose 16-byte slots
// (bits 2-4) are XOR-swizzled by bits 5-7: the mapping-A float4 stores and the
// mapping-B/C float2 accesses are all conflict-free.  Every value is the one
// the other Hadamard kernels produce.
// ---------------------------------------------------------------------------
constexpr int HP_K = 8192;
constexpr int HP_T = 256;

BN_DEV int hp_phys(int e) { return e ^ (((e >> 5) & 7) << 2); }

// Butterflies on pairs: stages whose element bit is in-thread bit 1 + i of the
// pair index's bit i, for pair-index strides 1, 2, 4, 8 (four stages).
BN_DEV void fwht_pairs16(uint64_t (&p)[16]) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if ((j & h) == 0) {
        const uint64_t a = p[j], b = p[j + h];
        p[j] = f2_add(a, b);
        p[j + h] = f2_sub(a, b);
      }
    }
  }
}

template <typename TIn, int PRE>
__global__ void __launch_bounds__(HP_T, 4)
hadamard_quant_i4_pair_kernel(const TIn* __restrict__ X, const float* __restrict__ B,
                              const float* __restrict__ gamma, float eps, float cb, uint8_t* __restrict__ Xq4,
                              float* __restrict__ s_x, float* __restrict__ T_dbg) {
  constexpr int NW = HP_T / 32;
  __shared__ __align__(16) float hs[HP_K];
  __shared__ float red[NW];
  pdl_launch_dependents();
  pdl_wait();                                // X may come from, and Xq4 may still be read by, the previous kernel
  const int m = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  float v[32];
  {
    const size_t off = (size_t)m * HP_K + (size_t)t * 32;
    constexpr int E = InVec<TIn>::E;
#pragma unroll
    for (int q = 0; q < 32 / E; ++q) {
      float tmp[E];
      load_chunk<PRE, TIn, E>(X + off + q * E, B + off + q * E, nullptr, tmp);
#pragma unroll
      for (int e = 0; e < E; ++e) v[q * E + e] = tmp[e];
    }
  }
  // ---- sum of squares: in-thread tree (first level fused), lanes, warps in order ----
  {
    float sq[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      float a, b;
      f2_unpack(f2_mul(f2_pack(v[2 * c], v[2 * c + 1]), f2_pack(v[2 * c], v[2 * c + 1])), a, b);
      sq[c] = __fadd_rn(a, b);
    }
    const float part = warp_tree_sum(tree_sum<16>(sq));
    if (lane == 0) red[warp] = part;
  }
  __syncthreads();
  float w[NW];
#pragma unroll
  for (int i = 0; i < NW; ++i) w[i] = red[i];
  const float ss = tree_sum<NW>(w);
  const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)HP_K), eps)));
  // ---- norm, stage 0 (inside each pair), stages 1-4 (mapping A) ----
  uint64_t p[16];
  {
    const uint64_t rr = f2_pack(r, r);
    const float* gp = gamma + (size_t)t * 32;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      uint64_t x = f2_mul(f2_pack(v[2 * j], v[2 * j + 1]), rr);
      if (gamma != nullptr) x = f2_mul(x, f2_pack(__ldg(gp + 2 * j), __ldg(gp + 2 * j + 1)));
      float a, b;
      f2_unpack(x, a, b);
      p[j] = f2_pack(__fadd_rn(a, b), __fsub_rn(a, b));
    }
  }
  fwht_pairs16(p);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int e = 32 * t + 4 * q;
    *reinterpret_cast<ulonglong2*>(hs + hp_phys(e)) = make_ulonglong2(p[2 * q], p[2 * q + 1]);
  }
  __syncthreads();
  // ---- stages 5-8 (mapping B: pair j holds elements (t & 15) << 1 | j << 5 | (t >> 4) << 9, +1) ----
  const int eb = ((t & 15) << 1) | ((t >> 4) << 9);
#pragma unroll
  for (int j = 0; j < 16; ++j) p[j] = *reinterpret_cast<const uint64_t*>(hs + hp_phys(eb | (j << 5)));
  fwht_pairs16(p);
#pragma unroll
  for (int j = 0; j < 16; ++j) *reinterpret_cast<uint64_t*>(hs + hp_phys(eb | (j << 5))) = p[j];
  __syncthreads();
  // ---- stages 9-12 (mapping C: pair j holds elements t << 1 | j << 9, +1) ----
#pragma unroll
  for (int j = 0; j < 16; ++j) p[j] = *reinterpret_cast<const uint64_t*>(hs + hp_phys((t << 1) | (j << 9)));
  fwht_pairs16(p);
  float amax = 0.f;
  {
    const uint64_t cc = f2_pack(cb, cb);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      p[j] = f2_mul(p[j], cc);
      float a, b;
      f2_unpack(p[j], a, b);
      amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
    }
  }
  amax = warp_max(amax);
  __syncthreads();                           // every thread has read red[] (the sum of squares)
  if (lane == 0) red[warp] = amax;
  __syncthreads();
#pragma unroll
  for (int i = 0; i < NW; ++i) amax = fmaxf(amax, red[i]);
  const float sc = __fdiv_rn(7.0f, fmaxf(amax, 1e-5f));
  if (T_dbg != nullptr) {
    float* dst = T_dbg + (size_t)m * HP_K;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float a, b;
      f2_unpack(p[j], a, b);
      *reinterpret_cast<float2*>(dst + ((t << 1) | (j << 9))) = make_float2(a, b);
    }
  }
  // ---- codes: pair j is byte t + 256 j (the even element in the low nibble) ----
  {
    // The products are packed; the rounding additions stay scalar: a packed
    // multiply followed by a packed add may be fused into one packed fma,
    // which would round t * s + 1.5 * 2^23 once instead of twice.
    const uint64_t ss2 = f2_pack(sc, sc);
    uint8_t* dst = Xq4 + (size_t)m * (HP_K / 2) + t;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float a, b;
      f2_unpack(f2_mul(p[j], ss2), a, b);
      dst[256 * j] = (uint8_t)pair_nibbles(rint_low_bits(a), rint_low_bits(b));
    }
  }
  if (t == 0) s_x[m] = sc;
}

// ---------------------------------------------------------------------------
// RMSNorm + Hadamard + int4 for blocks of b = 2^L <= 512 elements, one warp per
// block and one CTA per token (K / b <= 32 warps; e.g. K = 5632 in 11 blocks of
// 512, the down projection's input).  Lane j holds the E = b / 32 consecutive
// elements b w + E j .. of block w: stages of stride < E run in registers, the
// five stages of stride E .. b/2 pair lanes (xor shuffles: the lower lane keeps
// a + c, the upper a - c).  The sum of squares follows the fixed tree: in-lane,
// lanes, then the warps' block sums in order, padded with zero subtrees.  Every
// value is the one the other Hadamard kernels produce.
// ---------------------------------------------------------------------------
template <typename TIn, int L, int PRE>
__global__ void __launch_bounds__(1024)
hadamard_quant_i4_warp_kernel(const TIn* __restrict__ X, const float* __restrict__ B, int K,
                              const float* __restrict__ gamma, float eps, float cb, uint8_t* __restrict__ Xq4,
                              float* __restrict__ s_x, float* __restrict__ T_dbg) {
  constexpr int E = 1 << (L - 5);
  static_assert(L >= 6 && L <= 9, "2 to 16 elements per lane");
  __shared__ float red[32];
  pdl_launch_dependents();
  pdl_wait();                                // X may come from, and Xq4 may still be read by, the previous kernel
  const int m = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const size_t e0 = (size_t)warp * (E * 32) + (size_t)lane * E;      // first element of this lane
  float v[E];
  {
    constexpr int EV = InVec<TIn>::E;
    const size_t off = (size_t)m * K + e0;
    if constexpr (E >= EV) {
#pragma unroll
      for (int q = 0; q < E / EV; ++q) {
        float tmp[EV];
        load_chunk<PRE, TIn, EV>(X + off + q * EV, B + off + q * EV, nullptr, tmp);
#pragma unroll
        for (int e = 0; e < EV; ++e) v[q * EV + e] = tmp[e];
      }
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        float x;
        if constexpr (sizeof(TIn) == 4) x = reinterpret_cast<const float*>(X)[off + e];
        else x = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(X)[off + e] << 16);
        if constexpr (PRE == PRE_GLU) x = relu2_times(x, B[off + e]);
        v[e] = x;
      }
    }
  }
  // ---- sum of squares: in-lane tree, lanes, warps (zero-padded to 32) in order ----
  float sq[E];
#pragma unroll
  for (int c = 0; c < E; ++c) sq[c] = __fmul_rn(v[c], v[c]);
  float part = warp_tree_sum(tree_sum<E>(sq));
  if (lane == 0) red[warp] = part;
  __syncthreads();
  float wsum[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) wsum[i] = i < nw ? red[i] : 0.f;
  const float ss = tree_sum<32>(wsum);
  const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)K), eps)));
  if (gamma != nullptr) {
#pragma unroll
    for (int c = 0; c < E; ++c) v[c] = __fmul_rn(__fmul_rn(v[c], r), __ldg(gamma + e0 + c));
  } else {
#pragma unroll
    for (int c = 0; c < E; ++c) v[c] = __fmul_rn(v[c], r);
  }
  // ---- stages of stride 1 .. E/2 in registers, then E .. b/2 across lanes,
  // on packed fp32 pairs (elements 2j, 2j+1) except the stride-1 stage ----
  uint64_t pv[E / 2];
#pragma unroll
  for (int j = 0; j < E / 2; ++j) pv[j] = f2_pack(__fadd_rn(v[2 * j], v[2 * j + 1]), __fsub_rn(v[2 * j], v[2 * j + 1]));
#pragma unroll
  for (int h = 1; h < E / 2; h <<= 1) {
#pragma unroll
    for (int j = 0; j < E / 2; ++j) {
      if ((j & h) == 0) {
        const uint64_t a = pv[j], b = pv[j + h];
        pv[j] = f2_add(a, b);
        pv[j + h] = f2_sub(a, b);
      }
    }
  }
#pragma unroll
  for (int lb = 1; lb < 32; lb <<= 1) {
    // the lower lane keeps v + other, the upper other - v: (+-1) * v + other
    const float sg = (lane & lb) != 0 ? -1.0f : 1.0f;
    const uint64_t sg2 = f2_pack(sg, sg);
#pragma unroll
    for (int j = 0; j < E / 2; ++j) {
      float a, b;
      f2_unpack(pv[j], a, b);
      const float oa = __shfl_xor_sync(0xffffffffu, a, lb), ob = __shfl_xor_sync(0xffffffffu, b, lb);
      pv[j] = f2_fma(sg2, pv[j], f2_pack(oa, ob));
    }
  }
#pragma unroll
  for (int j = 0; j < E / 2; ++j) f2_unpack(pv[j], v[2 * j], v[2 * j + 1]);
  // ---- normalise, absmax over the token ----
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < E; ++c) {
    v[c] = __fmul_rn(v[c], cb);
    amax = fmaxf(amax, fabsf(v[c]));
  }
  amax = warp_max(amax);
  __syncthreads();                           // every warp has read red[] (the sum of squares)
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  for (int i = 0; i < nw; ++i) amax = fmaxf(amax, red[i]);
  const float sc = __fdiv_rn(7.0f, fmaxf(amax, 1e-5f));
  if (T_dbg != nullptr) {
#pragma unroll
    for (int c = 0; c < E; ++c) T_dbg[(size_t)m * K + e0 + c] = v[c];
  }
  // ---- E / 2 bytes of codes per lane, contiguous ----
  uint8_t* dst = Xq4 + (size_t)m * (K / 2) + e0 / 2;
  if constexpr (E >= 8) {
    uint32_t w[E / 8];
#pragma unroll
    for (int q = 0; q < E / 8; ++q) w[q] = pack_nibbles8(v + 8 * q, sc);
    if constexpr (E == 16) *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
    else *reinterpret_cast<uint32_t*>(dst) = w[0];
  } else {
#pragma unroll
    for (int c = 0; c < E; c += 2) dst[c / 2] = (uint8_t)pair_nibbles(nib(v[c], sc), nib(v[c + 1], sc));
  }
  if (threadIdx.x == 0) s_x[m] = sc;
}

template <typename TIn, int NT, int IT, int PRE>
static cudaError_t launch_q8(const void* X, const float* B, float* H, int M, int K, const float* gamma, float eps,
                             int8_t* Xq, float* s_x, cudaStream_t st) {
  return launch_pdl(quant_act_i8_kernel<TIn, NT, IT, PRE>, dim3(M), dim3(NT), 0, st, 1u,
                    static_cast<const TIn*>(X), B, H, K, gamma, eps, Xq, s_x);
}

template <typename TIn, int PRE>
static cudaError_t dispatch_q8(const void* X, const float* B, float* H, int M, int K, const float* gamma, float eps,
                               int8_t* Xq, float* s_x, cudaStream_t st) {
  constexpr int E = InVec<TIn>::E;
  int C = K / E, PC = 1;
  while (PC < C) PC <<= 1;
#define BN_Q8(NT, IT) launch_q8<TIn, NT, IT, PRE>(X, B, H, M, K, gamma, eps, Xq, s_x, st)
  // 512 chunks a token (K = 2048 fp32, 4096 bf16) with few tokens (up to four
  // per SM): more threads a token shorten its serial part.  Measured on B200,
  // per launch: 512 x 2048 fp32 with the residual add 4.8 -> 4.1 us (512
  // threads), without it 3.2 -> 3.1 us (256); 32 x 2048 with the add 2.4 ->
  // 2.0 us (256).  Many tokens keep 128 threads (4096 x 4096 bf16: 9.7 us,
  // against 13.4 with 256).  Every choice gives the same balanced tree over
  // the chunk index, hence the same bits.
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const bool few = M <= 4 * sms;
  if (PC <= 1024) {
    switch (PC <= 128 ? 1 : PC / 128) {
      case 1: return BN_Q8(128, 1);
      case 2: return BN_Q8(128, 2);
      case 4:
        if (few && PRE == PRE_ADD && M > 64) return BN_Q8(512, 1);
        if (few) return BN_Q8(256, 2);
        return BN_Q8(128, 4);
      case 8: return BN_Q8(128, 8);
    }
  } else {
    switch (PC / 256) {
      case 8: return BN_Q8(256, 8);
      case 16: return BN_Q8(256, 16);
    }
  }
#undef BN_Q8
  return cudaErrorInvalidValue;
}

cudaError_t run_quant_act_i8(const void* X, int bf16, int M, int K, const float* gamma, float eps,
                             int8_t* Xq, float* s_x, cudaStream_t st) {
  return bf16 ? dispatch_q8<uint16_t, PRE_NONE>(X, nullptr, nullptr, M, K, gamma, eps, Xq, s_x, st)
              : dispatch_q8<float, PRE_NONE>(X, nullptr, nullptr, M, K, gamma, eps, Xq, s_x, st);
}

cudaError_t run_add_quant_act_i8(const float* A, const float* B, int M, int K, const float* gamma, float eps,
                                 float* H, int8_t* Xq, float* s_x, cudaStream_t st) {
  return dispatch_q8<float, PRE_ADD>(A, B, H, M, K, gamma, eps, Xq, s_x, st);
}

template <typename TIn, int L, int PRE>
static cudaError_t launch_h4(const void* X, const float* B, int M, int K, const float* gamma, float eps,
                             uint8_t* Xq4, float* s_x, float* T_dbg, cudaStream_t st) {
  const int G = K / HT_R;
  int GP = 1;
  while (GP < G) GP <<= 1;
  const int TPB = GP >= 128 ? 1 : 128 / GP;
  const int threads = TPB * GP;
  const float cb = (float)(1.0 / sqrt((double)(1 << L)));
  // Blocks of 64 .. 512 elements and at most 32 of them: one warp per block.
  if constexpr (L >= 6 && L <= 9) {
    if (K / (1 << L) <= 32) {
      auto wk = hadamard_quant_i4_warp_kernel<TIn, L, PRE>;
      const float cbw = (float)(1.0 / sqrt((double)(1 << L)));
      return launch_pdl(wk, dim3(M), dim3(32 * (K >> L)), 0, st, 1u, static_cast<const TIn*>(X), B, K, gamma, eps,
                        cbw, Xq4, s_x, T_dbg);
    }
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // K = 8192 in one block: the packed-pair kernel.
  if constexpr (L == 13) {
    if (K == HP_K) {
      return launch_pdl(hadamard_quant_i4_pair_kernel<TIn, PRE>, dim3((unsigned)M), dim3(HP_T), 0, st, 1u,
                        static_cast<const TIn*>(X), B, gamma, eps, cb, Xq4, s_x, T_dbg);
    }
  }
  // K = 2048 / 4096 / 8192 / 16384, blocks of 1024 or more: one token per CTA
  // of K / 32 threads, 32 elements per thread.
  if constexpr (L >= 10) {
    const int W = K == 2048 ? 1 : K == 4096 ? 2 : K == 8192 ? 3 : K == 16384 ? 4 : 0;
    // 64 or 128 threads per token only with many tokens: measured on B200 at
    // 512 tokens of K = 2048 (the O projection's input) the one-CTA-per-token
    // kernel's 256 threads take 5.3 us per launch against 7.7 us here (two
    // warps per token leave the SMs short of warps)
    if (W != 0 && L <= 10 + W && (W >= 3 || M >= 16 * sms)) {
      const size_t ssmem = (size_t)(K + K / 32) * sizeof(float) + (size_t)K / 2;
      const unsigned grid = (unsigned)M;
#define BN_HS(WW)                                                                                           \
  do {                                                                                                      \
    if constexpr (L <= 10 + WW) {                                                                           \
      auto sk = hadamard_quant_i4_split_kernel<TIn, L, WW, PRE>;                                            \
      cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(sk), ssmem);                          \
      if (e != cudaSuccess) return e;                                                                       \
      return launch_pdl(sk, dim3(grid), dim3(32 << WW), ssmem, st, 1u, static_cast<const TIn*>(X), B, K,    \
                        gamma, eps, cb, Xq4, s_x, T_dbg);                                                   \
    }                                                                                                       \
  } while (0)
      if (W == 1) BN_HS(1);
      if (W == 2) BN_HS(2);
      if (W == 3) BN_HS(3);
      if (W == 4) BN_HS(4);
#undef BN_HS
    }
  }
  // Few tokens: the register kernel would leave most SMs idle; one CTA per token instead.
  if ((M + TPB - 1) / TPB < 2 * sms) {
    auto rk = hadamard_quant_i4_row_kernel<TIn, L, PRE>;
    const size_t rsmem = (size_t)(K + K / 8) * sizeof(float);
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(rk), rsmem);
    if (e != cudaSuccess) return e;
    return launch_pdl(rk, dim3(M), dim3(HR_THREADS), rsmem, st, 1u, static_cast<const TIn*>(X), B, K, gamma, eps, cb,
                      Xq4, s_x, T_dbg);
  }
  const size_t smem = (size_t)TPB * ((K + 2 * (K >> 7) + 3) & ~3) * sizeof(float) + (size_t)TPB * 4 * sizeof(float);
  auto kern = hadamard_quant_i4_kernel<TIn, L, PRE>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  const int grid = (M + TPB - 1) / TPB;
  return launch_pdl(kern, dim3(grid), dim3(threads), smem, st, 1u, static_cast<const TIn*>(X), B, M, K, GP, gamma,
                    eps, cb, Xq4, s_x, T_dbg);
}

template <typename TIn, int PRE>
static cudaError_t dispatch_h4(const void* X, const float* B, int M, int K, int L, const float* gamma, float eps,
                               uint8_t* Xq4, float* s_x, float* T_dbg, cudaStream_t st) {
#define BN_H4(LL) launch_h4<TIn, LL, PRE>(X, B, M, K, gamma, eps, Xq4, s_x, T_dbg, st)
  switch (L) {
    case 5: return BN_H4(5);
    case 6: return BN_H4(6);
    case 7: return BN_H4(7);
    case 8: return BN_H4(8);
    case 9: return BN_H4(9);
    case 10: return BN_H4(10);
    case 11: return BN_H4(11);
    case 12: return BN_H4(12);
    case 13: return BN_H4(13);
  }
#undef BN_H4
  return cudaErrorInvalidValue;
}

cudaError_t run_hadamard_quant_i4(const void* X, int bf16, int M, int K, int L, const float* gamma,
                                  float eps, uint8_t* Xq4, float* s_x, float* T_dbg, cudaStream_t st) {
  return bf16 ? dispatch_h4<uint16_t, PRE_NONE>(X, nullptr, M, K, L, gamma, eps, Xq4, s_x, T_dbg, st)
              : dispatch_h4<float, PRE_NONE>(X, nullptr, M, K, L, gamma, eps, Xq4, s_x, T_dbg, st);
}

cudaError_t run_glu_hadamard_quant_i4(const float* gate, const float* up, int M, int K, int L, const float* gamma,
                                      float eps, uint8_t* Xq4, float* s_x, cudaStream_t st) {
  return dispatch_h4<float, PRE_GLU>(gate, up, M, K, L, gamma, eps, Xq4, s_x, nullptr, st);
}

}  // namespace bitnet
