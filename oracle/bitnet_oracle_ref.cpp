// Second CPU oracle of the BitNet b1.58 BitLinear forward, in plain C++.
//
// TEST INFRASTRUCTURE, like bitnet_oracle.py beside it: only tests/ load it.
// It shares no code with the CUDA path or with the numpy oracle; the tests
// require the two oracles to agree bit for bit, so a slip in either shows.
// Built with -O2 -ffp-contract=off and no fast-math: every float operation is
// one IEEE-754 round-to-nearest-even operation, as written.  With -fopenmp the
// loops over tokens and output rows run on all cores; every element is still
// computed by the same operations in the same order, so the results do not
// change.
//
// Sources, by page title and section:
//  "LLM을 1.58비트로 파인튜닝: BitNet을 이용한 극단적인 양자화", section 양자화
//    메커니즘: weights scaled by the reciprocal of their mean absolute value,
//    rounded, clamped to [-1, 1]; activations quantised per token by absmax
//    into [-128, 127] after a norm.  Section 계산 패러다임: integer products.
//  "초저용량 LLM의 진화: BitNet v2 파헤치기", section 방법론: a Hadamard
//    transform before 4-bit activation quantisation.
//  "양자화(quantization) 1.58bit" (endplan.ai): the absmax factor 127/absmax;
//    three states carry log2(3) = 1.58 bits.
// Readings where the pages are silent are the same as the numpy oracle's:
// exact sum of |W| rounded once to fp64, RMSNorm with a balanced pairwise fp32
// sum, 1e-5 scale floors, Sylvester-order radix-2 Hadamard stages, 2-bit
// two's complement codes with weight 4j+i of a 16-weight word at bits 8i+2j,
// and five weights per byte as base-3 digits w + 1.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

const float kFloor = 1e-5f;

// Exact sum of |w| kept as an integer multiple of 2^-149 (the smallest fp32
// step) in 6 x 64-bit limbs, least significant first: 384 bits hold 2^31
// magnitudes below 2^128.
struct BigSum {
  uint64_t limb[6] = {0, 0, 0, 0, 0, 0};

  void add_shifted(uint64_t v, int shift) {        // += v * 2^shift, v < 2^55
    int li = shift / 64, bi = shift % 64;
    unsigned __int128 part = (unsigned __int128)v << bi;
    uint64_t carry = 0;
    for (int i = li; i < 6; ++i) {
      unsigned __int128 add = (unsigned __int128)limb[i] + (uint64_t)part + carry;
      limb[i] = (uint64_t)add;
      carry = (uint64_t)(add >> 64);
      part >>= 64;
      if (part == 0 && carry == 0) break;
    }
  }

  int top_bit() const {
    for (int i = 5; i >= 0; --i)
      if (limb[i]) return 64 * i + 63 - __builtin_clzll(limb[i]);
    return -1;
  }

  int bit(int b) const { return (int)((limb[b / 64] >> (b % 64)) & 1u); }

  bool any_below(int b) const {                    // any set bit at positions < b
    for (int i = 0; i < 6 && 64 * i < b; ++i) {
      const int hi = b - 64 * i;
      const uint64_t mask = hi >= 64 ? ~0ull : ((1ull << hi) - 1);
      if (limb[i] & mask) return true;
    }
    return false;
  }

  // The value times 2^-149, rounded once to double (nearest, ties to even).
  double to_double() const {
    const int t = top_bit();
    if (t < 0) return 0.0;
    uint64_t mant = 0;
    int low = t - 52;                              // lowest kept bit
    if (low < 0) low = 0;
    for (int b = t; b >= low; --b) mant = (mant << 1) | (uint64_t)bit(b);
    if (low > 0) {
      const int g = bit(low - 1);                  // first dropped bit
      const bool sticky = any_below(low - 1);
      if (g && (sticky || (mant & 1u))) ++mant;    // may carry into 2^53: ldexp keeps it exact
    }
    return std::ldexp((double)mant, low - 149);
  }
};

// Balanced pairwise sum of n floats: zero-pad to a power of two, then add
// adjacent pairs level by level.
float pairwise_sum(const float* v, int64_t n) {
  int64_t p = 1;
  while (p < n) p *= 2;
  std::vector<float> buf((size_t)p, 0.0f);
  std::memcpy(buf.data(), v, (size_t)n * sizeof(float));
  for (int64_t len = p; len > 1; len /= 2)
    for (int64_t i = 0; i < len / 2; ++i) buf[(size_t)i] = buf[(size_t)(2 * i)] + buf[(size_t)(2 * i + 1)];
  return buf[0];
}

int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

}  // namespace

extern "C" {

// threads the row loops use
int oc_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// sum |w| exactly, then one rounding to double.
double oc_exact_sum_abs(const float* w, int64_t n) {
  BigSum acc;
  // significands that share an exponent are summed first (exact in 64 bits)
  std::vector<uint64_t> per_exp(256, 0);
  for (int64_t i = 0; i < n; ++i) {
    uint32_t u;
    std::memcpy(&u, &w[i], 4);
    const uint32_t e = (u >> 23) & 0xFF, f = u & 0x7FFFFF;
    const uint64_t m = e ? (f | 0x800000u) : f;   // |w| = m * 2^(max(e,1) - 150)
    per_exp[e ? e : 1] += m;
  }
  for (int e = 1; e < 255; ++e)
    if (per_exp[(size_t)e]) acc.add_shifted(per_exp[(size_t)e], e - 1);   // 2^(e-150) = 2^(e-1) * 2^-149
  return acc.to_double();
}

// mean |W| (fp64 division of the exact sum, one rounding to fp32) and
// s_w = 1 / max(mean, 1e-5) in fp32.
void oc_weight_scale(const float* w, int64_t n, float* mean, float* s_w) {
  const float m = (float)(oc_exact_sum_abs(w, n) / (double)n);
  *mean = m;
  *s_w = 1.0f / (m > kFloor ? m : kFloor);
}

void oc_ternarize(const float* w, int64_t n, float s_w, int8_t* q) {
  for (int64_t i = 0; i < n; ++i) q[i] = (int8_t)clampi((int)std::nearbyint(w[i] * s_w), -1, 1);
}

// four 2-bit codes per byte: in the 32-bit word of weights 16g .. 16g+15,
// weight 16g + 4j + i at bits 8i + 2j, code = w & 3 (two's complement)
void oc_pack_ternary(const int8_t* q, int64_t N, int64_t K, uint8_t* pk) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t g = 0; g < K / 16; ++g) {
      uint32_t word = 0;
      for (int j = 0; j < 4; ++j)
        for (int i = 0; i < 4; ++i)
          word |= (uint32_t)(q[n * K + 16 * g + 4 * j + i] & 3) << (8 * i + 2 * j);
      for (int b = 0; b < 4; ++b) pk[n * (K / 4) + 4 * g + b] = (uint8_t)(word >> (8 * b));
    }
}

// five weights per byte: byte g = sum_i (w[5g+i] + 1) * 3^i, zero weights past
// K, each row row_bytes long
void oc_pack_trit5(const int8_t* q, int64_t N, int64_t K, int64_t row_bytes, uint8_t* pk5) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t g = 0; g < row_bytes; ++g) {
      int b = 0, p = 1;
      for (int i = 0; i < 5; ++i) {
        const int64_t k = 5 * g + i;
        b += (k < K ? q[n * K + k] + 1 : 1) * p;
        p *= 3;
      }
      pk5[n * row_bytes + g] = (uint8_t)b;
    }
}

// y = (x * r) * gamma with r = 1 / sqrt(sum(x*x) / K + eps), the sum by the
// balanced pairwise tree
void oc_rms_norm(const float* x, int64_t M, int64_t K, const float* gamma, float eps, float* y, float* r_out) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    std::vector<float> sq((size_t)K);
    const float* row = x + m * K;
    for (int64_t k = 0; k < K; ++k) sq[(size_t)k] = row[k] * row[k];
    const float ms = pairwise_sum(sq.data(), K) / (float)K;
    const float r = 1.0f / std::sqrt(ms + eps);
    if (r_out) r_out[m] = r;
    for (int64_t k = 0; k < K; ++k) {
      float v = row[k] * r;
      if (gamma) v = v * gamma[k];
      y[m * K + k] = v;
    }
  }
}

// s = qmax / max(max|y|, 1e-5); q = clamp(rint(y * s), qmin, qmax)
void oc_absmax_quantize(const float* y, int64_t M, int64_t K, int qmax, int qmin, int8_t* q, float* s) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) amax = std::fabs(y[m * K + k]) > amax ? std::fabs(y[m * K + k]) : amax;
    const float sc = (float)qmax / (amax > kFloor ? amax : kFloor);
    s[m] = sc;
    for (int64_t k = 0; k < K; ++k)
      q[m * K + k] = (int8_t)clampi((int)std::nearbyint(y[m * K + k] * sc), qmin, qmax);
  }
}

// Walsh-Hadamard transform in Sylvester order per block, in place: radix-2
// stages of stride h = 1, 2, ..., block/2, pair (a, c) -> (a + c, a - c),
// then every value times fp32(1 / sqrt(block))
void oc_hadamard(float* y, int64_t M, int64_t K, int64_t block) {
  const float c = (float)(1.0 / std::sqrt((double)block));
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t b0 = 0; b0 < K; b0 += block) {
      float* u = y + m * K + b0;
      for (int64_t h = 1; h < block; h *= 2)
        for (int64_t i = 0; i < block; ++i)
          if ((i & h) == 0) {
            const float a = u[i], d = u[i + h];
            u[i] = a + d;
            u[i + h] = a - d;
          }
      for (int64_t i = 0; i < block; ++i) u[i] = u[i] * c;
    }
}

// int4 codes, two per byte, code 2j in the low nibble
void oc_pack_int4(const int8_t* q, int64_t M, int64_t K, uint8_t* pk) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t j = 0; j < K / 2; ++j)
      pk[m * (K / 2) + j] = (uint8_t)((q[m * K + 2 * j] & 0xF) | ((q[m * K + 2 * j + 1] & 0xF) << 4));
}

// acc[m][n] = sum_k qx[m][k] * qw[n][k] in 64-bit integers
void oc_int_matmul(const int8_t* qx, const int8_t* qw, int64_t M, int64_t N, int64_t K, int64_t* acc) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      int64_t s = 0;
      for (int64_t k = 0; k < K; ++k) s += (int64_t)qx[m * K + k] * (int64_t)qw[n * K + k];
      acc[m * N + n] = s;
    }
}

// y = float(acc) * ((1 / s_x) * (1 / s_w)) in fp32
void oc_dequantize(const int64_t* acc, int64_t M, int64_t N, const float* s_x, float s_w, float* y) {
  const float rw = 1.0f / s_w;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    const float dq = (1.0f / s_x[m]) * rw;
    for (int64_t n = 0; n < N; ++n) y[m * N + n] = (float)acc[m * N + n] * dq;
  }
}

// a = (g * g) * up with g = max(gate, 0), fp32 (squared-ReLU gated unit)
void oc_relu2_glu(const float* gate, const float* up, int64_t n, float* a) {
  for (int64_t i = 0; i < n; ++i) {
    const float g = gate[i] > 0.0f ? gate[i] : 0.0f;
    a[i] = (g * g) * up[i];
  }
}

// out = a + b, fp32 (residual adds)
void oc_add(const float* a, const float* b, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = a[i] + b[i];
}

}  // extern "C"
