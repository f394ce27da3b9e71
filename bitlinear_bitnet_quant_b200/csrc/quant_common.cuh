// Pieces of the RMSNorm + absmax quantisers shared by act_quant.cu and the
// fused decode kernel (bitlinear_fused.cu): 16-byte input chunks and the
// fixed pairwise-tree reductions.
#pragma once

#include "common.cuh"

namespace bitnet {

// One 16-byte chunk of activations (E elements), read with a coherent load
// (the activations come from the previous kernel).
template <typename TIn> struct InVec;
template <> struct InVec<float> {
  static constexpr int E = 4;
  static BN_DEV void load(const float* p, float (&v)[4]) {
    uint4 u = ldg_v4(p);
    v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
  }
};
template <> struct InVec<uint16_t> {
  static constexpr int E = 8;
  static BN_DEV void load(const uint16_t* p, float (&v)[8]) {
    uint4 u = ldg_v4(p);
    v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
    v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
  }
};

// Balanced tree over N (power of two) register values, in index order.
template <int N>
BN_DEV float tree_sum(float (&a)[N]) {
#pragma unroll
  for (int s = 1; s < N; s <<= 1) {
#pragma unroll
    for (int i = 0; i < N; i += 2 * s) a[i] = __fadd_rn(a[i], a[i + s]);
  }
  return a[0];
}

// Tree over the 32 lanes: after offsets 1, 2, 4, 8, 16 every lane holds the
// sum in which lane pairs (2u, 2u+1), then quads, ... were combined in order.
BN_DEV float warp_tree_sum(float v) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// rint(x) for |x| < 2^22, as the low bits (two's complement) of the returned
// word.  x + 1.5 * 2^23 lies in [2^23, 2^24), where consecutive fp32 values
// are 1 apart, so the round-to-nearest-even addition rounds x to an integer
// with ties to even, and the sum's mantissa holds 1.5 * 2^23 + rint(x).  One
// full-rate fp32 add replaces a float-to-int conversion.
BN_DEV uint32_t rint_low_bits(float x) { return __float_as_uint(__fadd_rn(x, 12582912.0f)); }

// The low bytes of four rint_low_bits words, first argument in byte 0.
BN_DEV uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Low nibble of lo in bits 0-3 and low nibble of hi in bits 4-7 (bits 8-31
// keep lo's: only the low byte is meant).
BN_DEV uint32_t pair_nibbles(uint32_t lo, uint32_t hi) {
  uint32_t r;
  asm("bfi.b32 %0, %1, %2, 4, 4;" : "=r"(r) : "r"(hi), "r"(lo));
  return r;
}

// Two fp32 values in one 64-bit register and the sm_100 packed arithmetic on
// them (add / sub / mul .rn.f32x2): each half is rounded exactly as the scalar
// __fadd_rn / __fsub_rn / __fmul_rn of the same operands, so a packed stage
// gives the scalar stage's values at half the instructions.  A packed multiply
// whose result feeds a packed add can be contracted into a packed fma (one
// rounding): keep an add that must see the rounded product scalar.
BN_DEV uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
BN_DEV void f2_unpack(uint64_t r, float& lo, float& hi) { asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r)); }
BN_DEV uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
BN_DEV uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
BN_DEV uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// a * b + c with one rounding per half; with a = +-1 the product is exact, so
// the result is the rounded sum (or difference) itself.
BN_DEV uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

}  // namespace bitnet
