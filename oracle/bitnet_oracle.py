"""Plain CPU oracle of the BitNet b1.58 BitLinear forward (and the BitNet v2
H-BitLinear a4 variant).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run this module.
The product path (``bitlinear_bitnet_quant_b200``) never calls it, and this
module imports nothing from the product path: the two share no code.  Inputs
for both come from ``bitlinear_bitnet_quant_b200.workloads``, which holds no
arithmetic of the method.

Everything here is written for a reader to check against the pages by eye:
numpy element-wise fp32 operations (each one IEEE-754 correctly rounded, no
fused multiply-add), exact integer arithmetic, and float64 where the pages
do not fix a precision.  Sources, cited by page title and section:

[P1] "초저용량 LLM의 진화: BitNet v2 파헤치기 (1비트 LLM을 위한 4비트 활성화)",
     section 방법론 (method): H-BitLinear applies a Hadamard transform to the
     activations before 4-bit quantisation; all activations are 4-bit (a4).
[P2] "AI 혁신의 선두: 마이크로소프트의 1비트 LLM, BitNet b1.58 2B4T",
     section 주요 아키텍처 혁신 (key architecture): BitLinear with ternary
     {-1, 0, +1} weights from absmean quantisation; squared ReLU, no bias.
[P4] "LLM을 1.58비트로 파인튜닝: BitNet을 이용한 극단적인 양자화",
     section 양자화 메커니즘 (quantisation mechanism): weights use symmetric
     per-tensor quantisation whose scale is the reciprocal of the mean
     absolute weight; they are scaled, rounded, clamped to [-1, 1] and
     rescaled.  Activations use per-token absmax quantisation to 8 bits in
     [-128, 127], with a layer norm applied before the quantiser.
     Section 계산 패러다임 (compute paradigm): the matmul uses integer
     additions.  Section 주요 결과 (key results): weights are packed into
     int8 tensors (four ternary weights per byte).
[P5] "양자화(quantization) 1.58bit" (endplan.ai), absmax paragraph: divide by
     the largest magnitude and multiply by 127; with absmax 5.4 the
     "quantization factor" is 127/5.4 = 23.5 and dequantisation divides by it.
     Section "1.58비트는 어디서 나온거에요?": three states, log2(3) = 1.58 bits.

Readings where the pages are silent:

* Mean |W| is the exact sum of |W| rounded once to fp64, divided by N*K in
  fp64, rounded to fp32.  s_w = 1 / max(mean, 1e-5) in fp32.
* The norm is RMSNorm (no mean subtraction, no bias):
  ss = sum of x*x in fp32 by the balanced pairwise tree over indices (zero
  padded to a power of two); r = 1 / sqrt(ss / K + eps); y = (x * r) * gamma.
* Codes: s = qmax / max(absmax, 1e-5) in fp32; q = clamp(rint(y * s)) with
  round-half-to-even; qmax = 127 for int8, 7 for int4 (range [-8, 7]).
* Hadamard: Sylvester order, per block of b = largest power of two dividing
  K (or a given power of two), computed by radix-2 stages of stride
  1, 2, 4, ..., b/2 in fp32, then multiplied by fp32(1/sqrt(b)).
* Dequantisation: y = float(acc) * ((1 / s_x) * (1 / s_w)), all fp32.
* Packing: ternary codes as 2-bit two's complement (-1 -> 0b11); in each
  little-endian 32-bit word of 16 consecutive weights, weight 4*j + i sits at
  bits 8*i + 2*j (so byte i holds weights i, 4+i, 8+i, 12+i).  int4 codes:
  byte j holds code 2j in its low nibble and code 2j+1 in its high nibble.
* Denser weight storage (a reading built on P5's log2(3) = 1.58 bits; the pages
  give no format): five ternary weights per byte as base-3 digits,
  byte = sum_i (w_{5g+i} + 1) * 3^i for i = 0..4 (3^5 = 243 <= 256), i.e. 1.6
  bits per weight.  Weights past K count as 0; each row is padded to a
  multiple of 16 bytes with bytes of five zero weights (121).
* Attention core of the stacked layer (P2 names rotary position embedding;
  the pages give no formula): plain float64 definitions.  RoPE turns the pair
  (x[2i], x[2i+1]) of each head by p * 10000^(-2i/d); attention is per-head
  softmax(q k^T / sqrt(d)) v over the keys at positions up to the query's.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

F32 = np.float32
SCALE_FLOOR = F32(1e-5)
DEFAULT_EPS = 1e-6


# ---------------------------------------------------------------------------
# input dtype helper
# ---------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 is the top half of an fp32 bit pattern: widening is exact."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# weights: absmean ternarisation [P4 양자화 메커니즘, P2 주요 아키텍처 혁신]
# ---------------------------------------------------------------------------

def exact_sum_abs(w: np.ndarray) -> float:
    """Sum of |w| over every entry, exact, then rounded once to fp64.

    Each fp32 magnitude is m * 2**(e-24) with an integer significand
    m < 2**24 (np.frexp gives a = f * 2**e, 0.5 <= f < 1).  Significands
    sharing an exponent are summed as int64 (< 2**24 * 2**31, exact), and the
    per-exponent sums are combined as exact rationals.  float(Fraction) is
    round-to-nearest-even.
    """
    a = np.abs(np.asarray(w, dtype=np.float32)).ravel().astype(np.float64)
    frac, expo = np.frexp(a)
    mant = np.ldexp(frac, 24).astype(np.int64)
    total = Fraction(0)
    for e in np.unique(expo[mant != 0]):
        s = int(mant[expo == e].sum())
        total += Fraction(s) * Fraction(2) ** int(e - 24)
    return float(total)


def weight_scale(w: np.ndarray) -> tuple[np.float32, np.float32]:
    """(mean |W|, s_w): s_w is the reciprocal of the mean absolute weight."""
    n = int(np.asarray(w).size)
    mean = F32(exact_sum_abs(w) / float(n))        # fp64 divide, one rounding to fp32
    s_w = F32(1.0) / np.maximum(mean, SCALE_FLOOR)
    return mean, F32(s_w)


def ternarize(w: np.ndarray, s_w) -> np.ndarray:
    """Scale, round (half to even), clamp to [-1, 1]."""
    w32 = np.asarray(w, dtype=np.float32)
    return np.clip(np.rint(w32 * F32(s_w)), -1, 1).astype(np.int8)


def pack_ternary(q: np.ndarray) -> np.ndarray:
    """Four ternary codes per byte; [N, K] int8 -> [N, K/4] uint8 (K % 16 == 0)."""
    q = np.asarray(q, dtype=np.int8)
    N, K = q.shape
    assert K % 16 == 0
    f = (q.astype(np.int64) & 3).reshape(N, K // 16, 4, 4)   # [n, group, j, i]
    word = np.zeros((N, K // 16), dtype=np.uint64)
    for j in range(4):
        for i in range(4):
            word |= (f[:, :, j, i] << (8 * i + 2 * j)).astype(np.uint64)
    return np.ascontiguousarray(word.astype("<u4")).view(np.uint8).reshape(N, K // 4)


def unpack_ternary(pk: np.ndarray) -> np.ndarray:
    """Inverse of pack_ternary: [N, K/4] uint8 -> [N, K] int8."""
    pk = np.ascontiguousarray(pk, dtype=np.uint8)
    N, KB = pk.shape
    word = pk.view("<u4").astype(np.int64)                     # [N, K/16]
    out = np.zeros((N, KB // 4, 4, 4), dtype=np.int8)
    for j in range(4):
        for i in range(4):
            f = (word >> (8 * i + 2 * j)) & 3
            out[:, :, j, i] = np.where(f == 3, -1, f)
    return out.reshape(N, KB * 4)


def quantize_weights(w: np.ndarray):
    """Offline weight path: returns (packed [N, K/4] uint8, s_w fp32, codes int8)."""
    _, s_w = weight_scale(w)
    q = ternarize(w, s_w)
    return pack_ternary(q), s_w, q


def trit5_row_bytes(K: int) -> int:
    """Bytes per row of the five-weights-per-byte format: ceil(K / 5), padded to 16."""
    groups = (K + 4) // 5
    return (groups + 15) // 16 * 16


def pack_trit5(q: np.ndarray) -> np.ndarray:
    """Five ternary weights per byte as base-3 digits [P5, log2(3) = 1.58 bits]:
    byte g of a row = sum_i (q[5g + i] + 1) * 3**i; [N, K] int8 -> [N, trit5_row_bytes(K)] uint8."""
    q = np.asarray(q, dtype=np.int64)
    N, K = q.shape
    assert np.all(np.abs(q) <= 1)
    R = trit5_row_bytes(K)
    digits = np.ones((N, R * 5), dtype=np.int64)          # weight 0 (digit 1) past K and in the padding
    digits[:, :K] = q + 1
    digits = digits.reshape(N, R, 5)
    out = np.zeros((N, R), dtype=np.int64)
    for i in range(5):
        out += digits[:, :, i] * 3 ** i
    return out.astype(np.uint8)


def unpack_trit5(pk: np.ndarray, K: int) -> np.ndarray:
    """Inverse of pack_trit5: [N, trit5_row_bytes(K)] uint8 -> [N, K] int8."""
    b = np.asarray(pk, dtype=np.int64)
    N, R = b.shape
    assert R == trit5_row_bytes(K) and np.all(b <= 242)
    digits = np.zeros((N, R, 5), dtype=np.int64)
    for i in range(5):
        digits[:, :, i] = b % 3
        b = b // 3
    return (digits.reshape(N, R * 5)[:, :K] - 1).astype(np.int8)


# ---------------------------------------------------------------------------
# activations: RMSNorm then per-token absmax [P4 양자화 메커니즘, P5 absmax]
# ---------------------------------------------------------------------------

def pairwise_sum_f32(v: np.ndarray) -> np.ndarray:
    """fp32 sum over the last axis by the balanced binary tree over indices.

    The last axis is zero-padded to a power of two, then adjacent pairs
    (0,1), (2,3), ... are added level by level.
    """
    v = np.asarray(v, dtype=np.float32)
    n = v.shape[-1]
    p = 1
    while p < n:
        p *= 2
    if p > n:
        pad = np.zeros(v.shape[:-1] + (p - n,), dtype=np.float32)
        v = np.concatenate([v, pad], axis=-1)
    while v.shape[-1] > 1:
        v = v[..., 0::2] + v[..., 1::2]
    return v[..., 0]


def rms_norm(x: np.ndarray, gamma=None, eps: float = DEFAULT_EPS):
    """y = x * r * gamma with r = 1/sqrt(mean(x^2) + eps), fp32; returns (y, r)."""
    x = np.asarray(x, dtype=np.float32)
    K = x.shape[-1]
    ss = pairwise_sum_f32(x * x)
    ms = ss / F32(K)
    r = F32(1.0) / np.sqrt(ms + F32(eps))
    y = x * r[..., None]
    if gamma is not None:
        y = y * np.asarray(gamma, dtype=np.float32)
    return y, r


def absmax_quantize(y: np.ndarray, qmax: int, qmin: int):
    """Per-row absmax: s = qmax / max(max|y|, 1e-5); q = clamp(rint(y * s))."""
    y = np.asarray(y, dtype=np.float32)
    amax = np.max(np.abs(y), axis=-1)
    s = F32(qmax) / np.maximum(amax, SCALE_FLOOR)
    q = np.clip(np.rint(y * s[..., None]), qmin, qmax).astype(np.int8)
    return q, s.astype(np.float32)


def quant_act(x: np.ndarray, gamma=None, eps: float = DEFAULT_EPS):
    """BitLinear activation path: RMSNorm, then int8 absmax. Returns (q int8, s_x)."""
    y, _ = rms_norm(x, gamma, eps)
    return absmax_quantize(y, 127, -128)


# ---------------------------------------------------------------------------
# H-BitLinear: RMSNorm, Hadamard, per-token int4 [P1 방법론]
# ---------------------------------------------------------------------------

def default_had_block(K: int) -> int:
    """Largest power of two dividing K."""
    return K & (-K)


def fwht_f32(y: np.ndarray, block: int) -> np.ndarray:
    """Unnormalised Sylvester-order Walsh-Hadamard transform per block, fp32.

    Radix-2 stages of stride h = 1, 2, 4, ..., block/2; each stage replaces
    the pair (a, c) = (u[i], u[i+h]) (bit h of i clear) by (a + c, a - c).
    """
    y = np.asarray(y, dtype=np.float32)
    M, K = y.shape
    assert K % block == 0 and block & (block - 1) == 0
    u = y.reshape(M, K // block, block)
    h = 1
    while h < block:
        v = u.reshape(M, K // block, block // (2 * h), 2, h)
        a, c = v[..., 0, :], v[..., 1, :]
        u = np.stack([a + c, a - c], axis=-2).reshape(M, K // block, block)
        h *= 2
    return u.reshape(M, K)


def hadamard_norm_const(block: int) -> np.float32:
    """fp32(1/sqrt(block)), from the fp64 value."""
    return F32(1.0 / math.sqrt(block))


def hadamard_transform(y: np.ndarray, block: int) -> np.ndarray:
    """Normalised transform t = H_b y / sqrt(b) in fp32 (stages, then one multiply)."""
    return fwht_f32(y, block) * hadamard_norm_const(block)


def pack_int4(q: np.ndarray) -> np.ndarray:
    """[M, K] int8 in [-8, 7] -> [M, K/2] uint8, code 2j low nibble, 2j+1 high."""
    q = np.asarray(q, dtype=np.int8).astype(np.int64)
    lo = q[:, 0::2] & 0xF
    hi = q[:, 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_int4(pk: np.ndarray) -> np.ndarray:
    pk = np.asarray(pk, dtype=np.uint8).astype(np.int64)
    lo = pk & 0xF
    hi = pk >> 4
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((pk.shape[0], pk.shape[1] * 2), dtype=np.int8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def hadamard_quant_act(x: np.ndarray, gamma=None, eps: float = DEFAULT_EPS, had_block: int = 0):
    """H-BitLinear activation path.  Returns (packed int4, s_x, codes, t)."""
    x = np.asarray(x, dtype=np.float32)
    b = had_block or default_had_block(x.shape[-1])
    y, _ = rms_norm(x, gamma, eps)
    t = hadamard_transform(y, b)
    q, s = absmax_quantize(t, 7, -8)
    return pack_int4(q), s, q, t


# ---------------------------------------------------------------------------
# integer product and dequantisation [P4 계산 패러다임, 양자화 메커니즘; P5]
# ---------------------------------------------------------------------------

def int_matmul(qx: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k qx[m, k] * qw[n, k], exact in int64, checked to fit int32."""
    acc = np.asarray(qx, dtype=np.int64) @ np.asarray(qw, dtype=np.int64).T
    assert np.all(np.abs(acc) < 2 ** 31)
    return acc.astype(np.int32)


def dequantize(acc: np.ndarray, s_x: np.ndarray, s_w) -> np.ndarray:
    """y = float(acc) * ((1/s_x) * (1/s_w)) in fp32 (|acc| < 2**24 converts exactly)."""
    acc = np.asarray(acc, dtype=np.int32)
    assert np.all(np.abs(acc) < 2 ** 24)
    dq = (F32(1.0) / np.asarray(s_x, dtype=np.float32)) * (F32(1.0) / F32(s_w))
    return acc.astype(np.float32) * dq[:, None]


def dequantize_f64(acc: np.ndarray, s_x: np.ndarray, s_w) -> np.ndarray:
    """The same rescale in float64: acc / (s_x * s_w)."""
    return np.asarray(acc, dtype=np.float64) / (
        np.asarray(s_x, dtype=np.float64)[:, None] * float(s_w))


def linear(qx: np.ndarray, s_x: np.ndarray, qw: np.ndarray, s_w):
    """BitLinear product on codes: returns (acc int32, y fp32)."""
    acc = int_matmul(qx, qw)
    return acc, dequantize(acc, s_x, s_w)


def fake_quant_matmul_f64(qx, s_x, qw, s_w) -> np.ndarray:
    """Float64 matmul of the dequantised operands (q_x / s_x) @ (q_w / s_w)^T."""
    a = np.asarray(qx, dtype=np.float64) / np.asarray(s_x, dtype=np.float64)[:, None]
    b = np.asarray(qw, dtype=np.float64) / float(s_w)
    return a @ b.T


def bf16_round(y: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(y, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def bitlinear(x: np.ndarray, qw: np.ndarray, s_w, act_bits: int = 8, gamma=None,
              eps: float = DEFAULT_EPS, had_block: int = 0):
    """Whole BitLinear forward on fp32 input x and ternary codes qw.

    act_bits = 8: RMSNorm + int8; act_bits = 4: RMSNorm + Hadamard + int4.
    Returns dict(codes, s_x, acc, y).
    """
    if act_bits == 8:
        q, s = quant_act(x, gamma, eps)
    else:
        _, s, q, _ = hadamard_quant_act(x, gamma, eps, had_block)
    acc, y = linear(q, s, qw, s_w)
    return dict(codes=q, s_x=s, acc=acc, y=y)


# ---------------------------------------------------------------------------
# stacked layer chain [P2 주요 아키텍처 혁신 (squared ReLU, no bias), P1 방법론]
# ---------------------------------------------------------------------------

def squared_relu_glu(gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    """a = relu(gate)^2 * up, fp32: (g * g) * up with g = max(gate, 0)."""
    g = np.maximum(np.asarray(gate, dtype=np.float32), F32(0.0))
    return (g * g) * np.asarray(up, dtype=np.float32)


def chain_layer(x: np.ndarray, layer: dict, eps: float = DEFAULT_EPS) -> np.ndarray:
    """One layer of the BitLinear chain; layer[name] = (codes, s_w).

    Q/K/V/up/gate use int8 activations, O and down are H-BitLinear (int4).
    The attention core is outside BitLinear; over a context of one token it
    returns V, so O's input is V's output.  Residual adds are fp32.
    """
    x = np.asarray(x, dtype=np.float32)
    qx, sx = quant_act(x, None, eps)
    _, q = linear(qx, sx, *layer["q"])
    _, k = linear(qx, sx, *layer["k"])
    _, v = linear(qx, sx, *layer["v"])
    _, so, co, _ = hadamard_quant_act(v, None, eps)
    _, o = linear(co, so, *layer["o"])
    h = x + o
    qh, sh = quant_act(h, None, eps)
    _, up = linear(qh, sh, *layer["up"])
    _, gate = linear(qh, sh, *layer["gate"])
    a = squared_relu_glu(gate, up)
    _, sd, cd, _ = hadamard_quant_act(a, None, eps)
    _, d = linear(cd, sd, *layer["down"])
    return h + d


# ---------------------------------------------------------------------------
# attention core of the stacked layer [P2 주요 아키텍처 혁신: rotary position
# embedding; the BitLinear layers are the linear layers of a transformer's
# attention and FFN blocks, P4 BitNet 아키텍처]
#
# Plain float64 definitions (the pages fix no precision for this part):
#   RoPE: in each head of width d, the pair (x[2i], x[2i+1]) of a token at
#   position p turns by the angle p * theta_i, theta_i = 10000^(-2i/d) (the
#   rotary embedding's own pairing and base; the pages name the method only);
#   attention: per head, softmax(q k^T / sqrt(d)) v over the keys a query may
#   see (its own position and the earlier ones).
# ---------------------------------------------------------------------------

ROPE_BASE = 10000.0


def rope_inv_freq(head_dim: int, base: float = ROPE_BASE) -> np.ndarray:
    """theta_i = base^(-2i/d) for i < d/2, float64."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return base ** (-2.0 * i / head_dim)


def rope_f64(x: np.ndarray, positions, heads: int, base: float = ROPE_BASE) -> np.ndarray:
    """Rotary position embedding of rows x [M, heads*d] at `positions` [M], float64:
    (a, b) = (x[2i], x[2i+1]) -> (a cos t - b sin t, a sin t + b cos t), t = p * theta_i."""
    x = np.asarray(x, dtype=np.float64)
    M, HD = x.shape
    d = HD // heads
    ang = np.asarray(positions, dtype=np.float64)[:, None] * rope_inv_freq(d, base)[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    v = x.reshape(M, heads, d // 2, 2)
    a, b = v[..., 0], v[..., 1]
    out = np.empty_like(v)
    out[..., 0] = a * c - b * s
    out[..., 1] = a * s + b * c
    return out.reshape(M, HD)


def attention_weights_f64(q: np.ndarray, k: np.ndarray, visible: np.ndarray) -> np.ndarray:
    """Softmax weights of one head: p[i, j] = exp(s_ij - max_j s_ij) / sum_j(...) over
    the visible keys, s_ij = (q_i . k_j) / sqrt(d); invisible keys get weight 0."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    d = q.shape[-1]
    s = (q @ k.T) / math.sqrt(d)
    s = np.where(visible, s, -np.inf)
    m = np.max(s, axis=-1, keepdims=True)
    e = np.where(visible, np.exp(s - m), 0.0)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention_f64(q: np.ndarray, k: np.ndarray, v: np.ndarray, heads: int, visible: np.ndarray) -> np.ndarray:
    """Multi-head softmax attention, float64.  q [Mq, heads*d], k and v [Mk, heads*d],
    visible [Mq, Mk] boolean.  Returns [Mq, heads*d]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    d = q.shape[-1] // heads
    out = np.empty((q.shape[0], heads * d), dtype=np.float64)
    for h in range(heads):
        sl = slice(h * d, (h + 1) * d)
        out[:, sl] = attention_weights_f64(q[:, sl], k[:, sl], visible) @ v[:, sl]
    return out


def causal_mask(n_query: int, n_key: int, first_query_pos: int) -> np.ndarray:
    """Query r sits at position first_query_pos + r and sees keys 0 .. its own position."""
    qpos = first_query_pos + np.arange(n_query)[:, None]
    return np.arange(n_key)[None, :] <= qpos


def chain_layer_attention(x: np.ndarray, layer: dict, k_cache: np.ndarray, v_cache: np.ndarray, t0: int,
                          heads: int = 16, eps: float = DEFAULT_EPS) -> np.ndarray:
    """One stacked layer with the attention core.  x [B*L, hidden] fp32 holds B
    sequences of L tokens at positions t0 .. t0+L-1; k_cache, v_cache
    [B, T_cap, hidden] float64 receive this step's rotated keys and values.
    The attention output enters the O projection's quantiser as fp32.  With one
    token per sequence at position 0 this is chain_layer (the one-token context)."""
    x = np.asarray(x, dtype=np.float32)
    B = k_cache.shape[0]
    L = x.shape[0] // B
    qx, sx = quant_act(x, None, eps)
    _, q = linear(qx, sx, *layer["q"])
    _, k = linear(qx, sx, *layer["k"])
    _, v = linear(qx, sx, *layer["v"])
    pos = np.tile(t0 + np.arange(L), B)
    q_r = rope_f64(q, pos, heads)
    k_r = rope_f64(k, pos, heads)
    att = np.empty(q.shape, dtype=np.float64)
    for b in range(B):
        rows = slice(b * L, (b + 1) * L)
        k_cache[b, t0:t0 + L] = k_r[rows]
        v_cache[b, t0:t0 + L] = v[rows]
        att[rows] = attention_f64(q_r[rows], k_cache[b, :t0 + L], v_cache[b, :t0 + L], heads,
                                  causal_mask(L, t0 + L, t0))
    _, so, co, _ = hadamard_quant_act(att.astype(np.float32), None, eps)
    _, o = linear(co, so, *layer["o"])
    h = x + o
    qh, sh = quant_act(h, None, eps)
    _, up = linear(qh, sh, *layer["up"])
    _, gate = linear(qh, sh, *layer["gate"])
    a = squared_relu_glu(gate, up)
    _, sd, cd, _ = hadamard_quant_act(a, None, eps)
    _, d = linear(cd, sd, *layer["down"])
    return h + d
