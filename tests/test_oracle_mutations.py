"""Plant plausible mistakes in the oracle (on the CPU) and show the pins catch them.

Each mutation swaps one oracle function for a wrong variant — a dropped term,
a wrong sign, index or constant, a transposed operand — and at least one
check of tests/test_oracle_pins.py must then fail.
"""
import math

import numpy as np
import pytest

from oracle import bitnet_oracle as O
import test_oracle_pins as pins

F32 = np.float32
_orig = {name: getattr(O, name) for name in dir(O) if callable(getattr(O, name))}


def _absmax_128(y, qmax, qmin):
    return _orig["absmax_quantize"](y, qmax + 1 if qmax == 127 else qmax, qmin)


def _absmax_no_rint(y, qmax, qmin):
    y = np.asarray(y, np.float32)
    s = F32(qmax) / np.maximum(np.max(np.abs(y), axis=-1), O.SCALE_FLOOR)
    return np.clip(np.trunc(y * s[..., None]), qmin, qmax).astype(np.int8), s


def _scale_is_mean(w):
    mean, _ = _orig["weight_scale"](w)
    return mean, F32(mean)


def _scale_absmax(w):
    m = F32(np.max(np.abs(w)))
    return m, F32(1.0) / m


def _sum_drops_last(w):
    return _orig["exact_sum_abs"](np.asarray(w).ravel()[:-1])


def _fwht_wrong_sign(y, block):
    y = np.asarray(y, np.float32)
    M, K = y.shape
    u = y.reshape(M, K // block, block)
    h = 1
    while h < block:
        v = u.reshape(M, K // block, block // (2 * h), 2, h)
        a, c = v[..., 0, :], v[..., 1, :]
        u = np.stack([a + c, c - a], axis=-2).reshape(M, K // block, block)
        h *= 2
    return u.reshape(M, K)


def _fwht_adjacent_only(y, block):
    y = np.asarray(y, np.float32)
    M, K = y.shape
    u = y.reshape(M, K // block, block)
    for _ in range(int(np.log2(block))):
        v = u.reshape(M, K // block, block // 2, 2)
        a, c = v[..., 0], v[..., 1]
        u = np.stack([a + c, a - c], axis=-1).reshape(M, K // block, block)
    return u.reshape(M, K)


def _no_norm_const(block):
    return F32(1.0)


def _pack_transposed(q):
    q = np.asarray(q, np.int8)
    N, K = q.shape
    f = (q.astype(np.int64) & 3).reshape(N, K // 16, 4, 4)
    word = np.zeros((N, K // 16), np.uint64)
    for j in range(4):
        for i in range(4):
            word |= (f[:, :, j, i] << (8 * j + 2 * i)).astype(np.uint64)
    return np.ascontiguousarray(word.astype("<u4")).view(np.uint8).reshape(N, K // 4)


def _pack_int4_swapped(q):
    q = np.asarray(q, np.int8).astype(np.int64)
    return ((q[:, 1::2] & 0xF) | ((q[:, 0::2] & 0xF) << 4)).astype(np.uint8)


def _sequential_sum(v):
    v = np.asarray(v, np.float32)
    acc = np.zeros(v.shape[:-1], np.float32)
    for k in range(v.shape[-1]):
        acc = acc + v[..., k]
    return acc


def _rms_no_eps(x, gamma=None, eps=O.DEFAULT_EPS):
    return _orig["rms_norm"](x, gamma, 0.0)


def _rms_mean_of_abs(x, gamma=None, eps=O.DEFAULT_EPS):
    x = np.asarray(x, np.float32)
    ms = O.pairwise_sum_f32(np.abs(x)) / F32(x.shape[-1])
    r = F32(1.0) / np.sqrt(ms + F32(eps))
    y = x * r[..., None]
    return (y * gamma if gamma is not None else y), r


def _matmul_drop_last_k(qx, qw):
    return _orig["int_matmul"](np.asarray(qx)[:, :-1], np.asarray(qw)[:, :-1])


def _dequant_times(acc, s_x, s_w):
    return np.asarray(acc, np.float32) * (np.asarray(s_x, np.float32)[:, None] * F32(s_w))


def _ternarize_no_clamp(w, s_w):
    return np.rint(np.asarray(w, np.float32) * F32(s_w)).astype(np.int8)


def _trit5_digits_reversed(q):
    """Most significant digit first: a plausible slip in the base-3 order."""
    pk = _orig["pack_trit5"](q).astype(np.int64)
    out = np.zeros_like(pk)
    for i in range(5):
        out = out * 3 + pk % 3
        pk = pk // 3
    return out.astype(np.uint8)


def _trit5_offset_minus(q):
    """Digits w mod 3 instead of w + 1 (-1 -> 2, 0 -> 0, +1 -> 1)."""
    q = np.asarray(q, np.int64)
    N, K = q.shape
    R = O.trit5_row_bytes(K)
    d = np.zeros((N, R * 5), np.int64)
    d[:, :K] = q % 3
    d = d.reshape(N, R, 5)
    return sum(d[:, :, i] * 3 ** i for i in range(5)).astype(np.uint8)


def _glu_no_square(gate, up):
    """relu(gate) * up: the square dropped."""
    return np.maximum(np.asarray(gate, np.float32), F32(0.0)) * np.asarray(up, np.float32)


def _glu_gate_up_swapped(gate, up):
    return _orig["squared_relu_glu"](up, gate)


def _glu_abs_instead_of_relu(gate, up):
    g = np.abs(np.asarray(gate, np.float32))
    return (g * g) * np.asarray(up, np.float32)


def _chain_o_from_q(x, layer, eps=O.DEFAULT_EPS):
    """The O projection fed from Q instead of V."""
    swapped = dict(layer)
    swapped["v"] = layer["q"]
    return _orig["chain_layer"](x, swapped, eps)


def _chain_no_attention_residual(x, layer, eps=O.DEFAULT_EPS):
    """The attention residual dropped: the FFN runs on o instead of h = x + o."""
    x = np.asarray(x, np.float32)
    qx, sx = O.quant_act(x, None, eps)
    _, v = O.linear(qx, sx, *layer["v"])
    _, so, co, _ = O.hadamard_quant_act(v, None, eps)
    _, o = O.linear(co, so, *layer["o"])
    h = o
    qh, sh = O.quant_act(h, None, eps)
    _, up = O.linear(qh, sh, *layer["up"])
    _, gate = O.linear(qh, sh, *layer["gate"])
    _, sd, cd, _ = O.hadamard_quant_act(O.squared_relu_glu(gate, up), None, eps)
    _, d = O.linear(cd, sd, *layer["down"])
    return x + o + d


def _bf16_truncate(y):
    return (np.ascontiguousarray(y, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _bf16_ties_away(y):
    u = np.ascontiguousarray(y, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x8000) >> 16).astype(np.uint16)


def _rope_half_pairs(x, positions, heads, base=O.ROPE_BASE):
    """Pairs (i, i + d/2) instead of (2i, 2i + 1)."""
    x = np.asarray(x, np.float64)
    M, HD = x.shape
    d = HD // heads
    perm = np.concatenate([np.arange(0, d, 2), np.arange(1, d, 2)])
    inv = np.argsort(perm)
    xs = x.reshape(M, heads, d)[:, :, inv].reshape(M, HD)
    y = _orig["rope_f64"](xs, positions, heads, base)
    return y.reshape(M, heads, d)[:, :, perm].reshape(M, HD)


def _rope_turns_backwards(x, positions, heads, base=O.ROPE_BASE):
    return _orig["rope_f64"](x, -np.asarray(positions), heads, base)


def _rope_base_1e4_per_pair(head_dim, base=O.ROPE_BASE):
    i = np.arange(head_dim // 2, dtype=np.float64)
    return base ** (-i / head_dim)


def _attn_no_scale(q, k, visible):
    d = np.asarray(q).shape[-1]
    return _orig["attention_weights_f64"](np.asarray(q, np.float64) * math.sqrt(d), k, visible)


def _attn_scale_1_over_d(q, k, visible):
    d = np.asarray(q).shape[-1]
    return _orig["attention_weights_f64"](np.asarray(q, np.float64) / math.sqrt(d), k, visible)


def _attn_sees_future(q, k, visible):
    return _orig["attention_weights_f64"](q, k, np.ones_like(visible))


def _attn_normalises_keys(q, k, visible):
    """Softmax taken over the queries instead of the keys."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    s = np.where(visible, (q @ k.T) / math.sqrt(q.shape[-1]), -np.inf)
    e = np.where(visible, np.exp(s - np.max(s, axis=0, keepdims=True)), 0.0)
    return e / np.sum(e, axis=0, keepdims=True)


MUTATIONS = {
    "absmax_numerator_128": ("absmax_quantize", _absmax_128),
    "absmax_truncates": ("absmax_quantize", _absmax_no_rint),
    "weight_scale_is_mean": ("weight_scale", _scale_is_mean),
    "weight_scale_absmax": ("weight_scale", _scale_absmax),
    "weight_sum_drops_term": ("exact_sum_abs", _sum_drops_last),
    "ternarize_no_clamp": ("ternarize", _ternarize_no_clamp),
    "fwht_wrong_sign": ("fwht_f32", _fwht_wrong_sign),
    "fwht_wrong_pairs": ("fwht_f32", _fwht_adjacent_only),
    "hadamard_unnormalised": ("hadamard_norm_const", _no_norm_const),
    "pack_ternary_transposed": ("pack_ternary", _pack_transposed),
    "pack_int4_nibbles_swapped": ("pack_int4", _pack_int4_swapped),
    "sum_sequential": ("pairwise_sum_f32", _sequential_sum),
    "rms_no_eps": ("rms_norm", _rms_no_eps),
    "rms_mean_abs": ("rms_norm", _rms_mean_of_abs),
    "matmul_drops_term": ("int_matmul", _matmul_drop_last_k),
    "dequant_multiplies": ("dequantize", _dequant_times),
    "trit5_digits_reversed": ("pack_trit5", _trit5_digits_reversed),
    "trit5_digit_offset": ("pack_trit5", _trit5_offset_minus),
    "glu_no_square": ("squared_relu_glu", _glu_no_square),
    "glu_gate_up_swapped": ("squared_relu_glu", _glu_gate_up_swapped),
    "glu_abs_not_relu": ("squared_relu_glu", _glu_abs_instead_of_relu),
    "chain_o_from_q": ("chain_layer", _chain_o_from_q),
    "chain_drops_residual": ("chain_layer", _chain_no_attention_residual),
    "bf16_truncates": ("bf16_round", _bf16_truncate),
    "bf16_ties_away": ("bf16_round", _bf16_ties_away),
    "rope_half_pairs": ("rope_f64", _rope_half_pairs),
    "rope_backwards": ("rope_f64", _rope_turns_backwards),
    "rope_wrong_frequencies": ("rope_inv_freq", _rope_base_1e4_per_pair),
    "attention_unscaled": ("attention_weights_f64", _attn_no_scale),
    "attention_scale_1_over_d": ("attention_weights_f64", _attn_scale_1_over_d),
    "attention_sees_future": ("attention_weights_f64", _attn_sees_future),
    "attention_softmax_over_queries": ("attention_weights_f64", _attn_normalises_keys),
}


@pytest.mark.filterwarnings("ignore::RuntimeWarning")      # planted mistakes may divide by zero
@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for check in pins.CHECKS:
        try:
            check()
        except Exception:
            caught.append(check.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
