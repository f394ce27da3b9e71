"""Pins of the CPU oracle to facts it does not compute itself.

Each check is a plain function so that tests/test_oracle_mutations.py can
plant a mistake in the oracle and show that some check catches it.  Sources
are the pages' worked values (tests/golden/), closed forms, library routines
for special cases (scipy's Sylvester Hadamard, math.fsum, Python integers and
fractions) and brute force on tiny inputs.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import bitnet_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line)
    return rows


def _kv(name):
    out = {}
    for row in _golden(name):
        k, *v = row.split()
        out[k] = v
    return out


# ---------------------------------------------------------------- absmax -----

def check_absmax_worked_example():
    g = _kv("absmax_worked_example.txt")
    amax = float(g["absmax"][0])
    printed = float(g["factor_printed"][0])
    res = float(g["factor_printed_resolution"][0])
    vals = np.array([[amax, -2.1, 1.0, 0.3, -amax * 0.999, 0.0]], dtype=np.float32)
    q, s = O.absmax_quantize(vals, 127, -128)
    assert abs(float(s[0]) - printed) <= res, (s, printed)
    assert q[0, 0] == 127 and q[0, 5] == 0
    # every other code is round(v * 127 / 5.4) in exact rational arithmetic
    # (no value here sits within 1e-3 of a rounding tie)
    factor = Fraction(int(g["numerator"][0])) / Fraction(amax)
    for j, v in enumerate(vals[0]):
        exact = Fraction(float(v)) * factor
        assert abs(abs(exact - round(exact)) - Fraction(1, 2)) > Fraction(1, 1000)
        assert q[0, j] == round(exact), (j, v, q[0, j], float(exact))
    # dequantisation divides by the factor: error at most half a step
    deq = q.astype(np.float64) / float(s[0])
    assert np.all(np.abs(deq - vals.astype(np.float64)) <= 0.5 / float(s[0]) + 1e-9)


def check_int8_range_and_peak():
    rng = np.random.default_rng(3)
    y = (rng.standard_normal((64, 300)) * rng.uniform(0.01, 50, size=(64, 1))).astype(np.float32)
    q, s = O.absmax_quantize(y, 127, -128)
    assert q.min() >= -127 and q.max() <= 127        # |y*s| <= 127, so -128 never appears
    peak = np.abs(y).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(64), peak]) == 127)
    assert np.all(np.sign(q[np.arange(64), peak]) == np.sign(y[np.arange(64), peak]))
    # codes are nearest integers of y * 127 / max|y| (checked in float64)
    ref = y.astype(np.float64) * (127.0 / np.abs(y.astype(np.float64)).max(axis=1, keepdims=True))
    assert np.all(np.abs(q - ref) <= 0.5 + 1e-4)


def check_zero_row_floor():
    q, s = O.absmax_quantize(np.zeros((2, 64), np.float32), 127, -128)
    assert np.all(q == 0) and np.allclose(s, 127.0 / 1e-5, rtol=1e-6)


# ---------------------------------------------------------------- weights ----

def check_exact_sum_abs():
    rng = np.random.default_rng(5)
    w = (rng.standard_normal(20000) * np.exp2(rng.integers(-60, 40, size=20000))).astype(np.float32)
    w[:5] = [1e-45, -3e-40, 2.0 ** 100, -(2.0 ** -120), 0.0]     # subnormals, extremes
    assert O.exact_sum_abs(w) == math.fsum(abs(float(v)) for v in w)
    # brute force with Python integers in units of 2**-149 (the fp32 subnormal step)
    tiny = np.array([1.0, 2.0 ** -30, 2.0 ** -30, -3.5, 1e-45], dtype=np.float32)
    units = sum(int(abs(float(v)) * 2 ** 149) for v in tiny)
    assert O.exact_sum_abs(tiny) == float(Fraction(units, 2 ** 149))
    # integer-valued magnitudes: every term moves the exact sum
    ints = np.random.default_rng(6).integers(-1000, 1000, size=4097).astype(np.float32)
    assert O.exact_sum_abs(ints) == float(sum(abs(int(v)) for v in ints))
    const = np.full((64, 48), -0.375, np.float32)
    assert O.weight_scale(const)[0] == np.float32(0.375)


def check_absmean_zero_fraction():
    """For N(0, sigma) weights the zero band is |w| < m/2 with m = sigma*sqrt(2/pi),
    so P(0) = erf(1/(2*sqrt(pi))) = 0.3101 and P(+1) = P(-1) = 0.3449."""
    sigma = 0.02
    n = 1 << 20
    w = (np.random.default_rng(11).standard_normal(n) * sigma).astype(np.float32).reshape(1024, 1024)
    mean, s_w = O.weight_scale(w)
    assert abs(float(mean) - sigma * math.sqrt(2 / math.pi)) < 5 * sigma * 0.6 / math.sqrt(n)
    assert abs(float(s_w) * float(mean) - 1.0) < 1e-6
    q = O.ternarize(w, s_w)
    assert set(np.unique(q).tolist()) <= {-1, 0, 1}
    p0 = math.erf(1.0 / (2.0 * math.sqrt(math.pi)))
    sd = math.sqrt(p0 * (1 - p0) / n)
    assert abs(float(np.mean(q == 0)) - p0) < 5 * sd
    assert abs(float(np.mean(q == 1)) - (1 - p0) / 2) < 5 * sd
    assert abs(float(np.mean(q == -1)) - (1 - p0) / 2) < 5 * sd


def check_ternarize_thresholds():
    s_w = np.float32(4.0)                  # mean |W| = 0.25
    w = np.array([[0.1, 0.12, 0.125, 0.126, -0.125, -0.126, 0.375, 0.9, -5.0, 0.0]], np.float32)
    q = O.ternarize(w, s_w)
    # w*4 = .4 .48 .5 .504 -.5 -.504 1.5 3.6 -20 0 -> rint (half to even) then clamp
    assert q.tolist() == [[0, 0, 0, 1, 0, -1, 1, 1, -1, 0]]


def check_pack_layout_golden():
    g = _kv("ternary_pack_layout.txt")
    w = np.array([[int(v) for v in g["weights"]]], dtype=np.int8)
    expect = [int(b, 16) for b in g["bytes"]]
    pk = O.pack_ternary(w)
    assert pk.tolist() == [expect]
    assert O.unpack_ternary(pk).tolist() == w.tolist()
    rng = np.random.default_rng(2)
    q = rng.integers(-1, 2, size=(7, 64)).astype(np.int8)
    assert np.array_equal(O.unpack_ternary(O.pack_ternary(q)), q)
    assert O.pack_ternary(q).shape == (7, 16)


def check_int4_pack_golden():
    g = _kv("int4_pack_layout.txt")
    codes = np.array([[int(v) for v in g["codes"]]], dtype=np.int8)
    expect = [int(b, 16) for b in g["bytes"]]
    assert O.pack_int4(codes).tolist() == [expect]
    assert O.unpack_int4(O.pack_int4(codes)).tolist() == codes.tolist()


def check_trit5_pack_golden():
    rows = _golden("trit5_pack_layout.txt")
    g = {r.split()[0]: r.split()[1:] for r in rows if not r.startswith("single")}
    w = np.array([[int(v) for v in g["weights"]]], dtype=np.int8)
    pk = O.pack_trit5(w)
    assert pk.tolist() == [[int(b) for b in g["bytes"]]]
    assert O.unpack_trit5(pk, w.shape[1]).tolist() == w.tolist()
    for r in rows:
        if r.startswith("single"):
            *ws, b = [int(v) for v in r.split()[1:]]
            assert O.pack_trit5(np.array([ws], np.int8))[0, 0] == b


def check_trit5_is_a_bijection_on_five_weights():
    """All 3^5 five-weight groups map to the 243 distinct bytes 0..242 and back."""
    combos = np.array(np.meshgrid(*[[-1, 0, 1]] * 5, indexing="ij")).reshape(5, -1).T.astype(np.int8)
    b = O.pack_trit5(combos)[:, 0]
    assert sorted(b.tolist()) == list(range(243))
    assert np.array_equal(O.unpack_trit5(O.pack_trit5(combos), 5), combos)


def check_trit5_agrees_with_two_bit_packing():
    """Both storage formats hold the same weights; 1.6 bits per weight at K = 2560."""
    q = np.random.default_rng(5).integers(-1, 2, size=(9, 2560)).astype(np.int8)
    assert np.array_equal(O.unpack_trit5(O.pack_trit5(q), 2560), O.unpack_ternary(O.pack_ternary(q)))
    assert O.pack_trit5(q).shape == (9, 512) and 8 * 512 / 2560 == 1.6
    assert O.trit5_row_bytes(37) == 16 and O.trit5_row_bytes(80) == 16 and O.trit5_row_bytes(81) == 32


def check_packing_ratio_llama3_8b():
    """8B -> 2.8B only if the linear weights are four per byte and the
    embedding and output head stay unpacked."""
    g = {k: float(v[0]) for k, v in _kv("llama3_8b_packing.txt").items()}
    h, L, f = int(g["hidden"]), int(g["layers"]), int(g["intermediate"])
    kv = int(g["kv_heads"] * g["head_dim"])
    shapes = [(h, h), (kv, h), (kv, h), (h, h), (f, h), (f, h), (h, f)]  # q k v o gate up down
    linear = L * sum(n * k for n, k in shapes)
    embed = 2 * int(g["vocab"]) * h
    before = linear + embed
    # bytes the packer produces per weight, measured on a small matrix
    per_weight = O.pack_ternary(np.zeros((16, 128), np.int8)).size / (16 * 128)
    after = linear * per_weight + embed
    assert abs(before - g["claimed_before"]) / g["claimed_before"] < 0.01
    assert abs(after - g["claimed_after"]) / g["claimed_after"] < 0.01
    assert abs(math.log2(3) - 1.58) < 0.005          # "1.58 bits" for three states


# ---------------------------------------------------------------- RMSNorm ----

def _sym(tok):
    u = 2.0 ** -24
    return {"1": 1.0, "u": u, "1+2u": 1.0 + 2 * u, "1+8u": 1.0 + 8 * u}[tok]


def check_pairwise_sum_golden():
    for row in _golden("pairwise_sum_cases.txt"):
        vals, expect = row.split(";")
        v = np.array([_sym(t) for t in vals.split()], dtype=np.float32)
        got = O.pairwise_sum_f32(v[None, :])[0]
        assert float(got) == _sym(expect.strip()), (row, float(got))
    # integer-valued inputs below 2**24 sum exactly in any order
    ints = np.random.default_rng(1).integers(-1000, 1000, size=(5, 777)).astype(np.float32)
    assert np.array_equal(O.pairwise_sum_f32(ints), ints.astype(np.int64).sum(axis=1).astype(np.float32))
    # accuracy bound against the correctly rounded sum
    v = np.random.default_rng(4).standard_normal((3, 5000)).astype(np.float32) ** 2
    for r in range(3):
        exact = math.fsum(float(t) for t in v[r])
        assert abs(float(O.pairwise_sum_f32(v[r:r + 1])[0]) - exact) <= 13 * 2.0 ** -24 * exact


def check_rms_norm():
    rng = np.random.default_rng(9)
    x = (rng.standard_normal((16, 2560)) * 3).astype(np.float32)
    y, r = O.rms_norm(x, None, 1e-6)
    x64 = x.astype(np.float64)
    r64 = 1.0 / np.sqrt(np.mean(x64 * x64, axis=1) + 1e-6)
    assert np.allclose(r, r64, rtol=2e-6, atol=0)
    assert np.allclose(y, x64 * r64[:, None], rtol=3e-6, atol=1e-30)
    ms = np.mean(x64 * x64, axis=1)
    assert np.allclose(np.mean(y.astype(np.float64) ** 2, axis=1), ms / (ms + 1e-6), rtol=1e-5)
    gamma = rng.uniform(0.5, 2.0, size=2560).astype(np.float32)
    yg, _ = O.rms_norm(x, gamma, 1e-6)
    assert np.allclose(yg, y.astype(np.float64) * gamma, rtol=1e-6)
    z, rz = O.rms_norm(np.zeros((1, 256), np.float32), None, 1e-6)
    assert np.all(z == 0) and abs(float(rz[0]) - 1000.0) < 1e-2


# ---------------------------------------------------------------- Hadamard ---

def check_hadamard_sylvester():
    from scipy.linalg import hadamard   # Sylvester construction
    rng = np.random.default_rng(12)
    for b in (2, 8, 64, 512):
        H = hadamard(b).astype(np.float64)
        assert np.array_equal(H @ H.T, b * np.eye(b))
        eye = np.eye(b, dtype=np.float32)
        assert np.array_equal(O.fwht_f32(eye, b), H.T.astype(np.float32))   # FWHT(e_i) = column i
        y = rng.standard_normal((3, b)).astype(np.float32)
        u = O.fwht_f32(y, b).astype(np.float64)
        ref = y.astype(np.float64) @ H.T
        tol = math.log2(b) * 2.0 ** -23 * np.abs(y).sum(axis=1, keepdims=True)
        assert np.all(np.abs(u - ref) <= tol)
        t = O.hadamard_transform(y, b).astype(np.float64)
        assert np.allclose(np.linalg.norm(t, axis=1), np.linalg.norm(y, axis=1), rtol=1e-5)
        c = np.ones((1, b), np.float32)
        tc = O.hadamard_transform(c, b)
        assert abs(float(tc[0, 0]) - math.sqrt(b)) < 1e-5 * math.sqrt(b) and np.all(tc[0, 1:] == 0)
        ints = rng.integers(-8, 8, size=(2, b)).astype(np.float32)
        assert np.array_equal(O.fwht_f32(O.fwht_f32(ints, b), b), b * ints)   # H H = b I
    # block-diagonal: K = 3 blocks of 64, each transformed on its own
    y = rng.standard_normal((2, 192)).astype(np.float32)
    u = O.fwht_f32(y, 64)
    for k in range(3):
        assert np.array_equal(u[:, 64 * k:64 * k + 64], O.fwht_f32(y[:, 64 * k:64 * k + 64], 64))
    assert O.default_had_block(8192) == 8192 and O.default_had_block(5632) == 512
    assert O.default_had_block(2048) == 2048


def check_int4_quant():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((32, 1024)).astype(np.float32)
    pk, s, q, t = O.hadamard_quant_act(x, None, 1e-6, 0)
    assert q.min() >= -8 and q.max() <= 7 and q.min() >= -7      # symmetric 7 never yields -8
    peak = np.abs(t).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(32), peak]) == 7)
    ref = t.astype(np.float64) * (7.0 / np.abs(t.astype(np.float64)).max(axis=1, keepdims=True))
    assert np.all(np.abs(q - ref) <= 0.5 + 1e-4)
    assert np.array_equal(O.unpack_int4(pk), q)


# ---------------------------------------------------------------- product ----

def check_int_matmul_brute_force():
    rng = np.random.default_rng(6)
    qx = rng.integers(-128, 128, size=(3, 16)).astype(np.int8)
    qw = rng.integers(-1, 2, size=(5, 16)).astype(np.int8)
    acc = O.int_matmul(qx, qw)
    for m in range(3):
        for n in range(5):
            assert acc[m, n] == sum(int(qx[m, k]) * int(qw[n, k]) for k in range(16))


def check_dequant_matches_fake_quant():
    rng = np.random.default_rng(7)
    qx = rng.integers(-127, 128, size=(8, 256)).astype(np.int8)
    qw = rng.integers(-1, 2, size=(32, 256)).astype(np.int8)
    s_x = rng.uniform(1, 100, size=8).astype(np.float32)
    s_w = np.float32(37.5)
    acc, y = O.linear(qx, s_x, qw, s_w)
    ref = O.fake_quant_matmul_f64(qx, s_x, qw, s_w)
    assert np.allclose(O.dequantize_f64(acc, s_x, s_w), ref, rtol=1e-12, atol=1e-12)
    nz = acc != 0
    assert np.max(np.abs(y[nz] - ref[nz]) / np.abs(ref[nz])) < 1e-6
    assert np.all(y[~nz] == 0) and np.all(np.abs(ref[~nz]) < 1e-12)


def check_tiny_bitlinear_end_to_end():
    """Tiny BitLinear: integer path equals the float64 fake-quant matmul, and
    both approximate the full-precision RMSNorm(x) @ W^T."""
    from bitlinear_bitnet_quant_b200 import workloads as wl
    c = wl.tiny()
    pk, s_w, qw = O.quantize_weights(c["w"])
    out = O.bitlinear(c["x"], qw, s_w)
    ref = O.fake_quant_matmul_f64(out["codes"], out["s_x"], qw, s_w)
    nz = out["acc"] != 0
    assert np.max(np.abs(out["y"][nz] - ref[nz]) / np.abs(ref[nz])) < 1e-6
    y, _ = O.rms_norm(c["x"])
    full = y.astype(np.float64) @ c["w"].astype(np.float64).T
    err = np.linalg.norm(ref - full) / np.linalg.norm(full)
    assert err < 0.75, err       # ternary weights: a coarse approximation, not garbage


def check_chain_zero_weights_is_identity():
    x = np.random.default_rng(8).standard_normal((4, 64)).astype(np.float32)
    z = lambda n, k: (np.zeros((n, k), np.int8), O.weight_scale(np.zeros((n, k), np.float32))[1])
    layer = {"q": z(64, 64), "k": z(64, 64), "v": z(64, 64), "o": z(64, 64),
             "up": z(128, 64), "gate": z(128, 64), "down": z(64, 128)}
    assert np.array_equal(O.chain_layer(x, layer), x)


def check_squared_relu_glu_golden():
    gate, up, want = [], [], []
    for row in _golden("squared_relu_glu_cases.txt"):
        lhs, rhs = row.split(";")
        g, u = lhs.split()
        gate.append(float(g))
        up.append(float(u))
        want.append(float(rhs))
    got = O.squared_relu_glu(np.array([gate], np.float32), np.array([up], np.float32))
    assert got.dtype == np.float32
    assert np.array_equal(got[0], np.array(want, np.float32)), (got, want)


def check_bf16_round_golden():
    src, want = [], []
    for row in _golden("bf16_rne_cases.txt"):
        a, b = row.split()
        src.append(int(a, 16))
        want.append(int(b, 16))
    got = O.bf16_round(np.array(src, np.uint32).view(np.float32))
    assert [int(v) for v in got] == want, [hex(int(v)) for v in got]


def _tiny_chain_layer():
    """The hand-built layer of tests/golden/chain_layer_tiny.txt: (codes, s_w = 1) per projection."""
    H = F = 16
    n = np.arange(16)
    z = lambda r, c: np.zeros((r, c), np.int8)
    wq, wk, wv, wo = z(H, H), z(H, H), z(H, H), z(H, H)
    wup, wgate, wdown = z(F, H), z(F, H), z(H, F)
    wq[:, 0] = np.where(n % 2 == 0, 1, -1)
    wk[:, 0] = np.where(n % 4 < 2, 1, -1)
    wv[:, 0] = 1
    wo[:, 1] = 1
    wo[:, 2] = 1
    wup[:, 0] = 1
    wgate[:, 0] = 1
    wgate[n % 2 == 1, 1] = 1
    wdown[:, 1] = np.where(n % 2 == 0, 1, -1)
    wdown[:8, 0] = 1
    one = np.float32(1.0)
    return {"q": (wq, one), "k": (wk, one), "v": (wv, one), "o": (wo, one),
            "up": (wup, one), "gate": (wgate, one), "down": (wdown, one)}


def check_chain_layer_tiny_golden():
    want = np.array([float(r.split()[1]) for r in _golden("chain_layer_tiny.txt")])
    x = np.ones((1, 16), np.float32)
    got = O.chain_layer(x, _tiny_chain_layer())
    assert got.shape == (1, 16) and got.dtype == np.float32
    assert np.max(np.abs(got[0] - want) / np.abs(want)) < 1e-5, (got, want)


# -------------------------------------------------------------- attention ----

def check_rope_golden():
    for row in _golden("rope_worked_example.txt"):
        lhs, rhs = row.split(";")
        *x, pos = lhs.split()
        want = np.array([float(v) for v in rhs.split()])
        got = O.rope_f64(np.array([[float(v) for v in x]]), [int(pos)], heads=1)
        assert np.max(np.abs(got[0] - want)) < 1e-12, (got, want)


def check_rope_is_a_rotation():
    """Each pair keeps its length; two rotated vectors' dot product depends only on
    the distance of their positions; position 0 is the identity (any head count)."""
    rng = np.random.default_rng(31)
    q = rng.standard_normal((1, 4 * 128))
    k = rng.standard_normal((1, 4 * 128))
    rq = O.rope_f64(q, [37], heads=4)
    pair = lambda a: np.sqrt((a.reshape(-1, 2) ** 2).sum(axis=1))
    assert np.allclose(pair(rq), pair(q), rtol=1e-13)
    dots = [float(O.rope_f64(q, [p + t], 4)[0] @ O.rope_f64(k, [s + t], 4)[0]) for p, s, t in
            ((9, 4, 0), (9, 4, 100), (105, 100, 0))]
    assert abs(dots[0] - dots[1]) < 1e-9 and abs(dots[0] - dots[2]) < 1e-9
    assert np.array_equal(O.rope_f64(q, [0], 4), q)


def check_attention_closed_form():
    """Two keys whose scaled scores are ln 3 and 0: weights 3/4 and 1/4 exactly
    (the scale is 1/sqrt(d), d = 4)."""
    a = 2.0 * math.log(3.0)               # q . k1 = 2 ln 3, divided by sqrt(4) = ln 3
    q = np.array([[1.0, 0, 0, 0]])
    k = np.array([[a, 0, 0, 0], [0, 0, 0, 0]])
    v = np.array([[4.0, 0, 0, 8], [0, 4, 0, -8]])
    out = O.attention_f64(q, k, v, heads=1, visible=np.ones((1, 2), bool))
    assert np.max(np.abs(out - np.array([[3.0, 1.0, 0.0, 4.0]]))) < 1e-12, out


def check_attention_brute_force():
    """Two heads, three queries, causal: explicit loops with math.exp."""
    rng = np.random.default_rng(32)
    H, d, n = 2, 8, 3
    q, k, v = (rng.standard_normal((n, H * d)) for _ in range(3))
    mask = O.causal_mask(n, n, 0)
    got = O.attention_f64(q, k, v, H, mask)
    for h in range(H):
        sl = slice(h * d, (h + 1) * d)
        for i in range(n):
            sc = [sum(q[i, sl][t] * k[j, sl][t] for t in range(d)) / math.sqrt(d) for j in range(i + 1)]
            mx = max(sc)
            w = [math.exp(x - mx) for x in sc]
            tot = sum(w)
            ref = [sum(w[j] * v[j, sl][t] for j in range(i + 1)) / tot for t in range(d)]
            assert np.max(np.abs(got[i, sl] - np.array(ref))) < 1e-12


def check_attention_special_cases():
    rng = np.random.default_rng(33)
    q, k, v = (rng.standard_normal((5, 64)) for _ in range(3))
    # one visible key: the output is that key's value (the one-token context)
    one = O.attention_f64(q[:1], k[:1], v[:1], 2, np.ones((1, 1), bool))
    assert np.allclose(one, v[:1], rtol=0, atol=1e-15)
    # a zero query scores every key alike: the mean of the visible values
    z = O.attention_f64(np.zeros((1, 64)), k, v, 2, np.ones((1, 5), bool))
    assert np.allclose(z[0], v.mean(axis=0), atol=1e-14)
    # softmax weights are non-negative and sum to one over the visible keys
    w = O.attention_weights_f64(q[:, :32], k[:, :32], O.causal_mask(5, 5, 0))
    assert np.all(w >= 0) and np.allclose(w.sum(axis=1), 1.0, atol=1e-14)
    assert np.all(w[np.triu_indices(5, 1)] == 0)
    # causality: a later key or value cannot change an earlier output
    k2, v2 = k.copy(), v.copy()
    k2[4] += 3.0
    v2[4] -= 2.0
    m = O.causal_mask(5, 5, 0)
    assert np.array_equal(O.attention_f64(q, k, v, 2, m)[:4], O.attention_f64(q, k2, v2, 2, m)[:4])
    # a query at position 2 of a cached context sees keys 0..2
    assert np.array_equal(O.causal_mask(1, 5, 2)[0], [True, True, True, False, False])


def check_layer_attention_reduces_to_one_token_context():
    """A layer whose every sequence holds one token at position 0 attends over that
    token alone, so it equals the one-token-context layer bit for bit; with more
    tokens the attention changes the output."""
    layer = _tiny_chain_layer()
    x = np.random.default_rng(34).standard_normal((3, 16)).astype(np.float32)
    kc, vc = np.zeros((3, 4, 16)), np.zeros((3, 4, 16))
    got = O.chain_layer_attention(x, layer, kc, vc, 0, heads=1)
    assert np.array_equal(got, O.chain_layer(x, layer))
    rng = np.random.default_rng(35)
    rand = {n: (rng.integers(-1, 2, size=w.shape).astype(np.int8), np.float32(rng.uniform(20, 60)))
            for n, (w, _) in layer.items()}
    kc, vc = np.zeros((3, 4, 16)), np.zeros((3, 4, 16))
    assert np.array_equal(O.chain_layer_attention(x, rand, kc, vc, 0, heads=2), O.chain_layer(x, rand))
    kc, vc = np.zeros((1, 4, 16)), np.zeros((1, 4, 16))
    seq = O.chain_layer_attention(x, rand, kc, vc, 0, heads=2)       # one sequence of three tokens
    ref = O.chain_layer(x, rand)
    assert np.array_equal(seq[0], ref[0]) and not np.array_equal(seq[1:], ref[1:])


CHECKS = [v for k, v in sorted(globals().items()) if k.startswith("check_")]


@pytest.mark.parametrize("check", CHECKS, ids=[c.__name__ for c in CHECKS])
def test_pin(check):
    check()
