"""numpy-facing binding of the plain C++ oracle (bitnet_oracle_ref.cpp).

TEST INFRASTRUCTURE: only tests/ (which hold the numpy oracle and the C++ one
to the same bits) and bench.py's CPU-baseline leg use it.  build() compiles the library with g++ in-tree
(oracle/_build), with -ffp-contract=off, no fast-math, and OpenMP over tokens
and output rows (which changes no result).
"""
from __future__ import annotations

import ctypes
import os
import shutil
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bitnet_oracle_ref.cpp")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "libbitnet_oracle_ref.so")
FLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared"]

_lib = None


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        raise RuntimeError("a C++ compiler (g++) is needed for the C++ oracle")
    os.makedirs(OUT_DIR, exist_ok=True)
    subprocess.run([cxx, *FLAGS, SRC, "-o", LIB], check=True)
    return LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I64, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
        sig = {
            "oc_threads": (ctypes.c_int, []),
            "oc_exact_sum_abs": (ctypes.c_double, [P, I64]),
            "oc_weight_scale": (None, [P, I64, P, P]),
            "oc_ternarize": (None, [P, I64, F, P]),
            "oc_pack_ternary": (None, [P, I64, I64, P]),
            "oc_pack_trit5": (None, [P, I64, I64, I64, P]),
            "oc_rms_norm": (None, [P, I64, I64, P, F, P, P]),
            "oc_absmax_quantize": (None, [P, I64, I64, ctypes.c_int, ctypes.c_int, P, P]),
            "oc_hadamard": (None, [P, I64, I64, I64]),
            "oc_pack_int4": (None, [P, I64, I64, P]),
            "oc_int_matmul": (None, [P, P, I64, I64, I64, P]),
            "oc_dequantize": (None, [P, I64, I64, P, F, P]),
            "oc_relu2_glu": (None, [P, P, I64, P]),
            "oc_add": (None, [P, P, I64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def threads() -> int:
    return int(lib().oc_threads())


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def exact_sum_abs(w) -> float:
    w = _c(w, np.float32)
    return lib().oc_exact_sum_abs(_p(w), w.size)


def weight_scale(w):
    w = _c(w, np.float32)
    mean, s = np.zeros(1, np.float32), np.zeros(1, np.float32)
    lib().oc_weight_scale(_p(w), w.size, _p(mean), _p(s))
    return mean[0], s[0]


def quantize_weights(w):
    w = _c(w, np.float32)
    _, s_w = weight_scale(w)
    q = np.empty(w.shape, np.int8)
    lib().oc_ternarize(_p(w), w.size, float(s_w), _p(q))
    pk = np.empty((w.shape[0], w.shape[1] // 4), np.uint8)
    lib().oc_pack_ternary(_p(q), w.shape[0], w.shape[1], _p(pk))
    return pk, s_w, q


def pack_trit5(q, row_bytes: int):
    q = _c(q, np.int8)
    out = np.empty((q.shape[0], row_bytes), np.uint8)
    lib().oc_pack_trit5(_p(q), q.shape[0], q.shape[1], row_bytes, _p(out))
    return out


def rms_norm(x, gamma=None, eps: float = 1e-6):
    x = _c(x, np.float32)
    g = None if gamma is None else _c(gamma, np.float32)
    y, r = np.empty_like(x), np.empty(x.shape[0], np.float32)
    lib().oc_rms_norm(_p(x), x.shape[0], x.shape[1], _p(g), float(np.float32(eps)), _p(y), _p(r))
    return y, r


def absmax_quantize(y, qmax: int, qmin: int):
    y = _c(y, np.float32)
    q, s = np.empty(y.shape, np.int8), np.empty(y.shape[0], np.float32)
    lib().oc_absmax_quantize(_p(y), y.shape[0], y.shape[1], qmax, qmin, _p(q), _p(s))
    return q, s


def quant_act(x, gamma=None, eps: float = 1e-6):
    y, _ = rms_norm(x, gamma, eps)
    return absmax_quantize(y, 127, -128)


def hadamard_quant_act(x, gamma=None, eps: float = 1e-6, had_block: int = 0):
    x = _c(x, np.float32)
    K = x.shape[1]
    b = had_block or (K & -K)
    t, _ = rms_norm(x, gamma, eps)
    lib().oc_hadamard(_p(t), t.shape[0], K, b)
    q, s = absmax_quantize(t, 7, -8)
    pk = np.empty((x.shape[0], K // 2), np.uint8)
    lib().oc_pack_int4(_p(q), q.shape[0], K, _p(pk))
    return pk, s, q, t


def linear(qx, s_x, qw, s_w):
    qx, qw, s_x = _c(qx, np.int8), _c(qw, np.int8), _c(s_x, np.float32)
    M, K = qx.shape
    N = qw.shape[0]
    acc = np.empty((M, N), np.int64)
    lib().oc_int_matmul(_p(qx), _p(qw), M, N, K, _p(acc))
    y = np.empty((M, N), np.float32)
    lib().oc_dequantize(_p(acc), M, N, _p(s_x), float(s_w), _p(y))
    return acc, y


def relu2_glu(gate, up):
    gate, up = _c(gate, np.float32), _c(up, np.float32)
    a = np.empty_like(gate)
    lib().oc_relu2_glu(_p(gate), _p(up), gate.size, _p(a))
    return a


def add(a, b):
    a, b = _c(a, np.float32), _c(b, np.float32)
    out = np.empty_like(a)
    lib().oc_add(_p(a), _p(b), a.size, _p(out))
    return out


def chain_layer(x, layer: dict, eps: float = 1e-6):
    """One layer of the stacked chain from the C++ primitives; layer[name] = (codes, s_w).
    Q/K/V/up/gate take int8 activations, O and down int4 after the Hadamard transform;
    O's input is V's output (attention over one token); residual adds in fp32."""
    x = _c(x, np.float32)
    qx, sx = quant_act(x, None, eps)
    y = {}
    for name in ("q", "k", "v"):
        _, y[name] = linear(qx, sx, *layer[name])
    _, so, co, _ = hadamard_quant_act(y["v"], None, eps)
    _, o = linear(co, so, *layer["o"])
    h = add(x, o)
    qh, sh = quant_act(h, None, eps)
    _, up = linear(qh, sh, *layer["up"])
    _, gate = linear(qh, sh, *layer["gate"])
    _, sd, cd, _ = hadamard_quant_act(relu2_glu(gate, up), None, eps)
    _, d = linear(cd, sd, *layer["down"])
    return add(h, d)
