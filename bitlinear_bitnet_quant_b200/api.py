"""Thin Python binding of libbitnet.so (include/bitnet.h).

Argument marshalling only: every step of the BitLinear path runs in the
library's CUDA kernels.  PyTorch supplies device memory and the current
stream.  The functions keep the C names; outputs not passed in are allocated
with torch on the input's device.  Any nonzero status raises BitnetError.
If the library is missing, loading raises instead of falling back.
"""
from __future__ import annotations

import ctypes
import glob
import os
import re

import torch

from . import build_lib

_c_void_p = ctypes.c_void_p
_i64 = ctypes.c_int64

BITNET_F32 = 0
BITNET_BF16 = 1

_lib = None

# argument types of every entry point declared in include/bitnet.h
_SIGNATURES = {
    "bitnet_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "bitnet_abi_version": (ctypes.c_int, []),
    "bitnet_quantize_weights_workspace_size": (ctypes.c_size_t, [_i64, _i64]),
    "bitnet_quantize_weights": (ctypes.c_int, [_c_void_p, ctypes.c_int, _i64, _i64, _c_void_p, _c_void_p,
                                               _c_void_p, ctypes.c_size_t, _c_void_p]),
    "bitnet_quantize_weights_noalloc": (ctypes.c_int, [_c_void_p, ctypes.c_int, _i64, _i64, _c_void_p,
                                                       _c_void_p, _c_void_p]),
    "bitnet_quant_act": (ctypes.c_int, [_c_void_p, ctypes.c_int, _i64, _i64, _c_void_p, ctypes.c_float,
                                        _c_void_p, _c_void_p, _c_void_p]),
    "bitnet_hadamard_quant_act": (ctypes.c_int, [_c_void_p, ctypes.c_int, _i64, _i64, _c_void_p, ctypes.c_float,
                                                 ctypes.c_int, _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "bitnet_linear": (ctypes.c_int, [_c_void_p, ctypes.c_int, _c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i64,
                                     _c_void_p, ctypes.c_int, _c_void_p, _c_void_p]),
    "bitnet_bitlinear": (ctypes.c_int, [_c_void_p, ctypes.c_int, _i64, _i64, _c_void_p, ctypes.c_float,
                                        _c_void_p, _c_void_p, _i64, _c_void_p, ctypes.c_int, _c_void_p, _c_void_p,
                                        _c_void_p]),
    "bitnet_add_quant_act": (ctypes.c_int, [_c_void_p, _c_void_p, _i64, _i64, _c_void_p, ctypes.c_float, _c_void_p,
                                            _c_void_p, _c_void_p, _c_void_p]),
    "bitnet_glu_hadamard_quant_act": (ctypes.c_int, [_c_void_p, _c_void_p, _i64, _i64, _c_void_p, ctypes.c_float,
                                                     ctypes.c_int, _c_void_p, _c_void_p, _c_void_p]),
    "bitnet_add": (ctypes.c_int, [_c_void_p, _c_void_p, _c_void_p, _i64, _c_void_p]),
    "bitnet_relu2_glu": (ctypes.c_int, [_c_void_p, _c_void_p, _c_void_p, _i64, _c_void_p]),
    "bitnet_trit5_row_bytes": (ctypes.c_size_t, [_i64]),
    "bitnet_repack_trit5": (ctypes.c_int, [_c_void_p, _i64, _i64, _c_void_p, _c_void_p]),
    "bitnet_linear_trit5": (ctypes.c_int, [_c_void_p, ctypes.c_int, _c_void_p, _c_void_p, _c_void_p, _i64, _i64,
                                           _i64, _c_void_p, ctypes.c_int, _c_void_p, _c_void_p]),
    "bitnet_linear_kernel": (ctypes.c_int, [_c_void_p, ctypes.c_int, _c_void_p, _c_void_p, _c_void_p, _i64, _i64,
                                            _i64, _c_void_p, ctypes.c_int, _c_void_p, ctypes.c_int, _c_void_p]),
    "bitnet_bitlinear_kernel": (ctypes.c_int, [_c_void_p, ctypes.c_int, _i64, _i64, _c_void_p, ctypes.c_float,
                                               _c_void_p, _c_void_p, _i64, _c_void_p, ctypes.c_int, _c_void_p,
                                               _c_void_p, ctypes.c_int, _c_void_p]),
    "bitnet_linear_group": (ctypes.c_int, [_c_void_p, ctypes.c_int, _c_void_p, _i64, _i64, ctypes.c_int,
                                           ctypes.POINTER(_c_void_p), ctypes.POINTER(_c_void_p),
                                           ctypes.POINTER(_i64), ctypes.POINTER(_c_void_p), ctypes.c_int,
                                           _c_void_p]),
    "bitnet_rope_append": (ctypes.c_int, [_c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i64, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_double, _c_void_p, _c_void_p, _i64, _c_void_p]),
    "bitnet_attention": (ctypes.c_int, [_c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i64, ctypes.c_int,
                                        ctypes.c_int, _i64, _c_void_p, _c_void_p]),
    "bitnet_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int)]),
    "bitnet_measure_i8_mma": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, _c_void_p, _c_void_p,
                                             _c_void_p]),
    "bitnet_selftest_wait_timeout": (ctypes.c_int, [_c_void_p]),
}


class BitnetError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: status {status} ({status_string(status)})")


def header_functions() -> list[str]:
    """Names of the functions the headers under include/ declare."""
    names = []
    for h in sorted(glob.glob(os.path.join(build_lib.INCLUDE, "*.h"))):
        with open(h) as f:
            names += re.findall(r"^BITNET_API\s+[\w\s\*]+?\b(bitnet_\w+)\s*\(", f.read(), flags=re.M)
    return names


def lib() -> ctypes.CDLL:
    """Load libbitnet.so (built in-tree by build_lib); raises if it is missing."""
    global _lib
    if _lib is None:
        path = build_lib.LIB
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m bitlinear_bitnet_quant_b200.build_lib`")
        L = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().bitnet_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise BitnetError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return BITNET_F32
    if t.dtype == torch.bfloat16:
        return BITNET_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: fp32 or bf16 expected")


def _require(t: torch.Tensor, name: str):
    if not (t.is_cuda and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------

def bitnet_quantize_weights_workspace_size(N: int, K: int) -> int:
    return int(lib().bitnet_quantize_weights_workspace_size(N, K))


def bitnet_quantize_weights(W: torch.Tensor, pkW=None, s_w=None, workspace=None, stream=None):
    """Absmean ternarisation + packing.  Returns (pkW uint8 [N, K/4], s_w fp32 [1])."""
    _require(W, "W")
    N, K = W.shape
    dev = W.device
    pkW = torch.empty((N, K // 4), dtype=torch.uint8, device=dev) if pkW is None else pkW
    s_w = torch.empty((1,), dtype=torch.float32, device=dev) if s_w is None else s_w
    ws_bytes = bitnet_quantize_weights_workspace_size(N, K)
    workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev) if workspace is None else workspace
    _check("bitnet_quantize_weights", lib().bitnet_quantize_weights(
        _ptr(W), _dtype_code(W), N, K, _ptr(pkW), _ptr(s_w), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return pkW, s_w


def bitnet_quantize_weights_noalloc(W: torch.Tensor, pkW: torch.Tensor, s_w: torch.Tensor, stream=None):
    """Same as bitnet_quantize_weights, but the library allocates nothing: the
    caller passes the outputs, and the scratch is a fixed array in the library."""
    _require(W, "W")
    _require(pkW, "pkW")
    N, K = W.shape
    _check("bitnet_quantize_weights_noalloc", lib().bitnet_quantize_weights_noalloc(
        _ptr(W), _dtype_code(W), N, K, _ptr(pkW), _ptr(s_w), _stream(stream)))
    return pkW, s_w


def bitnet_quant_act(X: torch.Tensor, gamma=None, eps: float = 1e-6, Xq=None, s_x=None, stream=None):
    """RMSNorm + per-token absmax int8.  Returns (Xq int8 [M, K], s_x fp32 [M])."""
    _require(X, "X")
    M, K = X.shape
    Xq = torch.empty((M, K), dtype=torch.int8, device=X.device) if Xq is None else Xq
    s_x = torch.empty((M,), dtype=torch.float32, device=X.device) if s_x is None else s_x
    _check("bitnet_quant_act", lib().bitnet_quant_act(
        _ptr(X), _dtype_code(X), M, K, _ptr(gamma), float(eps), _ptr(Xq), _ptr(s_x), _stream(stream)))
    return Xq, s_x


def bitnet_hadamard_quant_act(X: torch.Tensor, gamma=None, eps: float = 1e-6, had_block: int = 0,
                              Xq4=None, s_x=None, want_t: bool = False, stream=None):
    """RMSNorm + Hadamard + per-token int4.  Returns (Xq4 uint8 [M, K/2], s_x [M], t or None)."""
    _require(X, "X")
    M, K = X.shape
    Xq4 = torch.empty((M, K // 2), dtype=torch.uint8, device=X.device) if Xq4 is None else Xq4
    s_x = torch.empty((M,), dtype=torch.float32, device=X.device) if s_x is None else s_x
    T = torch.empty((M, K), dtype=torch.float32, device=X.device) if want_t else None
    _check("bitnet_hadamard_quant_act", lib().bitnet_hadamard_quant_act(
        _ptr(X), _dtype_code(X), M, K, _ptr(gamma), float(eps), int(had_block), _ptr(Xq4), _ptr(s_x),
        _ptr(T), _stream(stream)))
    return Xq4, s_x, T


def bitnet_add_quant_act(A: torch.Tensor, B: torch.Tensor, gamma=None, eps: float = 1e-6, H=None, Xq=None, s_x=None,
                         stream=None):
    """H = A + B (fp32), then the int8 quantiser of H.  Returns (H, Xq, s_x)."""
    _require(A, "A")
    _require(B, "B")
    M, K = A.shape
    H = torch.empty_like(A) if H is None else H
    Xq = torch.empty((M, K), dtype=torch.int8, device=A.device) if Xq is None else Xq
    s_x = torch.empty((M,), dtype=torch.float32, device=A.device) if s_x is None else s_x
    _check("bitnet_add_quant_act", lib().bitnet_add_quant_act(
        _ptr(A), _ptr(B), M, K, _ptr(gamma), float(eps), _ptr(H), _ptr(Xq), _ptr(s_x), _stream(stream)))
    return H, Xq, s_x


def bitnet_glu_hadamard_quant_act(gate: torch.Tensor, up: torch.Tensor, gamma=None, eps: float = 1e-6,
                                  had_block: int = 0, Xq4=None, s_x=None, stream=None):
    """x = relu(gate)^2 * up (fp32), then the Hadamard int4 quantiser of x.  Returns (Xq4, s_x)."""
    _require(gate, "gate")
    _require(up, "up")
    M, K = gate.shape
    Xq4 = torch.empty((M, K // 2), dtype=torch.uint8, device=gate.device) if Xq4 is None else Xq4
    s_x = torch.empty((M,), dtype=torch.float32, device=gate.device) if s_x is None else s_x
    _check("bitnet_glu_hadamard_quant_act", lib().bitnet_glu_hadamard_quant_act(
        _ptr(gate), _ptr(up), M, K, _ptr(gamma), float(eps), int(had_block), _ptr(Xq4), _ptr(s_x), _stream(stream)))
    return Xq4, s_x


def bitnet_linear(Xq: torch.Tensor, act_bits: int, s_x: torch.Tensor, pkW: torch.Tensor, s_w: torch.Tensor,
                  out_dtype=torch.float32, Y=None, want_acc: bool = False, stream=None, kernel: int = 0):
    """Ternary x int8/int4 product + dequantisation.  Returns (Y [M, N], acc int32 or None).
    kernel != 0 picks the kernel family for this call (bitnet_linear_kernel)."""
    _require(Xq, "Xq")
    _require(pkW, "pkW")
    M = Xq.shape[0]
    N, KB = pkW.shape
    K = KB * 4
    Y = torch.empty((M, N), dtype=out_dtype, device=Xq.device) if Y is None else Y
    acc = torch.empty((M, N), dtype=torch.int32, device=Xq.device) if want_acc else None
    args = (_ptr(Xq), int(act_bits), _ptr(s_x), _ptr(pkW), _ptr(s_w), M, N, K, _ptr(Y), _dtype_code(Y), _ptr(acc))
    if kernel:
        _check("bitnet_linear_kernel", lib().bitnet_linear_kernel(*args, int(kernel), _stream(stream)))
    else:
        _check("bitnet_linear", lib().bitnet_linear(*args, _stream(stream)))
    return Y, acc


def bitnet_linear_group(Xq: torch.Tensor, act_bits: int, s_x: torch.Tensor, weights, out_dtype=torch.float32,
                        Ys=None, stream=None):
    """Several products sharing Xq and s_x in one launch.  weights: [(pkW, s_w), ...]
    (1 to 4 entries, same K).  Returns the list of outputs [M, N_g]."""
    _require(Xq, "Xq")
    M = Xq.shape[0]
    count = len(weights)
    K = weights[0][0].shape[1] * 4
    for pk, _ in weights:
        _require(pk, "pkW")
    if Ys is None:
        Ys = [torch.empty((M, pk.shape[0]), dtype=out_dtype, device=Xq.device) for pk, _ in weights]
    arr = lambda ts: (_c_void_p * count)(*[t.data_ptr() for t in ts])
    Ns = (_i64 * count)(*[pk.shape[0] for pk, _ in weights])
    _check("bitnet_linear_group", lib().bitnet_linear_group(
        _ptr(Xq), int(act_bits), _ptr(s_x), M, K, count, arr([w[0] for w in weights]), arr([w[1] for w in weights]),
        Ns, arr(Ys), _dtype_code(Ys[0]), _stream(stream)))
    return Ys


def bitnet_trit5_row_bytes(K: int) -> int:
    """Bytes per row of the five-weights-per-byte format."""
    return int(lib().bitnet_trit5_row_bytes(int(K)))


def bitnet_repack_trit5(pkW: torch.Tensor, pk5=None, stream=None):
    """2-bit packed weights [N, K/4] -> five weights per byte [N, bitnet_trit5_row_bytes(K)] uint8."""
    _require(pkW, "pkW")
    N, KB = pkW.shape
    K = KB * 4
    pk5 = torch.empty((N, bitnet_trit5_row_bytes(K)), dtype=torch.uint8, device=pkW.device) if pk5 is None else pk5
    _check("bitnet_repack_trit5", lib().bitnet_repack_trit5(_ptr(pkW), N, K, _ptr(pk5), _stream(stream)))
    return pk5


def bitnet_linear_trit5(Xq: torch.Tensor, act_bits: int, s_x: torch.Tensor, pk5: torch.Tensor, s_w: torch.Tensor,
                        K: int, out_dtype=torch.float32, Y=None, want_acc: bool = False, stream=None):
    """bitnet_linear with the weights five per byte (decode shapes).  Returns (Y [M, N], acc int32 or None)."""
    _require(Xq, "Xq")
    _require(pk5, "pk5")
    M = Xq.shape[0]
    N = pk5.shape[0]
    Y = torch.empty((M, N), dtype=out_dtype, device=Xq.device) if Y is None else Y
    acc = torch.empty((M, N), dtype=torch.int32, device=Xq.device) if want_acc else None
    _check("bitnet_linear_trit5", lib().bitnet_linear_trit5(
        _ptr(Xq), int(act_bits), _ptr(s_x), _ptr(pk5), _ptr(s_w), M, N, int(K), _ptr(Y), _dtype_code(Y),
        _ptr(acc), _stream(stream)))
    return Y, acc


def bitnet_bitlinear(X: torch.Tensor, pkW: torch.Tensor, s_w: torch.Tensor, gamma=None, eps: float = 1e-6,
                     out_dtype=torch.float32, Y=None, Xq=None, s_x=None, stream=None, kernel: int = 0):
    """Fused BitLinear forward with int8 activations (RMSNorm + absmax int8 +
    ternary product + dequantisation).  Returns (Y [M, N], Xq [M, K], s_x [M]).
    kernel != 0 picks the kernels for this call (bitnet_bitlinear_kernel; 4 = one fused kernel)."""
    _require(X, "X")
    _require(pkW, "pkW")
    M, K = X.shape
    N = pkW.shape[0]
    dev = X.device
    Y = torch.empty((M, N), dtype=out_dtype, device=dev) if Y is None else Y
    Xq = torch.empty((M, K), dtype=torch.int8, device=dev) if Xq is None else Xq
    s_x = torch.empty((M,), dtype=torch.float32, device=dev) if s_x is None else s_x
    args = (_ptr(X), _dtype_code(X), M, K, _ptr(gamma), float(eps), _ptr(pkW), _ptr(s_w), N, _ptr(Y), _dtype_code(Y),
            _ptr(Xq), _ptr(s_x))
    if kernel:
        _check("bitnet_bitlinear_kernel", lib().bitnet_bitlinear_kernel(*args, int(kernel), _stream(stream)))
    else:
        _check("bitnet_bitlinear", lib().bitnet_bitlinear(*args, _stream(stream)))
    return Y, Xq, s_x


def bitnet_add(a: torch.Tensor, b: torch.Tensor, out=None, stream=None):
    """fp32 residual add: out = a + b."""
    out = torch.empty_like(a) if out is None else out
    _check("bitnet_add", lib().bitnet_add(_ptr(a), _ptr(b), _ptr(out), a.numel(), _stream(stream)))
    return out


def bitnet_relu2_glu(gate: torch.Tensor, up: torch.Tensor, out=None, stream=None):
    """Squared-ReLU gated unit: out = relu(gate)^2 * up (fp32)."""
    out = torch.empty_like(gate) if out is None else out
    _check("bitnet_relu2_glu", lib().bitnet_relu2_glu(_ptr(gate), _ptr(up), _ptr(out), gate.numel(),
                                                      _stream(stream)))
    return out


def bitnet_rope_append(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, Kc: torch.Tensor, Vc: torch.Tensor,
                       B: int, L: int, t0: int, heads: int, base: float = 10000.0, stream=None):
    """Rotary embedding of Q (in place) and K; rotated K and V rows written into
    the caches Kc, Vc [B, T_cap, heads*d] at positions t0 .. t0+L-1."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (Kc, "Kc"), (Vc, "Vc")):
        _require(t, n)
    d = Q.shape[1] // heads
    _check("bitnet_rope_append", lib().bitnet_rope_append(
        _ptr(Q), _ptr(K), _ptr(V), B, L, t0, heads, d, float(base), _ptr(Kc), _ptr(Vc), Kc.shape[1],
        _stream(stream)))


def bitnet_attention(Q: torch.Tensor, Kc: torch.Tensor, Vc: torch.Tensor, B: int, L: int, t0: int, heads: int,
                     A=None, stream=None):
    """Causal softmax attention of the rows Q [B*L, heads*d] over the caches.  Returns A."""
    for t, n in ((Q, "Q"), (Kc, "Kc"), (Vc, "Vc")):
        _require(t, n)
    A = torch.empty_like(Q) if A is None else A
    d = Q.shape[1] // heads
    _check("bitnet_attention", lib().bitnet_attention(
        _ptr(Q), _ptr(Kc), _ptr(Vc), B, L, t0, heads, d, Kc.shape[1], _ptr(A), _stream(stream)))
    return A


def bitnet_measure_i8_mma(n_mma: int, bn: int, ctas: int, stream=None):
    """Enqueues the int8 tensor-core throughput measurement; returns the (cycles,
    nanoseconds) device tensors [ctas] it fills."""
    cyc = torch.zeros((ctas,), dtype=torch.int64, device="cuda")
    ns = torch.zeros((ctas,), dtype=torch.int64, device="cuda")
    _check("bitnet_measure_i8_mma", lib().bitnet_measure_i8_mma(int(n_mma), int(bn), int(ctas), _ptr(cyc), _ptr(ns),
                                                                _stream(stream)))
    return cyc, ns


def bitnet_selftest_wait_timeout(stream=None) -> None:
    """Enqueues the bounded-wait self-test (a wait that runs out after ~2 s)."""
    _check("bitnet_selftest_wait_timeout", lib().bitnet_selftest_wait_timeout(_stream(stream)))


def bitnet_device_error() -> int:
    code = ctypes.c_int(0)
    _check("bitnet_device_error", lib().bitnet_device_error(ctypes.byref(code)))
    return code.value


def bitlinear_forward(X: torch.Tensor, pkW: torch.Tensor, s_w: torch.Tensor, act_bits: int = 8, gamma=None,
                      eps: float = 1e-6, had_block: int = 0, out_dtype=torch.float32, Y=None, Xq=None, s_x=None,
                      stream=None):
    """One BitLinear forward: quantise the activations, then the ternary
    product.  Y, Xq and s_x may be passed in to reuse buffers across calls
    (Xq: [M, K] int8 for act_bits 8, [M, K/2] uint8 packed int4 for 4)."""
    if act_bits == 8:
        Y, _, _ = bitnet_bitlinear(X, pkW, s_w, gamma, eps, out_dtype=out_dtype, Y=Y, Xq=Xq, s_x=s_x,
                                   stream=stream)
        return Y
    Xq, s_x, _ = bitnet_hadamard_quant_act(X, gamma, eps, had_block, Xq4=Xq, s_x=s_x, stream=stream)
    Y, _ = bitnet_linear(Xq, act_bits, s_x, pkW, s_w, out_dtype=out_dtype, Y=Y, stream=stream)
    return Y
