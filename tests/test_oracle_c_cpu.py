"""The plain C++ oracle and the numpy oracle, written separately from the same
definitions, must agree bit for bit.  A slip in either (an order of
operations, a rounding, a bit layout) shows up here, on the CPU."""
import numpy as np
import pytest

from bitlinear_bitnet_quant_b200 import workloads as wl
from oracle import bitnet_oracle as O
from oracle import c_oracle as C


def _bits(a):
    return np.asarray(a, np.float32).view(np.uint32)


@pytest.mark.parametrize("shape,seed", [((64, 256), 0), ((7, 48), 1), ((300, 1040), 2)])
def test_weights_agree(shape, seed):
    w = wl.weights(*shape, seed=seed)
    w[0, :5] = [0.0, -0.0, 1e-40, -3e-39, 6e4]          # zeros, subnormals, a large value
    pk_o, s_o, q_o = O.quantize_weights(w)
    pk_c, s_c, q_c = C.quantize_weights(w)
    assert C.exact_sum_abs(w) == O.exact_sum_abs(w)
    assert _bits(s_c) == _bits(s_o)
    assert np.array_equal(q_c, q_o) and np.array_equal(pk_c, pk_o)


def test_exact_sum_rounds_once():
    """Terms whose plain fp64 running sum loses the small ones."""
    w = np.array([2.0 ** 60, 1.0, 1.0, -(2.0 ** 60)] + [2.0 ** -140] * 3, np.float32)
    assert C.exact_sum_abs(w) == O.exact_sum_abs(w) == float(2 * 2 ** 60 + 2 + 3 * 2.0 ** -140)


@pytest.mark.parametrize("M,K,use_gamma", [(5, 256, False), (3, 2560, True), (4, 1040, False), (2, 8192, True)])
def test_quant_act_agrees(M, K, use_gamma):
    x = wl.add_entry_outliers(np.random.default_rng(K), wl.gaussian(np.random.default_rng(M), (M, K)), 0.01, 20.0)
    x[0] = 0.0
    gamma = np.random.default_rng(3).uniform(0.5, 1.5, K).astype(np.float32) if use_gamma else None
    q_o, s_o = O.quant_act(x, gamma, 1e-6)
    q_c, s_c = C.quant_act(x, gamma, 1e-6)
    assert np.array_equal(_bits(s_c), _bits(s_o)) and np.array_equal(q_c, q_o)


@pytest.mark.parametrize("M,K,b", [(3, 1024, 0), (2, 5632, 0), (4, 8192, 0), (2, 2048, 256)])
def test_hadamard_quant_agrees(M, K, b):
    x = wl.student_t(np.random.default_rng(K + b), (M, K))
    pk_o, s_o, q_o, t_o = O.hadamard_quant_act(x, None, 1e-6, b)
    pk_c, s_c, q_c, t_c = C.hadamard_quant_act(x, None, 1e-6, b)
    assert np.array_equal(_bits(t_c), _bits(t_o))
    assert np.array_equal(_bits(s_c), _bits(s_o))
    assert np.array_equal(q_c, q_o) and np.array_equal(pk_c, pk_o)


def test_linear_agrees():
    rng = np.random.default_rng(9)
    qx = rng.integers(-128, 128, size=(6, 1024)).astype(np.int8)
    qw = rng.integers(-1, 2, size=(40, 1024)).astype(np.int8)
    s_x = rng.uniform(0.5, 200, 6).astype(np.float32)
    s_w = np.float32(17.25)
    acc_o, y_o = O.linear(qx, s_x, qw, s_w)
    acc_c, y_c = C.linear(qx, s_x, qw, s_w)
    assert np.array_equal(acc_c, acc_o) and np.array_equal(_bits(y_c), _bits(y_o))


@pytest.mark.parametrize("N,K", [(3, 12), (5, 2560), (2, 37)])
def test_trit5_agrees(N, K):
    q = np.random.default_rng(N + K).integers(-1, 2, size=(N, K)).astype(np.int8)
    assert np.array_equal(C.pack_trit5(q, O.trit5_row_bytes(K)), O.pack_trit5(q))


def test_chain_layer_agrees():
    """One stacked layer (int8 and int4 projections, squared-ReLU GLU, fp32
    residuals) at a reduced width, through both oracles."""
    H, F = 256, 704                                  # 704 = 11 blocks of 64 for the Hadamard
    shapes = {"q": (H, H), "k": (H, H), "v": (H, H), "o": (H, H), "up": (F, H), "gate": (F, H), "down": (H, F)}
    layer = {}
    for i, (name, (n, k)) in enumerate(sorted(shapes.items())):
        _, s_w, q = O.quantize_weights(wl.weights(n, k, seed=i))
        layer[name] = (q, s_w)
    x = wl.gaussian(np.random.default_rng(4), (6, H))
    y_o = O.chain_layer(x, layer)
    y_c = C.chain_layer(x, layer)
    assert np.array_equal(_bits(y_c), _bits(y_o))
