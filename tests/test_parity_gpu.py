"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bar: codes, packed weights, scales and int32 accumulators bit-exact; fp32
outputs bit-exact to the oracle's fixed fp32 formula and within 1e-5 relative
of its float64 rescale; bf16 outputs equal the round-to-nearest-even of the
oracle's fp32 output.  Hadamard outputs bit-exact, and within 1e-5 of the
largest magnitude of a float64 transform of the same normalised input.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from bitlinear_bitnet_quant_b200 import workloads as wl  # noqa: E402
from oracle import bitnet_oracle as O  # noqa: E402

pytestmark = pytest.mark.gpu

api = None


@pytest.fixture(scope="module", autouse=True)
def _lib():
    global api
    from bitlinear_bitnet_quant_b200 import api as _api, build_lib
    build_lib.build()
    api = _api
    api.lib()
    yield
    assert api.bitnet_device_error() == 0


def dev(a: np.ndarray, dtype=None) -> "torch.Tensor":
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == "bf16":
        t = t.view(torch.int16).view(torch.bfloat16) if a.dtype == np.uint16 else t.to(torch.bfloat16)
    return t.cuda()


def x_inputs(x, dtype):
    """(device tensor, fp32 values the oracle sees) for fp32 values or bf16 bits."""
    if dtype == "bf16":
        bits = x if x.dtype == np.uint16 else wl.f32_to_bf16_bits(x)
        return dev(bits, "bf16"), O.bf16_bits_to_f32(bits)
    return dev(x.astype(np.float32)), x.astype(np.float32)


def host(t):
    return t.cpu().numpy()


# ------------------------------------------------------------------ weights --

@pytest.mark.parametrize("N,K,dtype", [(256, 256, "f32"), (384, 1024, "f32"), (128, 2560, "bf16"),
                                       (130, 48, "f32"), (6912, 2560, "f32")])
def test_quantize_weights(N, K, dtype):
    w = wl.weights(N, K, seed=N + K)
    if dtype == "bf16":
        bits = wl.f32_to_bf16_bits(w)
        wd, w_or = dev(bits, "bf16"), O.bf16_bits_to_f32(bits)
    else:
        wd, w_or = dev(w), w
    pk, s_w = api.bitnet_quantize_weights(wd)
    pk_o, s_o, q_o = O.quantize_weights(w_or)
    assert host(s_w)[0].view(np.uint32) == np.float32(s_o).view(np.uint32)
    assert np.array_equal(host(pk), pk_o)


def test_quantize_weights_edge_cases():
    zero = np.zeros((128, 64), np.float32)
    pk, s_w = api.bitnet_quantize_weights(dev(zero))
    assert host(s_w)[0] == np.float32(1.0) / np.float32(1e-5) and not host(pk).any()
    rng = np.random.default_rng(1)
    wide = (rng.standard_normal((64, 256)) * np.exp2(rng.integers(-140, 120, (64, 256)))).astype(np.float32)
    wide[0, :4] = [1e-45, -1e-44, 3e38, -2e-38]
    pk, s_w = api.bitnet_quantize_weights(dev(wide))
    pk_o, s_o, _ = O.quantize_weights(wide)
    assert host(s_w)[0] == s_o and np.array_equal(host(pk), pk_o)
    const = np.full((32, 32), -0.02, np.float32)
    pk, s_w = api.bitnet_quantize_weights(dev(const))
    pk_o, s_o, q_o = O.quantize_weights(const)
    assert host(s_w)[0] == s_o and np.array_equal(host(pk), pk_o) and np.all(q_o == -1)


# ------------------------------------------------------------------ int8 act --

@pytest.mark.parametrize("M,K,dtype,use_gamma", [
    (1, 16, "f32", False), (3, 48, "bf16", True), (17, 256, "f32", False), (8, 256, "f32", True),
    (16, 2560, "bf16", False), (129, 4096, "bf16", False), (5, 2048, "bf16", True),
    (7, 5632, "bf16", False), (2, 16384, "bf16", False), (3, 16384, "f32", True), (33, 1040, "f32", False),
    (40, 2048, "f32", True), (600, 2048, "f32", False), (700, 4096, "bf16", True)])
def test_quant_act(M, K, dtype, use_gamma):
    x = wl.add_entry_outliers(np.random.default_rng(M * K), wl.gaussian(np.random.default_rng(K), (M, K)),
                              0.005, 30.0)
    xd, x_or = x_inputs(x, dtype)
    gamma = np.random.default_rng(7).uniform(0.5, 1.5, K).astype(np.float32) if use_gamma else None
    q, s = api.bitnet_quant_act(xd, dev(gamma) if use_gamma else None, 1e-6)
    q_o, s_o = O.quant_act(x_or, gamma, 1e-6)
    assert np.array_equal(host(s).view(np.uint32), s_o.view(np.uint32))
    assert np.array_equal(host(q), q_o)


@pytest.mark.parametrize("K,dtype", [(4096, "bf16"), (2048, "f32"), (2560, "bf16"), (96, "f32")])
def test_quant_act_rows_independent_of_call_size(K, dtype):
    """A token's codes and scale do not depend on the other tokens of the call."""
    x = wl.add_entry_outliers(np.random.default_rng(K), wl.gaussian(np.random.default_rng(K + 1), (65, K)),
                              0.005, 30.0)
    xd, _ = x_inputs(x, dtype)
    q_warp, s_warp = api.bitnet_quant_act(xd[:64].contiguous(), None, 1e-6)
    q_cta, s_cta = api.bitnet_quant_act(xd, None, 1e-6)
    assert np.array_equal(host(s_warp).view(np.uint32), host(s_cta)[:64].view(np.uint32))
    assert np.array_equal(host(q_warp), host(q_cta)[:64])


def test_quant_act_edge_rows():
    K = 512
    x = np.zeros((6, K), np.float32)
    x[1, 100] = 3.5                            # single spike
    x[2, :] = np.where(np.arange(K) % 2 == 0, 2.0, -2.0)   # every element at +-absmax
    x[3, :] = 1e-30                            # tiny but nonzero
    x[4, :] = np.linspace(-1, 1, K)
    x[5, :7] = [6e4, -6e4, 1, 2, 3, 4, 5]      # large values
    for dtype in ("f32", "bf16"):
        xd, x_or = x_inputs(x, dtype)
        q, s = api.bitnet_quant_act(xd, None, 1e-6)
        q_o, s_o = O.quant_act(x_or, None, 1e-6)
        assert np.array_equal(host(s), s_o) and np.array_equal(host(q), q_o)
    assert np.all(q_o[0] == 0) and q_o[1, 100] == 127 and np.all(np.abs(q_o[2]) == 127)


def test_quant_act_full_prefill():
    c = wl.prefill(with_weights=False)
    xd, x_or = x_inputs(c["x"], "bf16")
    q, s = api.bitnet_quant_act(xd, None, 1e-6)
    q_o, s_o = O.quant_act(x_or, None, 1e-6)
    assert np.array_equal(host(s), s_o) and np.array_equal(host(q), q_o)


# ------------------------------------------------------------------ Hadamard --

def _check_hadamard(x, dtype, had_block, gamma=None):
    xd, x_or = x_inputs(x, dtype)
    q4, s, t = api.bitnet_hadamard_quant_act(xd, dev(gamma) if gamma is not None else None, 1e-6,
                                             had_block, want_t=True)
    pk_o, s_o, q_o, t_o = O.hadamard_quant_act(x_or, gamma, 1e-6, had_block)
    assert np.array_equal(host(t).view(np.uint32), t_o.view(np.uint32))
    assert np.array_equal(host(s), s_o)
    assert np.array_equal(host(q4), pk_o)
    # against a float64 transform of the same normalised input
    b = had_block or O.default_had_block(x.shape[1])
    y, _ = O.rms_norm(x_or, gamma, 1e-6)
    y64 = y.astype(np.float64).reshape(y.shape[0], -1, b)
    h = 1
    while h < b:
        v = y64.reshape(y.shape[0], -1, b // (2 * h), 2, h)
        y64 = np.stack([v[..., 0, :] + v[..., 1, :], v[..., 0, :] - v[..., 1, :]], axis=-2).reshape(y64.shape)
        h *= 2
    t64 = y64.reshape(y.shape) / math.sqrt(b)
    err = np.abs(host(t).astype(np.float64) - t64).max(axis=1)
    assert np.all(err <= 1e-5 * np.abs(t64).max(axis=1) + 1e-30)


@pytest.mark.parametrize("M,K,b,dtype", [
    (1, 128, 0, "f32"), (5, 256, 32, "bf16"), (33, 1024, 64, "bf16"), (3, 1024, 256, "f32"),
    (9, 2048, 0, "bf16"), (7, 5632, 0, "bf16"), (4, 8192, 0, "bf16"), (2, 8192, 1024, "f32"),
    (130, 4096, 4096, "bf16"), (3, 16384, 8192, "bf16"), (17, 1536, 512, "f32")])
def test_hadamard_quant(M, K, b, dtype):
    rng = np.random.default_rng(M + K + b)
    x = wl.add_channel_outliers(rng, wl.student_t(rng, (M, K)), 0.005, 50.0)
    _check_hadamard(x, dtype, b)


@pytest.mark.parametrize("M,K,b,dtype", [(2400, 2048, 0, "bf16"), (700, 5632, 0, "f32"), (4800, 256, 32, "f32")])
def test_hadamard_quant_many_tokens(M, K, b, dtype):
    """Enough tokens for the register kernel (few tokens take the one-CTA-per-
    token kernel): both must give the same bits as the oracle."""
    x = wl.student_t(np.random.default_rng(M + K), (M, K))
    _check_hadamard(x, dtype, b)


@pytest.mark.parametrize("M,K,b,dtype,use_gamma", [(640, 4096, 0, "bf16", False), (600, 8192, 1024, "f32", False),
                                                   (700, 16384, 8192, "bf16", True), (620, 8192, 0, "f32", True),
                                                   (900, 4096, 2048, "f32", False), (300, 8192, 0, "bf16", True),
                                                   (2400, 4096, 0, "bf16", False)])
def test_hadamard_quant_split_kernel(M, K, b, dtype, use_gamma):
    """Many tokens at K = 4096 / 8192 / 16384 with blocks of 1024 or more: the
    kernels that spread a token over K/32 threads (three index-bit groups;
    packed fp32 pairs for one block of 8192)."""
    rng = np.random.default_rng(M + K + b)
    x = wl.add_channel_outliers(rng, wl.student_t(rng, (M, K)), 0.005, 50.0)
    x[0] = 0
    x[1] = 0
    x[1, K // 3] = 3.0
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float32) if use_gamma else None
    _check_hadamard(x, dtype, b, gamma)


def test_hadamard_gamma_and_edges():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((6, 1024)).astype(np.float32)
    x[0] = 0
    x[1] = 0; x[1, 17] = 2.0
    x[2] = 1.0
    _check_hadamard(x, "f32", 0, rng.uniform(0.5, 2, 1024).astype(np.float32))


def test_hadamard_full_config():
    c = wl.hbitlinear(with_weights=False)
    _check_hadamard(c["x"], "bf16", 0)


# ------------------------------------------------------------------ linear ----

def _random_codes(M, N, K, act_bits, seed):
    rng = np.random.default_rng(seed)
    lo, hi = (-128, 128) if act_bits == 8 else (-8, 8)
    qx = rng.integers(lo, hi, size=(M, K)).astype(np.int8)
    qw = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    s_x = rng.uniform(0.5, 200, size=M).astype(np.float32)
    return qx, qw, s_x, np.float32(rng.uniform(5, 60))


def _run_linear(qx, qw, s_x, s_w, act_bits, out, path):
    xq_dev = dev(qx) if act_bits == 8 else dev(O.pack_int4(qx))
    Y, acc = api.bitnet_linear(xq_dev, act_bits, dev(s_x), dev(O.pack_ternary(qw)),
                               dev(np.array([s_w], np.float32)),
                               out_dtype=torch.float32 if out == "f32" else torch.bfloat16, want_acc=True,
                               kernel=path)
    torch.cuda.synchronize()
    return Y, acc


def _check_linear(qx, qw, s_x, s_w, act_bits, out, path, rows=None):
    Y, acc = _run_linear(qx, qw, s_x, s_w, act_bits, out, path)
    Y, acc = host(Y.float() if out == "bf16" else Y), host(acc)
    if rows is not None:
        Y, acc, qx, s_x = Y[rows], acc[rows], qx[rows], s_x[rows]
    acc_o, y_o = O.linear(qx, s_x, qw, s_w)
    assert np.array_equal(acc, acc_o)
    if out == "f32":
        assert np.array_equal(Y.view(np.uint32), y_o.view(np.uint32))
        ref = O.dequantize_f64(acc_o, s_x, s_w)
        nz = acc_o != 0
        assert np.max(np.abs(Y[nz] - ref[nz]) / np.abs(ref[nz]), initial=0) <= 1e-5
    else:
        assert np.array_equal(O.bf16_round(Y), O.bf16_round(y_o))


@pytest.mark.parametrize("path", [1, 2])
@pytest.mark.parametrize("M,N,K,act_bits,out", [
    (1, 128, 128, 8, "f32"), (2, 256, 256, 8, "f32"), (3, 256, 256, 8, "bf16"), (16, 384, 1024, 8, "f32"),
    (17, 400, 256, 8, "f32"), (100, 256, 2560, 8, "bf16"), (129, 256, 512, 8, "f32"),
    (300, 272, 384, 8, "f32"), (257, 128, 1024, 8, "f32"),
    (1, 128, 256, 4, "f32"), (5, 256, 1024, 4, "f32"), (33, 400, 512, 4, "bf16"), (200, 256, 2048, 4, "f32"),
    (16, 1024, 2560, 4, "f32"), (32, 1152, 2560, 8, "bf16"), (9, 128, 128, 8, "f32")])
def test_linear_random_codes(M, N, K, act_bits, out, path):
    qx, qw, s_x, s_w = _random_codes(M, N, K, act_bits, M * 7 + N + K)
    _check_linear(qx, qw, s_x, s_w, act_bits, out, path)


@pytest.mark.parametrize("M,N,K,act_bits,out", [
    (1, 16, 512, 8, "f32"), (1, 1, 512, 8, "f32"), (3, 200, 1024, 8, "bf16"), (8, 1000, 1536, 8, "f32"),
    (9, 4096, 512, 8, "f32"), (16, 6912, 2560, 8, "bf16"), (16, 300, 8192, 8, "f32"), (5, 64, 16384, 8, "f32"),
    (1, 20000, 1024, 8, "f32"), (16, 2368, 4608, 8, "f32"),
    (2, 512, 4608, 4, "f32"), (16, 2048, 5632, 4, "f32"), (7, 333, 2560, 4, "bf16"), (1, 48, 512, 4, "f32"),
    (17, 1000, 2048, 8, "f32"), (32, 5632, 2048, 8, "bf16"), (32, 2048, 5632, 4, "f32"), (24, 333, 512, 4, "f32"),
    (31, 100, 10240, 8, "f32")])
def test_linear_decode_kernel(M, N, K, act_bits, out):
    """The one-pass warp-MMA kernel (up to 32 tokens): ragged N, one, two and
    four token groups, K of 1 to 32 segments (one and several activation
    batches)."""
    qx, qw, s_x, s_w = _random_codes(M, N, K, act_bits, M * 13 + N + K)
    _check_linear(qx, qw, s_x, s_w, act_bits, out, path=3)


# ------------------------------------------------- five weights per byte ----

@pytest.mark.parametrize("N,K", [(3, 16), (7, 48), (64, 2560), (300, 8192), (1, 16384), (5, 1040), (129, 80)])
def test_repack_trit5(N, K):
    """2-bit packed -> five per byte, bit-exact against the oracle's packing of the same codes."""
    qw = np.random.default_rng(N * K).integers(-1, 2, size=(N, K)).astype(np.int8)
    pk5 = api.bitnet_repack_trit5(dev(O.pack_ternary(qw)))
    torch.cuda.synchronize()
    assert np.array_equal(host(pk5), O.pack_trit5(qw))


@pytest.mark.parametrize("M,N,K,act_bits,out", [
    (1, 16, 512, 8, "f32"), (1, 1, 512, 8, "f32"), (4, 6912, 2560, 8, "f32"), (8, 1000, 1536, 8, "bf16"),
    (9, 4096, 512, 8, "f32"), (16, 6912, 2560, 8, "f32"), (16, 300, 8192, 8, "f32"), (5, 64, 16384, 8, "f32"),
    (17, 1000, 2048, 8, "f32"), (32, 2048, 5632, 4, "f32"), (7, 333, 2560, 4, "bf16"), (24, 333, 512, 4, "f32")])
def test_linear_trit5(M, N, K, act_bits, out):
    """The decode kernel reading five-per-byte weights (packed by the oracle): int32
    accumulators and outputs bit-exact against the oracle and against the 2-bit path."""
    qx, qw, s_x, s_w = _random_codes(M, N, K, act_bits, M * 17 + N + K)
    xq_dev = dev(qx) if act_bits == 8 else dev(O.pack_int4(qx))
    odt = torch.float32 if out == "f32" else torch.bfloat16
    Y5, acc5 = api.bitnet_linear_trit5(xq_dev, act_bits, dev(s_x), dev(O.pack_trit5(qw)),
                                       dev(np.array([s_w], np.float32)), K, out_dtype=odt, want_acc=True)
    torch.cuda.synchronize()
    Y2, _ = _run_linear(qx, qw, s_x, s_w, act_bits, out, path=3)
    Y5h = host(Y5.float() if out == "bf16" else Y5)
    acc_o, y_o = O.linear(qx, s_x, qw, s_w)
    assert np.array_equal(host(acc5), acc_o)
    if out == "f32":
        assert np.array_equal(Y5h.view(np.uint32), y_o.view(np.uint32))
    else:
        assert np.array_equal(O.bf16_round(Y5h), O.bf16_round(y_o))
    assert torch.equal(Y5.view(torch.int16 if out == "bf16" else torch.int32),
                       Y2.view(torch.int16 if out == "bf16" else torch.int32))


def test_trit5_end_to_end_from_fp32_weights():
    """bitnet_quantize_weights -> bitnet_repack_trit5 -> bitnet_linear_trit5 on the decode
    workload's weights (sampled rows), against the oracle."""
    c = wl.decode(4)
    w = c["w"]
    pk, s_w = api.bitnet_quantize_weights(dev(w))
    pk5 = api.bitnet_repack_trit5(pk)
    xd, x_or = x_inputs(c["x"], "bf16")
    xq, s_x = api.bitnet_quant_act(xd, None, 1e-6)
    Y, acc = api.bitnet_linear_trit5(xq, 8, s_x, pk5, s_w, w.shape[1], want_acc=True)
    torch.cuda.synchronize()
    _, s_o, q_o = O.quantize_weights(w)
    assert np.array_equal(host(pk5), O.pack_trit5(q_o))
    qx_o, sx_o = O.quant_act(x_or, None, 1e-6)
    rows = np.random.default_rng(3).choice(w.shape[0], 256, replace=False)
    acc_o, y_o = O.linear(qx_o, sx_o, q_o[rows], s_o)
    assert np.array_equal(host(acc)[:, rows], acc_o)
    assert np.array_equal(host(Y)[:, rows].view(np.uint32), y_o.view(np.uint32))


def test_linear_decode_kernel_rejects_other_shapes():
    qx, qw, s_x, s_w = _random_codes(33, 64, 512, 8, 1)
    with pytest.raises(api.BitnetError):
        _run_linear(qx, qw, s_x, s_w, 8, "f32", path=3)
    qx, qw, s_x, s_w = _random_codes(4, 64, 384, 8, 2)
    with pytest.raises(api.BitnetError):
        _run_linear(qx, qw, s_x, s_w, 8, "f32", path=3)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_linear_decode_full(M):
    c = wl.decode(M)
    xd, x_or = x_inputs(c["x"], "bf16")
    pk, s_w = api.bitnet_quantize_weights(dev(c["w"]))
    q, s = api.bitnet_quant_act(xd, None, 1e-6)
    Y, acc = api.bitnet_linear(q, 8, s, pk, s_w, want_acc=True)
    pk_o, s_wo, qw_o = O.quantize_weights(c["w"])
    q_o, s_o = O.quant_act(x_or, None, 1e-6)
    acc_o, y_o = O.linear(q_o, s_o, qw_o, s_wo)
    assert np.array_equal(host(acc), acc_o)
    assert np.array_equal(host(Y).view(np.uint32), y_o.view(np.uint32))


@pytest.mark.parametrize("M,K,Ns,act_bits,out", [
    (1, 2048, [2048, 2048, 2048], 8, "f32"),          # the chain's Q/K/V at one token
    (16, 2560, [6912, 128], 8, "bf16"),
    (32, 2048, [5632, 5632], 8, "f32"),               # up/gate at the chain's decode batch
    (9, 1024, [200, 1000, 48, 16], 4, "f32"),         # ragged N, int4 activations, four matrices
    (33, 512, [384, 130], 8, "f32"),                  # tensor-core kernel, ragged N
    (130, 1024, [256, 520, 128], 4, "bf16"),
    (512, 2048, [2048, 2048, 2048], 8, "f32"),        # the chain's Q/K/V at 512 tokens
])
def test_linear_group(M, K, Ns, act_bits, out):
    """Several matrices sharing the activations in one launch: each output equals
    the oracle's product bit for bit, and the separate bitnet_linear call."""
    rng = np.random.default_rng(M * 7 + K + len(Ns))
    lo, hi = (-128, 128) if act_bits == 8 else (-8, 8)
    qx = rng.integers(lo, hi, size=(M, K)).astype(np.int8)
    s_x = rng.uniform(0.5, 200, size=M).astype(np.float32)
    xq = dev(qx) if act_bits == 8 else dev(O.pack_int4(qx))
    mats, ws = [], []
    for N in Ns:
        qw = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
        s_w = np.float32(rng.uniform(5, 60))
        mats.append((qw, s_w))
        ws.append((dev(O.pack_ternary(qw)), dev(np.array([s_w], np.float32))))
    od = torch.float32 if out == "f32" else torch.bfloat16
    Ys = api.bitnet_linear_group(xq, act_bits, dev(s_x), ws, out_dtype=od)
    torch.cuda.synchronize()
    for (qw, s_w), Y, (pk, sw) in zip(mats, Ys, ws):
        _, y_o = O.linear(qx, s_x, qw, s_w)
        got = host(Y.float()) if out == "bf16" else host(Y)
        if out == "f32":
            assert np.array_equal(got.view(np.uint32), y_o.view(np.uint32))
        else:
            assert np.array_equal(host(Y.view(torch.int16)).view(np.uint16), O.bf16_round(y_o))
        Y1, _ = api.bitnet_linear(xq, act_bits, dev(s_x), pk, sw, out_dtype=od)
        assert torch.equal(Y1, Y)


@pytest.mark.parametrize("M,N,K,act_bits,out", [(128, 2048, 2048, 8, "f32"), (512, 2048, 5632, 4, "f32"),
                                              (100, 384, 1024, 8, "bf16"), (64, 640, 4096, 4, "f32")])
def test_linear_split_k_wide_tiles(M, N, K, act_bits, out):
    """Few 64- or 128-token tiles: K split over a cluster, partial sums meeting in
    the leader's shared memory; bit-exact like every other launch shape."""
    qx, qw, s_x, s_w = _random_codes(M, N, K, act_bits, seed=M * 3 + N + K)
    _check_linear(qx, qw, s_x, s_w, act_bits, out, path=2)
    # and through the tensor-store epilogue (no accumulator output)
    od = torch.float32 if out == "f32" else torch.bfloat16
    xq = dev(qx) if act_bits == 8 else dev(O.pack_int4(qx))
    Y, _ = api.bitnet_linear(xq, act_bits, dev(s_x), dev(O.pack_ternary(qw)), dev(np.array([s_w], np.float32)),
                             out_dtype=od)
    _, y_o = O.linear(qx, s_x, qw, s_w)
    if out == "f32":
        assert np.array_equal(host(Y).view(np.uint32), y_o.view(np.uint32))
    else:
        assert np.array_equal(O.bf16_round(host(Y.float())), O.bf16_round(y_o))


@pytest.mark.parametrize("M,N,K,act_bits,out", [(130, 520, 512, 8, "f32"), (33, 300, 1024, 4, "bf16"),
                                              (256, 768, 2048, 8, "bf16"), (200, 260, 384, 4, "f32"),
                                              (5, 256, 256, 8, "f32")])
def test_linear_256_row_tile(M, N, K, act_bits, out):
    """The tcgen05 kernel with two accumulators (256 weight rows per CTA), forced
    at small and ragged shapes: bit-exact accumulators and outputs."""
    qx, qw, s_x, s_w = _random_codes(M, N, K, act_bits, seed=M + N + K)
    _check_linear(qx, qw, s_x, s_w, act_bits, out, path=4)


@pytest.mark.parametrize("M,N,K,out", [(130, 520, 512, "f32"), (300, 1000, 1024, "bf16"), (65, 128, 256, "f32"),
                                      (1000, 1200, 768, "bf16"), (4096, 640, 256, "f32")])
def test_linear_persistent(M, N, K, out):
    """The persistent tcgen05 kernel (one CTA per SM looping over 128 x 128
    tiles, two accumulators, its own epilogue warps), forced at small and ragged
    shapes: bit-exact accumulators (per-element epilogue) and outputs (staged,
    one bulk store per tile)."""
    qx, qw, s_x, s_w = _random_codes(M, N, K, 8, seed=M + 3 * N + K)
    _check_linear(qx, qw, s_x, s_w, 8, out, path=5)
    xq, pk = dev(qx), dev(O.pack_ternary(qw))
    od = torch.float32 if out == "f32" else torch.bfloat16
    Y5, _ = api.bitnet_linear(xq, 8, dev(s_x), pk, dev(np.array([s_w], np.float32)), out_dtype=od, kernel=5)
    Y2, _ = api.bitnet_linear(xq, 8, dev(s_x), pk, dev(np.array([s_w], np.float32)), out_dtype=od, kernel=2)
    torch.cuda.synchronize()
    assert api.bitnet_device_error() == 0
    assert torch.equal(Y5, Y2)


def test_linear_group_many_tiles():
    """A group whose tiles fill several waves: every output equals the
    oracle's product."""
    rng = np.random.default_rng(77)
    M, K, Ns = 1024, 512, (4096, 5632)
    qx = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    s_x = rng.uniform(0.5, 200, size=M).astype(np.float32)
    mats, ws = [], []
    for N in Ns:
        qw = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
        s_w = np.float32(rng.uniform(5, 60))
        mats.append((qw, s_w))
        ws.append((dev(O.pack_ternary(qw)), dev(np.array([s_w], np.float32))))
    Ys = api.bitnet_linear_group(dev(qx), 8, dev(s_x), ws, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert api.bitnet_device_error() == 0
    for (qw, s_w), Y in zip(mats, Ys):
        _, y_o = O.linear(qx, s_x, qw, s_w)
        assert np.array_equal(host(Y).view(np.uint32), y_o.view(np.uint32))


# ------------------------------------------------------- fused BitLinear ----

def _check_bitlinear(M, N, K, dtype, use_gamma, out, path=0, seed=0):
    rng = np.random.default_rng(seed + M * 31 + K)
    x = wl.add_entry_outliers(rng, wl.gaussian(rng, (M, K)), 0.005, 30.0)
    xd, x_or = x_inputs(x, dtype)
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float32) if use_gamma else None
    w = wl.weights(N, K, seed=seed + N)
    pk, s_w = api.bitnet_quantize_weights(dev(w))
    Y, q, s = api.bitnet_bitlinear(xd, pk, s_w, dev(gamma) if use_gamma else None, 1e-6,
                                   out_dtype=torch.float32 if out == "f32" else torch.bfloat16, kernel=path)
    torch.cuda.synchronize()
    assert api.bitnet_device_error() == 0
    _, s_wo, qw_o = O.quantize_weights(w)
    q_o, s_o = O.quant_act(x_or, gamma, 1e-6)
    assert np.array_equal(host(s).view(np.uint32), s_o.view(np.uint32))
    assert np.array_equal(host(q), q_o)
    acc_o, y_o = O.linear(q_o, s_o, qw_o, s_wo)
    if out == "f32":
        assert np.array_equal(host(Y).view(np.uint32), y_o.view(np.uint32))
    else:
        assert np.array_equal(O.bf16_round(host(Y.float())), O.bf16_round(y_o))


@pytest.mark.parametrize("M,N,K,dtype,use_gamma,out", [
    (1, 6912, 2560, "bf16", False, "f32"), (4, 6912, 2560, "bf16", False, "f32"),
    (16, 6912, 2560, "bf16", False, "bf16"), (3, 200, 512, "f32", True, "f32"), (8, 1000, 1536, "bf16", True, "f32"),
    (9, 2048, 2048, "f32", False, "f32"), (17, 5632, 2048, "f32", True, "f32"), (32, 2048, 2048, "f32", False, "bf16"),
    (32, 300, 4096, "bf16", False, "f32"), (16, 300, 8192, "bf16", False, "f32"), (12, 16, 4608, "bf16", False, "f32"),
    (1, 1, 512, "bf16", False, "f32")])
def test_bitlinear_fused(M, N, K, dtype, use_gamma, out):
    """One kernel: clusters of 8 CTAs quantise every eighth token each and
    share the codes through distributed shared memory; the codes, scales and
    outputs match the oracle bit for bit (ragged N, 1 to 4 token groups, K of
    1 to 16 segments, grids padded to whole clusters)."""
    _check_bitlinear(M, N, K, dtype, use_gamma, out, path=4)
    _check_bitlinear(M, N, K, dtype, use_gamma, out, path=0)     # the two-kernel default


@pytest.mark.parametrize("M,N,K,path", [(40, 512, 1024, 0), (4, 256, 384, 0), (16, 6912, 2560, 2),
                                        (5, 300, 1024, 3), (2, 128, 16384, 0), (3, 100, 1024, 1)])
def test_bitlinear_two_kernel_paths(M, N, K, path):
    """The quantiser and the selected linear kernel in sequence."""
    _check_bitlinear(M, N, K, "bf16", False, "f32", path=path)


def test_bitlinear_fused_rejects_other_shapes():
    for M, K in ((33, 512), (4, 384), (40, 1024), (32, 8192)):
        with pytest.raises(api.BitnetError):
            _check_bitlinear(M, 64, K, "bf16", False, "f32", path=4)


def test_linear_prefill_sampled():
    c = wl.prefill()
    xd, x_or = x_inputs(c["x"], "bf16")
    pk, s_w = api.bitnet_quantize_weights(dev(c["w"]))
    q, s = api.bitnet_quant_act(xd, None, 1e-6)
    Y, acc = api.bitnet_linear(q, 8, s, pk, s_w, out_dtype=torch.bfloat16, want_acc=True)
    rows = np.random.default_rng(0).choice(c["M"], size=12, replace=False)
    rows = np.concatenate([rows, [0, c["M"] - 1]])
    _, s_wo, qw_o = O.quantize_weights(c["w"])
    q_o, s_o = O.quant_act(x_or[rows], None, 1e-6)
    acc_o, y_o = O.linear(q_o, s_o, qw_o, s_wo)
    assert np.array_equal(host(acc)[rows], acc_o)
    assert np.array_equal(O.bf16_round(host(Y.float())[rows]), O.bf16_round(y_o))
    # the launch the bench times (no accumulator output: 256-row tiles and the
    # tensor-store epilogue) gives the same bits everywhere
    Y2, _ = api.bitnet_linear(q, 8, s, pk, s_w, out_dtype=torch.bfloat16)
    assert torch.equal(Y2.view(torch.int16), Y.view(torch.int16))
    assert np.array_equal(O.bf16_round(host(Y2.float())[rows]), O.bf16_round(y_o))


@pytest.mark.parametrize("M,N,K,out", [(2048, 4736, 512, "f32"), (2100, 4800, 1024, "bf16")])
def test_linear_256_row_tile_store_path(M, N, K, out):
    """Enough tiles for the automatic 256-row choice, with the tensor-store
    epilogue (no accumulator output), including a ragged last row block and
    token tile: sampled rows against the oracle, and every element against
    the 128-row tile."""
    qx, qw, s_x, s_w = _random_codes(M, N, K, 8, seed=M + N)
    od = torch.float32 if out == "f32" else torch.bfloat16
    args = (dev(qx), 8, dev(s_x), dev(O.pack_ternary(qw)), dev(np.array([s_w], np.float32)))
    Y, _ = api.bitnet_linear(*args, out_dtype=od)
    Y2, _ = api.bitnet_linear(*args, out_dtype=od, kernel=2)
    rows = np.concatenate([np.random.default_rng(2).choice(M, size=10, replace=False), [0, M - 1]])
    _, y_o = O.linear(qx[rows], s_x[rows], qw, s_w)
    got = host(Y.float())[rows]
    if out == "f32":
        assert np.array_equal(got.view(np.uint32), y_o.view(np.uint32))
    else:
        assert np.array_equal(O.bf16_round(got), O.bf16_round(y_o))
    Y3, _ = api.bitnet_linear(*args, out_dtype=od, kernel=4)
    assert torch.equal(Y.view(torch.int16) if out == "bf16" else Y, Y3.view(torch.int16) if out == "bf16" else Y3)
    # the 128-row kernel on the same operands (its own launch shape)
    assert torch.equal(Y.float(), Y2.float())


def test_hbitlinear_sampled():
    c = wl.hbitlinear()
    xd, x_or = x_inputs(c["x"], "bf16")
    pk, s_w = api.bitnet_quantize_weights(dev(c["w"]))
    q4, s, _ = api.bitnet_hadamard_quant_act(xd, None, 1e-6, 0)
    Y, acc = api.bitnet_linear(q4, 4, s, pk, s_w, want_acc=True)
    rows = np.concatenate([np.random.default_rng(1).choice(c["M"], size=14, replace=False), [0, c["M"] - 1]])
    _, s_wo, qw_o = O.quantize_weights(c["w"])
    _, s_o, q_o, _ = O.hadamard_quant_act(x_or[rows], None, 1e-6, 0)
    acc_o, y_o = O.linear(q_o, s_o, qw_o, s_wo)
    assert np.array_equal(host(acc)[rows], acc_o)
    assert np.array_equal(host(Y)[rows].view(np.uint32), y_o.view(np.uint32))


def test_tiny_bitlinear_forward():
    c = wl.tiny()
    pk, s_w = api.bitnet_quantize_weights(dev(c["w"]))
    Y = api.bitlinear_forward(dev(c["x"]), pk, s_w)
    _, s_wo, qw_o = O.quantize_weights(c["w"])
    out = O.bitlinear(c["x"], qw_o, s_wo)
    assert np.array_equal(host(Y), out["y"])
    ref = O.fake_quant_matmul_f64(out["codes"], out["s_x"], qw_o, s_wo)
    nz = out["acc"] != 0
    assert np.max(np.abs(host(Y)[nz] - ref[nz]) / np.abs(ref[nz])) <= 1e-5


# ------------------------------------------------------------------ chain -----

def _chain_weights(layers):
    from bitlinear_bitnet_quant_b200 import chain
    gpu, ora = [], []
    for l in range(layers):
        w = wl.chain_weights(l)
        gpu.append(chain.quantize_layer({k: dev(v) for k, v in w.items()}))
        oq = {}
        for k, v in w.items():
            _, s_w, q = O.quantize_weights(v)
            oq[k] = (q, s_w)
        ora.append(oq)
    return gpu, ora


@pytest.mark.parametrize("M,rows", [(32, None), (512, [0, 1, 77, 255, 256, 400, 510, 511])])
def test_chain_two_layers(M, rows):
    """Two stacked layers at full width (hidden 2048, FFN 5632); every op is per
    token, so the oracle follows sampled token rows through both layers."""
    from bitlinear_bitnet_quant_b200 import chain
    gpu_w, ora_w = _chain_weights(2)
    x = wl.chain_input(M)
    ch = chain.BitLinearChain(gpu_w, M, wl.CHAIN_HIDDEN, wl.CHAIN_FFN, torch.device("cuda"))
    out = host(ch.forward(dev(x)))
    sel = np.arange(M) if rows is None else np.array(rows)
    ref = x[sel]
    for lw in ora_w:
        ref = O.chain_layer(ref, lw)
    assert np.array_equal(out[sel].view(np.uint32), ref.view(np.uint32))


def test_chain_24_layers():
    """All 24 stacked layers of the chain workload, each with its own weights, at
    both batch sizes (32 decode tokens, 512 prefill tokens).  Every op is per
    token, so the plain C++ oracle (held bit for bit to the numpy oracle by the
    CPU tests; OpenMP over rows) follows sampled token rows through all 24
    layers, from its own quantisation of the fp32 weights."""
    from bitlinear_bitnet_quant_b200 import chain
    from oracle import c_oracle as C
    gpu_w, ora_w = [], []
    for l in range(24):
        w = wl.chain_weights(l)
        gpu_w.append(chain.quantize_layer({k: dev(v) for k, v in w.items()}))
        oq = {}
        for k, v in w.items():
            _, s_w, q = C.quantize_weights(v)
            oq[k] = (q, s_w)
        ora_w.append(oq)
        del w
    for M, rows in ((32, [0, 5, 18, 31]), (512, [0, 129, 300, 511])):
        x = wl.chain_input(M)
        ch = chain.BitLinearChain(gpu_w, M, wl.CHAIN_HIDDEN, wl.CHAIN_FFN, torch.device("cuda"))
        out = host(ch.forward(dev(x)))
        ref = x[rows]
        for lw in ora_w:
            ref = C.chain_layer(ref, lw)
        assert np.all(np.isfinite(ref))
        assert np.array_equal(out[rows].view(np.uint32), ref.view(np.uint32)), M


@pytest.mark.parametrize("M,K,use_gamma", [(3, 2048, False), (32, 2048, True), (5, 16, False), (17, 5632, False),
                                             (2, 16384, True), (300, 2048, True), (512, 2048, False)])
def test_add_quant_act(M, K, use_gamma):
    """Residual add folded into the int8 quantiser: H, codes and scales equal
    bitnet_add followed by bitnet_quant_act, bit for bit."""
    rng = np.random.default_rng(M * 3 + K)
    a = wl.gaussian(rng, (M, K))
    b = wl.gaussian(rng, (M, K), 0.5)
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float32) if use_gamma else None
    H, q, s = api.bitnet_add_quant_act(dev(a), dev(b), dev(gamma) if use_gamma else None, 1e-6)
    h_o = a + b
    q_o, s_o = O.quant_act(h_o, gamma, 1e-6)
    assert np.array_equal(host(H).view(np.uint32), h_o.view(np.uint32))
    assert np.array_equal(host(s).view(np.uint32), s_o.view(np.uint32))
    assert np.array_equal(host(q), q_o)


@pytest.mark.parametrize("M,K,b", [(3, 5632, 0), (32, 5632, 0), (4, 2048, 0), (7, 8192, 1024), (2, 1024, 32),
                                   (5, 8192, 0)])
def test_glu_hadamard_quant_act(M, K, b):
    """Squared-ReLU gated unit folded into the Hadamard int4 quantiser: codes
    and scales equal bitnet_relu2_glu followed by bitnet_hadamard_quant_act."""
    rng = np.random.default_rng(M * 5 + K)
    gate = wl.gaussian(rng, (M, K))
    up = wl.gaussian(rng, (M, K))
    q4, s = api.bitnet_glu_hadamard_quant_act(dev(gate), dev(up), None, 1e-6, b)
    pk_o, s_o, _, _ = O.hadamard_quant_act(O.squared_relu_glu(gate, up), None, 1e-6, b)
    assert np.array_equal(host(s).view(np.uint32), s_o.view(np.uint32))
    assert np.array_equal(host(q4), pk_o)


def test_elementwise_glue():
    rng = np.random.default_rng(21)
    a = rng.standard_normal(4096 * 3).astype(np.float32)
    b = rng.standard_normal(4096 * 3).astype(np.float32)
    s = host(api.bitnet_add(dev(a), dev(b)))
    assert np.array_equal(s, a + b)
    g = host(api.bitnet_relu2_glu(dev(a), dev(b)))
    assert np.array_equal(g, O.squared_relu_glu(a, b))


# -------------------------------------------------------------- attention -----
#
# Rotary embedding and softmax attention decide no integer code; they are
# compared with the oracle's float64 definitions within the bound the fp32
# arithmetic allows (u = 2^-24):
#   rotation, computed in fp64 and rounded once: |error| <= u * |pair|;
#   attention: each score q.k/sqrt(d) is a 128-term fp32 dot product, off by at
#   most E_j = (128 + 3) u sqrt(1/d) sum_i |q_i k_ji| (accumulation, scaling and
#   the rounding of the rotated inputs); the softmax weights then move by a
#   relative 2E (E = max_j E_j), expf by 2 ulp and the running rescaling by
#   about 2 u per key, so each output is within (2E + (8 + 2n) u) max_j |v_j|.

U32 = 2.0 ** -24


def _attention_tol(q, k, v, mask, heads):
    """Per (query, head) bound of the fp32 attention against float64."""
    d = q.shape[1] // heads
    tol = np.zeros((q.shape[0], heads))
    for h in range(heads):
        sl = slice(h * d, (h + 1) * d)
        mag = np.abs(q[:, sl]).astype(np.float64) @ np.abs(k[:, sl]).astype(np.float64).T / math.sqrt(d)
        mag = np.where(mask, mag, 0.0)
        E = 131 * U32 * mag.max(axis=1)
        n = mask.sum(axis=1)
        vmax = np.array([np.abs(v[mask[i]][:, sl]).max() for i in range(q.shape[0])])
        tol[:, h] = (2 * E + (8 + 2 * n) * U32) * vmax * 1.05 + 1e-30
    return tol


def _check_attention(got, ref, tol, heads):
    d = got.shape[1] // heads
    err = np.abs(got.astype(np.float64) - ref).reshape(got.shape[0], heads, d).max(axis=2)
    assert np.all(err <= tol), (err / tol).max()


def _rand_rows(rng, n, HD, scale=0.6):
    return (rng.standard_normal((n, HD)) * scale).astype(np.float32)


@pytest.mark.parametrize("B,L,t0,heads", [(1, 64, 0, 16), (2, 40, 0, 16), (3, 20, 37, 2), (32, 1, 512, 16),
                                          (4, 5, 100, 4), (2, 1, 0, 16), (1, 512, 0, 16), (1, 300, 0, 2),
                                          (2, 130, 70, 4), (1, 200, 0, 4)])
def test_rope_append_and_attention(B, L, t0, heads):
    """RoPE of Q and K, the cache append, and causal attention over the cache,
    on the prefill kernel (16 or more queries per sequence: pairs of query
    blocks sharing their keys over two CTAs, an odd middle block split in half)
    and the decode kernel (fewer)."""
    rng = np.random.default_rng(B * 1000 + L * 10 + t0)
    HD = heads * 128
    T_cap = t0 + L + 3
    q, k, v = (_rand_rows(rng, B * L, HD) for _ in range(3))
    # earlier positions of the caches: already rotated keys and values
    kc0 = _rand_rows(rng, B * T_cap, HD).reshape(B, T_cap, HD)
    vc0 = _rand_rows(rng, B * T_cap, HD).reshape(B, T_cap, HD)
    Qd, Kd, Vd = dev(q), dev(k), dev(v)
    Kc, Vc = dev(kc0), dev(vc0)
    api.bitnet_rope_append(Qd, Kd, Vd, Kc, Vc, B, L, t0, heads)
    A = api.bitnet_attention(Qd, Kc, Vc, B, L, t0, heads)
    torch.cuda.synchronize()
    qr, kcg, vcg, a = host(Qd), host(Kc), host(Vc), host(A)
    pos = np.tile(t0 + np.arange(L), B)
    q_ref = O.rope_f64(q, pos, heads)
    k_ref = O.rope_f64(k, pos, heads)
    pair = lambda x: np.repeat(np.sqrt((x.astype(np.float64).reshape(x.shape[0], -1, 2) ** 2).sum(-1)), 2, axis=1)
    assert np.all(np.abs(qr - q_ref) <= U32 * pair(q) * 1.001 + 1e-38)
    for b in range(B):
        rows = slice(t0, t0 + L)
        kg = kcg[b, rows]
        assert np.all(np.abs(kg - k_ref[b * L:(b + 1) * L]) <= U32 * pair(k[b * L:(b + 1) * L]) * 1.001 + 1e-38)
        assert np.array_equal(vcg[b, rows], v[b * L:(b + 1) * L])
        # rows outside the step are untouched
        assert np.array_equal(kcg[b, :t0], kc0[b, :t0]) and np.array_equal(kcg[b, t0 + L:], kc0[b, t0 + L:])
        mask = O.causal_mask(L, t0 + L, t0)
        ref = O.attention_f64(qr[b * L:(b + 1) * L], kcg[b, :t0 + L], vcg[b, :t0 + L], heads, mask)
        tol = _attention_tol(qr[b * L:(b + 1) * L], kcg[b, :t0 + L], vcg[b, :t0 + L], mask, heads)
        _check_attention(a[b * L:(b + 1) * L], ref, tol, heads)
    if t0 == 0 and L == 1:
        assert np.array_equal(a, v)                 # one visible key: its value, exactly


def test_chain_with_attention_prefill_then_decode():
    """Two full-width layers (hidden 2048, 16 heads, FFN 5632) with the attention
    core: a 24-token prefill of 2 sequences, then one decode step.  Layer by
    layer, the GPU's own layer input goes to the oracle: K and V bit-exact; the
    rotation and attention within their fp32 bounds; and from the GPU's
    attention output on, everything bit-exact (O, residual, up/gate, gated
    unit, down)."""
    from bitlinear_bitnet_quant_b200 import chain
    gpu_w, ora_w = _chain_weights(2)
    B, L, H, heads = 2, 24, wl.CHAIN_HIDDEN, 16
    T_cap = L + 1
    x_pre = wl.chain_input(B * L, seed=5)
    x_dec = wl.chain_input(B, seed=6)
    pre = chain.BitLinearChain(gpu_w, B * L, H, wl.CHAIN_FFN, torch.device("cuda"),
                               attention=dict(B=B, L=L, T_cap=T_cap, heads=heads))
    dec = chain.BitLinearChain(gpu_w, B, H, wl.CHAIN_FFN, torch.device("cuda"),
                               attention=dict(B=B, L=1, T_cap=T_cap, heads=heads))
    dec.kc, dec.vc = pre.kc, pre.vc                  # the decode step continues the prefill's caches
    ora_k = [np.zeros((B, T_cap, H)) for _ in range(2)]
    ora_v = [np.zeros((B, T_cap, H)) for _ in range(2)]
    for ch, x0, t0, Ls in ((pre, x_pre, 0, L), (dec, x_dec, L, 1)):
        ch.t0 = t0
        parts = (dev(x0),)
        x_in = x0
        for li, (w, lw) in enumerate(zip(gpu_w, ora_w)):
            h, d = ch.layer(parts, w, None, li)
            torch.cuda.synchronize()
            qx, sx = O.quant_act(x_in, None, 1e-6)
            _, q = O.linear(qx, sx, *lw["q"])
            _, k = O.linear(qx, sx, *lw["k"])
            _, v = O.linear(qx, sx, *lw["v"])
            assert np.array_equal(host(ch.k), k) and np.array_equal(host(ch.v), v)
            pos = np.tile(t0 + np.arange(Ls), B)
            q_r, k_r = O.rope_f64(q, pos, heads), O.rope_f64(k, pos, heads)
            for b in range(B):
                ora_k[li][b, t0:t0 + Ls] = k_r[b * Ls:(b + 1) * Ls]
                ora_v[li][b, t0:t0 + Ls] = v[b * Ls:(b + 1) * Ls]
            att_g = host(ch.att)
            qg = host(ch.q)
            kcg, vcg = host(ch.kc[li]), host(ch.vc[li])
            for b in range(B):
                sl = slice(b * Ls, (b + 1) * Ls)
                mask = O.causal_mask(Ls, t0 + Ls, t0)
                ref = O.attention_f64(q_r[sl], ora_k[li][b, :t0 + Ls], ora_v[li][b, :t0 + Ls], heads, mask)
                tol = _attention_tol(qg[sl], kcg[b, :t0 + Ls], vcg[b, :t0 + Ls], mask, heads)
                _check_attention(att_g[sl], ref, tol, heads)
            # from the GPU's attention output on, the oracle follows bit for bit
            _, so, co, _ = O.hadamard_quant_act(att_g, None, 1e-6)
            _, o = O.linear(co, so, *lw["o"])
            hh = x_in + o
            qh, sh = O.quant_act(hh, None, 1e-6)
            _, up = O.linear(qh, sh, *lw["up"])
            _, gate = O.linear(qh, sh, *lw["gate"])
            _, sd, cd, _ = O.hadamard_quant_act(O.squared_relu_glu(gate, up), None, 1e-6)
            _, dd = O.linear(cd, sd, *lw["down"])
            assert np.array_equal(host(h), hh) and np.array_equal(host(d), dd)
            x_in = hh + dd
            parts = (h, d)


# ------------------------------------------------------------ measurement -----

def test_measure_i8_mma_runs():
    """The int8 tensor-core throughput measurement completes on every SM, and its
    cycle count is plausible: at least half the cycles that 128 x bn x 32 MACs
    per MMA take at 8192 MACs per clock and SM (about the nominal dense rate)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for bn in (128, 256):
        cyc, ns = api.bitnet_measure_i8_mma(2048, bn, sms)
        torch.cuda.synchronize()
        c, t = host(cyc), host(ns)
        assert np.all(c > 0) and np.all(t > 0)
        assert np.all(c >= 2048 * (128 * bn * 32 // 8192) * 0.5)
    assert api.bitnet_device_error() == 0


def test_bounded_wait_gives_up_and_reports():
    """A pipeline wait that nothing completes gives up after its time limit,
    records a code in the device error flag and lets the kernel exit: the
    context stays usable and the next call computes correctly."""
    assert api.bitnet_device_error() == 0
    api.bitnet_selftest_wait_timeout()
    torch.cuda.synchronize()
    assert api.bitnet_device_error() == 1          # the code of a timed-out "full" wait
    assert api.bitnet_device_error() == 0          # reading clears it
    qx, qw, s_x, s_w = _random_codes(40, 256, 512, 8, seed=77)
    _check_linear(qx, qw, s_x, s_w, 8, "f32", path=2)
