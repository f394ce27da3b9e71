"""bitnet_quantize_weights_noalloc against bitnet_quantize_weights.

The no-allocation variant exists for callers that may not allocate device
memory themselves -- a plugin inside an application that owns every device
allocation, a runtime that reserves its memory up front, or code that must
not take the implicit synchronisation of cudaMalloc/cudaFree.  It keeps its
scratch in a fixed array inside the library, so two calls in a row must each
start from cleared scratch and match the workspace version bit for bit.

This file is named so that pytest collects it last; it also passes on its own
in a fresh process.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from bitlinear_bitnet_quant_b200 import workloads as wl  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from bitlinear_bitnet_quant_b200 import api, build_lib
    build_lib.build()
    return api.lib()


def _reference(W):
    from bitlinear_bitnet_quant_b200 import api
    pk, s_w = api.bitnet_quantize_weights(W)
    torch.cuda.synchronize()
    return pk.cpu().numpy(), s_w.cpu().numpy()


def _noalloc(L, W, code):
    """Calls the C entry point directly; the test owns inputs and outputs."""
    N, K = W.shape
    pk = torch.full((N, K // 4), 0xAA, dtype=torch.uint8, device=W.device)
    s_w = torch.full((1,), -1.0, dtype=torch.float32, device=W.device)
    stream = torch.cuda.current_stream().cuda_stream
    st = L.bitnet_quantize_weights_noalloc(ctypes.c_void_p(W.data_ptr()), code, N, K,
                                           ctypes.c_void_p(pk.data_ptr()), ctypes.c_void_p(s_w.data_ptr()),
                                           ctypes.c_void_p(stream))
    assert st == 0, st
    torch.cuda.synchronize()
    return pk.cpu().numpy(), s_w.cpu().numpy()


def test_noalloc_matches_workspace_version_twice(L):
    # two calls in a row with different tensors: the shared scratch must be
    # cleared by each call, so the second result must not carry the first's sum
    w1 = torch.from_numpy(wl.weights(384, 1024, seed=11)).cuda()
    bits = wl.f32_to_bf16_bits(wl.weights(256, 2560, seed=12) * np.float32(3.0))
    w2 = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    got1 = _noalloc(L, w1, 0)
    got2 = _noalloc(L, w2, 1)
    ref1 = _reference(w1)
    ref2 = _reference(w2)
    assert np.array_equal(got1[0], ref1[0]) and got1[1].view(np.uint32) == ref1[1].view(np.uint32)
    assert np.array_equal(got2[0], ref2[0]) and got2[1].view(np.uint32) == ref2[1].view(np.uint32)
    # and once more with the first tensor: same answer as the first call
    again = _noalloc(L, w1, 0)
    assert np.array_equal(again[0], ref1[0]) and again[1] == ref1[1]


def test_noalloc_zero_tensor_after_a_nonzero_one(L):
    # an all-zero tensor right after a nonzero one: the floor scale 1/1e-5 and
    # all-zero codes, exactly as the workspace version gives
    w1 = torch.from_numpy(wl.weights(128, 512, seed=13)).cuda()
    z = torch.zeros((128, 512), dtype=torch.float32, device="cuda")
    _noalloc(L, w1, 0)
    got = _noalloc(L, z, 0)
    ref = _reference(z)
    assert np.all(got[0] == 0) and np.array_equal(got[0], ref[0])
    assert got[1].view(np.uint32) == ref[1].view(np.uint32)
    assert got[1][0] == np.float32(1.0) / np.float32(1e-5)


def test_noalloc_rejects_tensors_beyond_its_limit(L):
    big = 1 << 16                      # N*K = 2^32 > 2^31 - 1 weights
    st = L.bitnet_quantize_weights_noalloc(ctypes.c_void_p(0x10000), 0, big, big,
                                           ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), None)
    assert st == 2                     # BITNET_ERR_SHAPE, nothing enqueued
    huge = 1 << 40                     # N*K would overflow 64 bits: still refused
    st = L.bitnet_quantize_weights_noalloc(ctypes.c_void_p(0x10000), 0, huge, huge,
                                           ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), None)
    assert st == 2
