"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/bitnet.h declares, and rejects bad arguments on the
host before touching CUDA (no compute call is made here)."""

import pytest

from bitlinear_bitnet_quant_b200 import api, build_lib

ALIGNED = 0x10000          # fake device addresses: never dereferenced, validation fails first
MISALIGNED = 0x10008


@pytest.fixture(scope="module")
def L():
    build_lib.build()
    return api.lib()


def test_exports_every_declared_symbol(L):
    names = api.header_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(api._SIGNATURES)


def test_status_strings(L):
    for code in range(8):
        assert api.status_string(code)
    assert api.status_string(0) == "ok"
    assert api.status_string(99) == "unknown status"
    assert L.bitnet_abi_version() == 2
    assert L.bitnet_quantize_weights_workspace_size(4096, 4096) >= 80


def _linear(L, **kw):
    a = dict(Xq=ALIGNED, act_bits=8, s_x=ALIGNED, pkW=ALIGNED, s_w=ALIGNED, M=4, N=256, K=256,
             Y=ALIGNED, y_dtype=0, acc=None)
    a.update(kw)
    return L.bitnet_linear(a["Xq"], a["act_bits"], a["s_x"], a["pkW"], a["s_w"], a["M"], a["N"], a["K"],
                           a["Y"], a["y_dtype"], a["acc"], None)


def test_linear_validation(L):
    assert _linear(L, act_bits=5) == 4
    assert _linear(L, y_dtype=7) == 4
    assert _linear(L, K=100) == 2
    assert _linear(L, K=64) == 2
    assert _linear(L, K=65536 + 128) == 2
    assert _linear(L, N=0) == 2
    assert _linear(L, M=-1) == 2
    assert _linear(L, M=0) == 0                 # empty batch: nothing to do
    assert _linear(L, Xq=None) == 1
    assert _linear(L, Y=None) == 1
    assert _linear(L, Xq=MISALIGNED) == 3
    assert _linear(L, pkW=MISALIGNED) == 3
    assert _linear(L, acc=MISALIGNED) == 3
    assert _linear(L, s_w=ALIGNED + 2) == 3


def test_quant_act_validation(L):
    q = lambda **kw: L.bitnet_quant_act(kw.get("X", ALIGNED), kw.get("dt", 1), kw.get("M", 4), kw.get("K", 256),
                                        kw.get("gamma"), 1e-6, kw.get("Xq", ALIGNED), kw.get("s", ALIGNED), None)
    assert q(dt=3) == 4
    assert q(K=24) == 2 and q(K=0) == 2 and q(K=16384 + 16) == 2
    assert q(M=0) == 0
    assert q(X=None) == 1 and q(s=None) == 1
    assert q(X=MISALIGNED) == 3 and q(gamma=MISALIGNED) == 3


def test_hadamard_validation(L):
    h = lambda **kw: L.bitnet_hadamard_quant_act(kw.get("X", ALIGNED), 1, kw.get("M", 4), kw.get("K", 1024), None,
                                                 1e-6, kw.get("b", 0), kw.get("Xq", ALIGNED), ALIGNED,
                                                 kw.get("T"), None)
    assert h(K=1000) == 2
    assert h(b=48) == 2            # not a power of two
    assert h(b=16) == 2            # below the smallest block
    assert h(b=2048) == 2          # does not divide K
    assert h(K=128 * 3, b=256) == 2
    assert h(M=0) == 0
    assert h(Xq=None) == 1
    assert h(T=MISALIGNED) == 3


def test_weights_validation(L):
    w = lambda **kw: L.bitnet_quantize_weights(kw.get("W", ALIGNED), kw.get("dt", 0), kw.get("N", 16),
                                               kw.get("K", 64), kw.get("pk", ALIGNED), ALIGNED,
                                               kw.get("ws", ALIGNED), kw.get("wsb", 128), None)
    assert w(dt=2) == 4
    assert w(K=24) == 2 and w(N=0) == 2 and w(N=1 << 20, K=1 << 12) == 2
    assert w(N=1 << 40, K=1 << 40) == 2 and w(N=1 << 62, K=16) == 2      # products that would overflow
    assert w(ws=None) == 7 and w(wsb=8) == 7
    assert w(W=None) == 1
    assert w(pk=MISALIGNED) == 3


def test_bitlinear_validation(L):
    def b(**kw):
        a = dict(X=ALIGNED, dt=1, M=4, K=512, gamma=None, pkW=ALIGNED, s_w=ALIGNED, N=256, Y=ALIGNED, yt=0,
                 Xq=ALIGNED, s_x=ALIGNED)
        a.update(kw)
        return L.bitnet_bitlinear(a["X"], a["dt"], a["M"], a["K"], a["gamma"], 1e-6, a["pkW"], a["s_w"], a["N"],
                                  a["Y"], a["yt"], a["Xq"], a["s_x"], None)
    assert b(dt=2) == 4 and b(yt=3) == 4
    assert b(K=100) == 2 and b(K=64) == 2 and b(K=16384 + 128) == 2 and b(N=0) == 2 and b(M=-1) == 2
    assert b(M=0) == 0
    assert b(X=None) == 1 and b(Xq=None) == 1 and b(s_x=None) == 1 and b(Y=None) == 1 and b(pkW=None) == 1
    assert b(X=MISALIGNED) == 3 and b(Xq=MISALIGNED) == 3 and b(gamma=MISALIGNED) == 3
    assert b(s_x=ALIGNED + 2) == 3


def test_fused_quantiser_validation(L):
    aq = lambda **kw: L.bitnet_add_quant_act(kw.get("A", ALIGNED), kw.get("B", ALIGNED), kw.get("M", 4),
                                             kw.get("K", 256), None, 1e-6, kw.get("H", ALIGNED), ALIGNED, ALIGNED,
                                             None)
    assert aq(K=24) == 2 and aq(M=-1) == 2 and aq(M=0) == 0
    assert aq(B=None) == 1 and aq(H=None) == 1
    assert aq(A=MISALIGNED) == 3 and aq(H=MISALIGNED) == 3
    gh = lambda **kw: L.bitnet_glu_hadamard_quant_act(kw.get("g", ALIGNED), kw.get("u", ALIGNED), kw.get("M", 4),
                                                      kw.get("K", 1024), None, 1e-6, kw.get("b", 0), ALIGNED,
                                                      ALIGNED, None)
    assert gh(K=1000) == 2 and gh(b=48) == 2 and gh(K=16384, b=0) == 2 and gh(M=0) == 0
    assert gh(u=None) == 1 and gh(g=MISALIGNED) == 3


def test_trit5_validation(L):
    assert L.bitnet_trit5_row_bytes(2560) == 512 and L.bitnet_trit5_row_bytes(37) == 16
    assert L.bitnet_trit5_row_bytes(81) == 32 and L.bitnet_trit5_row_bytes(0) == 0
    rp = lambda **kw: L.bitnet_repack_trit5(kw.get("pk", ALIGNED), kw.get("N", 8), kw.get("K", 512),
                                            kw.get("out", ALIGNED), None)
    assert rp(K=24) == 2 and rp(K=0) == 2 and rp(N=0) == 2 and rp(N=1 << 62, K=1 << 20) == 2
    assert rp(pk=None) == 1 and rp(out=None) == 1
    assert rp(pk=MISALIGNED) == 3 and rp(out=MISALIGNED) == 3

    def lt(**kw):
        a = dict(Xq=ALIGNED, bits=8, s_x=ALIGNED, pk=ALIGNED, s_w=ALIGNED, M=4, N=256, K=2560, Y=ALIGNED, yt=0)
        a.update(kw)
        return L.bitnet_linear_trit5(a["Xq"], a["bits"], a["s_x"], a["pk"], a["s_w"], a["M"], a["N"], a["K"],
                                     a["Y"], a["yt"], None, None)
    assert lt(bits=2) == 4 and lt(yt=5) == 4
    assert lt(M=33) == 2 and lt(M=0) == 2 and lt(K=384) == 2 and lt(K=16384 + 512) == 2 and lt(N=0) == 2
    assert lt(pk=None) == 1 and lt(Y=None) == 1
    assert lt(pk=MISALIGNED) == 3 and lt(s_w=ALIGNED + 2) == 3


def test_linear_group_validation(L):
    import ctypes
    P, I64 = ctypes.c_void_p, ctypes.c_int64

    def grp(count=2, N=(256, 128), pk=ALIGNED, Y=ALIGNED, sw=ALIGNED, M=4, K=512, bits=8, yt=0, Xq=ALIGNED,
            n_arr=True):
        ptrs = lambda v: (P * 4)(*([v] * 4))
        Ns = (I64 * 4)(*(list(N) + [128] * (4 - len(N)))) if n_arr else None
        return L.bitnet_linear_group(Xq, bits, ALIGNED, M, K, count, ptrs(pk), ptrs(sw), Ns, ptrs(Y), yt, None)
    assert grp(bits=5) == 4 and grp(yt=2) == 4
    assert grp(count=0) == 2 and grp(count=5) == 2
    assert grp(K=100) == 2 and grp(N=(256, 0)) == 2 and grp(M=-1) == 2
    assert grp(M=0) == 0
    assert grp(n_arr=False) == 1 and grp(pk=None) == 1 and grp(Xq=None) == 1
    assert grp(pk=MISALIGNED) == 3 and grp(Y=MISALIGNED) == 3 and grp(sw=ALIGNED + 2) == 3


def test_kernel_choice_is_per_call(L):
    """The kernel family is an argument of the call (no process-wide switch):
    values outside the documented ones are refused before anything is enqueued."""
    lk = lambda kernel, **kw: L.bitnet_linear_kernel(ALIGNED, 8, ALIGNED, ALIGNED, ALIGNED, kw.get("M", 4), 256,
                                                     kw.get("K", 256), ALIGNED, 0, None, kernel, None)
    assert lk(6) == 2 and lk(-1) == 2
    assert lk(3, M=33, K=512) == 2 and lk(3, K=384) == 2          # outside the decode kernel's range
    assert lk(5) == 2 and lk(5, M=128, K=384) == 2                # persistent kernel: > 64 tokens, even K steps
    assert lk(1, M=0) == 0 and lk(2, M=0) == 0
    bk = lambda kernel, **kw: L.bitnet_bitlinear_kernel(ALIGNED, 1, kw.get("M", 4), kw.get("K", 512), None, 1e-6,
                                                        ALIGNED, ALIGNED, 256, ALIGNED, 0, ALIGNED, ALIGNED, kernel,
                                                        None)
    assert bk(5) == 2 and bk(-1) == 2 and bk(4, M=0) == 0
    assert not hasattr(api, "bitnet_set_linear_path")


def test_oracle_and_product_share_no_code():
    """The product package never imports the oracle, the oracle never imports the
    product, and the C++ oracle includes nothing from the CUDA sources."""
    import ast
    import glob
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

    def imports(path):
        tree = ast.parse(open(path).read())
        names = set()
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                names.update(a.name.split(".")[0] for a in node.names)
            elif isinstance(node, ast.ImportFrom) and node.module:
                names.add(node.module.split(".")[0])
        return names

    for path in glob.glob(os.path.join(root, "bitlinear_bitnet_quant_b200", "*.py")):
        assert "oracle" not in imports(path), path
    for path in glob.glob(os.path.join(root, "oracle", "*.py")):
        assert "bitlinear_bitnet_quant_b200" not in imports(path), path
    cpp = open(os.path.join(root, "oracle", "bitnet_oracle_ref.cpp")).read()
    assert "csrc" not in cpp and ".cuh" not in cpp and "bitnet.h" not in cpp
    for path in glob.glob(os.path.join(root, "bitlinear_bitnet_quant_b200", "csrc", "*")):
        assert "oracle" not in open(path).read().lower(), path


def test_python_binding_refuses_host_tensors():
    """No CPU fallback: every compute entry of the binding refuses host tensors
    before anything runs."""
    import torch
    from bitlinear_bitnet_quant_b200 import api
    x = torch.zeros(4, 512)
    w = torch.zeros(256, 512)
    pk = torch.zeros(256, 128, dtype=torch.uint8)
    sw = torch.ones(1)
    xq = torch.zeros(4, 512, dtype=torch.int8)
    sx = torch.ones(4)
    calls = [
        lambda: api.bitnet_quantize_weights(w),
        lambda: api.bitnet_quant_act(x),
        lambda: api.bitnet_hadamard_quant_act(x),
        lambda: api.bitnet_linear(xq, 8, sx, pk, sw),
        lambda: api.bitnet_bitlinear(x, pk, sw),
        lambda: api.bitnet_repack_trit5(pk),
        lambda: api.bitnet_linear_trit5(xq, 8, sx, torch.zeros(256, 112, dtype=torch.uint8), sw, 512),
        lambda: api.bitlinear_forward(x, pk, sw),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()
