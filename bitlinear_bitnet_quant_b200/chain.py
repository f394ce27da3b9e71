"""Stacked BitLinear layers through the C ABI.

One layer, as the BitNet pages describe the model around BitLinear: the
linear layers of attention and FFN are BitLinear (int8 activations), and in
BitNet v2 the O and down projections are H-BitLinear (Hadamard + int4).
Per layer, with fp32 residuals:

    q, k, v = BitLinear(x)                      (one int8 quantisation of x,
                                                 one launch for the three)
    o = H-BitLinear(attention(q, k, v))         (rotary embedding, key/value
                                                 cache, causal softmax; without
                                                 a cache, a one-token context,
                                                 which returns V)
    h = x + o
    up, gate = BitLinear(h)                     (one int8 quantisation of h,
                                                 one launch for the two)
    a = relu(gate)^2 * up                       (squared-ReLU gated unit)
    x' = h + H-BitLinear(a)                     (down projection)

Every step is a kernel of libbitnet.so; this module only sequences the calls
and owns the activation buffers (allocated once per batch size).  The
element-wise steps run inside the quantiser that consumes them: h = x + o in
the quantisation of h, a in the Hadamard quantisation of a, and x' = h + d
in the next layer's first quantisation (a final add after the last layer).
"""
from __future__ import annotations

import torch

from . import api

PROJ = ("q", "k", "v", "o", "up", "gate", "down")
H_BITS = {"o": 4, "down": 4}


def quantize_layer(weights: dict, stream=None) -> dict:
    """fp32/bf16 device weights {name: [N, K]} -> {name: (packed, s_w)}."""
    return {name: api.bitnet_quantize_weights(weights[name].contiguous(), stream=stream) for name in PROJ}


class BitLinearChain:
    """Runs a list of quantised layers on a batch of M tokens of width `hidden`.

    attention=None: the attention core over a one-token context (O's input is V).
    attention=dict(B=..., L=..., T_cap=..., heads=...): the M = B*L rows are B
    sequences of L tokens each; every layer keeps a key/value cache
    [B, T_cap, hidden] (allocated here) and runs rotary embedding, the cache
    append and causal softmax attention; forward(x, t0) places the step's
    tokens at positions t0 .. t0+L-1."""

    def __init__(self, layers: list, M: int, hidden: int, ffn: int, device, eps: float = 1e-6, attention=None):
        self.layers = layers
        self.M, self.hidden, self.ffn, self.eps = M, hidden, ffn, eps
        self.attention = attention
        if attention is not None:
            B, L, T_cap = attention["B"], attention["L"], attention["T_cap"]
            assert B * L == M and L <= T_cap
            self.heads = attention.get("heads", 16)
            self.rope_base = attention.get("base", 10000.0)
            self.kc = [torch.empty((B, T_cap, hidden), dtype=torch.float32, device=device) for _ in layers]
            self.vc = [torch.empty((B, T_cap, hidden), dtype=torch.float32, device=device) for _ in layers]
            self.att = torch.empty((M, hidden), dtype=torch.float32, device=device)
        self.t0 = 0
        f32 = dict(dtype=torch.float32, device=device)
        e = lambda *shape: torch.empty(shape, **f32)
        self.x = [e(M, hidden), e(M, hidden)]          # layer input, chain output
        self.xq = torch.empty((M, hidden), dtype=torch.int8, device=device)
        self.sx = e(M)
        self.q, self.k, self.v, self.o, self.h, self.d = (e(M, hidden) for _ in range(6))
        self.v4 = torch.empty((M, hidden // 2), dtype=torch.uint8, device=device)
        self.sv = e(M)
        self.hq = torch.empty((M, hidden), dtype=torch.int8, device=device)
        self.sh = e(M)
        self.up, self.gate = e(M, ffn), e(M, ffn)
        self.a4 = torch.empty((M, ffn // 2), dtype=torch.uint8, device=device)
        self.sa = e(M)

    def layer(self, x_parts, w: dict, stream=None, index: int = 0):
        """One layer.  x_parts: (x,) or (h_prev, d_prev), whose sum is the
        layer input.  Returns (h, d), whose sum is the layer output.  Buffers
        are reused from layer to layer: every kernel waits for the one before
        it, so a buffer is rewritten only after its last reader has finished."""
        A, s = api, stream
        if len(x_parts) == 1:
            x = x_parts[0]
            A.bitnet_quant_act(x, None, self.eps, Xq=self.xq, s_x=self.sx, stream=s)
        else:
            x = self.x[0]
            A.bitnet_add_quant_act(x_parts[0], x_parts[1], None, self.eps, H=x, Xq=self.xq, s_x=self.sx, stream=s)
        A.bitnet_linear_group(self.xq, 8, self.sx, [w["q"], w["k"], w["v"]], Ys=[self.q, self.k, self.v], stream=s)
        if self.attention is None:
            att = self.v                                   # a one-token context returns V
        else:
            B, L = self.attention["B"], self.attention["L"]
            A.bitnet_rope_append(self.q, self.k, self.v, self.kc[index], self.vc[index], B, L, self.t0, self.heads,
                                 self.rope_base, stream=s)
            att = A.bitnet_attention(self.q, self.kc[index], self.vc[index], B, L, self.t0, self.heads, A=self.att,
                                     stream=s)
        A.bitnet_hadamard_quant_act(att, None, self.eps, 0, Xq4=self.v4, s_x=self.sv, stream=s)
        A.bitnet_linear(self.v4, 4, self.sv, *w["o"], Y=self.o, stream=s)
        A.bitnet_add_quant_act(x, self.o, None, self.eps, H=self.h, Xq=self.hq, s_x=self.sh, stream=s)
        A.bitnet_linear_group(self.hq, 8, self.sh, [w["up"], w["gate"]], Ys=[self.up, self.gate], stream=s)
        A.bitnet_glu_hadamard_quant_act(self.gate, self.up, None, self.eps, 0, Xq4=self.a4, s_x=self.sa, stream=s)
        A.bitnet_linear(self.a4, 4, self.sa, *w["down"], Y=self.d, stream=s)
        return self.h, self.d

    def forward(self, x: torch.Tensor, stream=None, t0: int = 0) -> torch.Tensor:
        """x: [M, hidden] fp32 on the device; returns the last layer's output
        (one of the chain's own buffers).  t0: position of each sequence's first
        token in this step (with attention)."""
        self.t0 = t0
        parts = (x,)
        for i, w in enumerate(self.layers):
            parts = self.layer(parts, w, stream, i)
        api.bitnet_add(parts[0], parts[1], out=self.x[1], stream=stream)
        return self.x[1]

    # kernels launched per forward: per layer 2 int8 quantisers (the second, and
    # from the second layer on the first, with the residual add folded in), 4
    # linear launches (Q/K/V in one, O, up/gate in one, down), 2 Hadamard
    # quantisers (one with the gated unit folded in); one residual add after
    # the last layer
    @property
    def launches(self) -> int:
        return (8 if self.attention is None else 10) * len(self.layers) + 1

    def packed_bytes(self) -> int:
        return sum(pk.numel() for w in self.layers for pk, _ in w.values())
