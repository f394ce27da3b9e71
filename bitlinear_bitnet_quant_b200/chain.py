"""Stacked BitLinear layers through the C ABI.

One layer, as the BitNet pages describe the model around BitLinear: the
linear layers of attention and FFN are BitLinear (int8 activations), and in
BitNet v2 the O and down projections are H-BitLinear (Hadamard + int4).
Per layer, with fp32 residuals:

    q, k, v = BitLinear(x)                      (one int8 quantisation of x,
                                                 in q's call; k, v reuse it)
    o = H-BitLinear(v)                          (attention over a one-token
                                                 context returns V)
    h = x + o
    up, gate = BitLinear(h)                     (one int8 quantisation of h,
                                                 in up's call; gate reuses it)
    a = relu(gate)^2 * up                       (squared-ReLU gated unit)
    x' = h + H-BitLinear(a)                     (down projection)

Every step is a kernel of libbitnet.so; this module only sequences the calls
and owns the activation buffers (allocated once per batch size).
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
    """Runs a list of quantised layers on a batch of M tokens of width `hidden`."""

    def __init__(self, layers: list, M: int, hidden: int, ffn: int, device, eps: float = 1e-6):
        self.layers = layers
        self.M, self.hidden, self.ffn, self.eps = M, hidden, ffn, eps
        f32 = dict(dtype=torch.float32, device=device)
        e = lambda *shape: torch.empty(shape, **f32)
        self.x = [e(M, hidden), e(M, hidden)]          # ping-pong layer inputs
        self.xq = torch.empty((M, hidden), dtype=torch.int8, device=device)
        self.sx = e(M)
        self.q, self.k, self.v, self.o, self.h, self.d = (e(M, hidden) for _ in range(6))
        self.v4 = torch.empty((M, hidden // 2), dtype=torch.uint8, device=device)
        self.sv = e(M)
        self.hq = torch.empty((M, hidden), dtype=torch.int8, device=device)
        self.sh = e(M)
        self.up, self.gate, self.a = e(M, ffn), e(M, ffn), e(M, ffn)
        self.a4 = torch.empty((M, ffn // 2), dtype=torch.uint8, device=device)
        self.sa = e(M)

    def layer(self, x: torch.Tensor, w: dict, out: torch.Tensor, stream=None) -> torch.Tensor:
        A, s = api, stream
        # q: bitnet_bitlinear quantises x (codes and scales kept for k, v)
        A.bitnet_bitlinear(x, *w["q"], None, self.eps, Y=self.q, Xq=self.xq, s_x=self.sx, stream=s)
        for name, Y in (("k", self.k), ("v", self.v)):
            A.bitnet_linear(self.xq, 8, self.sx, *w[name], Y=Y, stream=s)
        A.bitnet_hadamard_quant_act(self.v, None, self.eps, 0, Xq4=self.v4, s_x=self.sv, stream=s)
        A.bitnet_linear(self.v4, 4, self.sv, *w["o"], Y=self.o, stream=s)
        A.bitnet_add(x, self.o, out=self.h, stream=s)
        A.bitnet_bitlinear(self.h, *w["up"], None, self.eps, Y=self.up, Xq=self.hq, s_x=self.sh, stream=s)
        A.bitnet_linear(self.hq, 8, self.sh, *w["gate"], Y=self.gate, stream=s)
        A.bitnet_relu2_glu(self.gate, self.up, out=self.a, stream=s)
        A.bitnet_hadamard_quant_act(self.a, None, self.eps, 0, Xq4=self.a4, s_x=self.sa, stream=s)
        A.bitnet_linear(self.a4, 4, self.sa, *w["down"], Y=self.d, stream=s)
        A.bitnet_add(self.h, self.d, out=out, stream=s)
        return out

    def forward(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        """x: [M, hidden] fp32 on the device; returns the last layer's output
        (one of the chain's own buffers)."""
        cur = x
        for i, w in enumerate(self.layers):
            cur = self.layer(cur, w, self.x[i % 2], stream)
        return cur

    # kernels launched per forward: per layer 2 BitLinear calls (a quantiser
    # and a linear layer each), 5 further linear layers, 2 Hadamard
    # quantisers, 2 adds, 1 gated unit
    @property
    def launches(self) -> int:
        return 14 * len(self.layers)

    def packed_bytes(self) -> int:
        return sum(pk.numel() for w in self.layers for pk, _ in w.values())
