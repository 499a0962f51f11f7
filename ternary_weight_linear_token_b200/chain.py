"""Decode chain: a stack of decoder layers' BitLinear projections run for one
token (M = 1), each projection re-quantising its own input per token.

Per layer: q = BitLinear_qkv(x)[:, :d]; o = BitLinear_o(q);
u = ReLU^2(BitLinear_up(o)); d = BitLinear_down(u); x <- rms_norm(d).

Attention, RoPE and the KV cache are not part of the BitLinear path; the first
d columns of the fused QKV output stand in for the attention output.  The
model card (BitNet b1.58 2B4T, 模型详情 -> 架构) names ReLU^2 in the FFN and a
"subln" normalisation without giving its formula; the weightless RMS
normalisation between layers is the plain stand-in (without it the squared
activations vanish within a few layers).

Every step is a call of the C-ABI library on one stream; ``run`` launches
5 kernels per layer and can be captured in a CUDA graph (``capture``).
"""

from __future__ import annotations

import torch

from . import bitnet_quantize_weights, bitnet_rms_norm, bitnet_w158a8_matmul


class DecodeChain:
    def __init__(self, weights, device="cuda:0", weights_static: bool = True):
        """weights: list over layers of a list of 4 (W [N, K] float tensor,
        relu2) pairs in the order qkv, o, up, down.  Weights are quantised on
        the device once, here."""
        self.device = torch.device(device)
        self.weights_static = weights_static
        self.layers = []
        for layer in weights:
            proj = []
            for W, relu2 in layer:
                W = W.to(self.device).contiguous()
                packed, gamma = bitnet_quantize_weights(W)
                proj.append(dict(packed=packed, gamma=gamma, N=W.shape[0], K=W.shape[1],
                                 relu2=relu2))
            self.layers.append(proj)
        d = self.layers[0][1]["K"]
        self.d = d
        # activation buffers, one per step, kept so every link can be checked
        self.x_in = torch.zeros((1, d), dtype=torch.bfloat16, device=self.device)
        self.outs = []
        for proj in self.layers:
            bufs = [torch.empty((1, p["N"]), dtype=torch.bfloat16, device=self.device) for p in proj]
            bufs.append(torch.empty((1, d), dtype=torch.bfloat16, device=self.device))  # norm out
            self.outs.append(bufs)
        self.graph = None

    @property
    def packed_bytes(self) -> int:
        return sum(p["packed"].numel() for layer in self.layers for p in layer)

    def _bl(self, x, p, y):
        bitnet_w158a8_matmul(x, p["packed"], p["gamma"], relu2=p["relu2"], Y=y,
                             weights_static=self.weights_static)

    def run(self, x0: torch.Tensor | None = None) -> torch.Tensor:
        if x0 is not None:
            self.x_in.copy_(x0)
        x = self.x_in
        for proj, bufs in zip(self.layers, self.outs):
            qkv, o, up, down = proj
            self._bl(x, qkv, bufs[0])
            q = bufs[0][:, : self.d]          # contiguous for one token
            self._bl(q, o, bufs[1])
            self._bl(bufs[1], up, bufs[2])
            self._bl(bufs[2], down, bufs[3])
            bitnet_rms_norm(bufs[3], Y=bufs[4])
            x = bufs[4]
        return x

    def capture(self) -> torch.cuda.CUDAGraph:
        """Capture one token through the whole stack in a CUDA graph."""
        s = torch.cuda.Stream(self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            self.run()  # warm-up outside capture
        torch.cuda.current_stream(self.device).wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run()
        self.graph = g
        return g

    def launches_per_token(self) -> int:
        return 5 * len(self.layers)
