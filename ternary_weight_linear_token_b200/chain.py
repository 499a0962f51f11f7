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

Two ways to run it, both through the C-ABI library on one stream and both
capturable in a CUDA graph (``capture``):
  * per launch (default): ``run`` makes one call per projection, 4 kernels
    per layer (each layer's QKV call normalises its input itself,
    ``bitnet_rms_norm_w158a8_matmul``) plus one normalisation at the end;
  * persistent (``persistent=True``): ``run`` makes one call of
    ``bitnet_decode_chain``, one kernel for the whole stack, with the
    normalisation folded into the next layer's QKV projection.
Both fill the same buffers (``outs``), so every link can be checked.
"""

from __future__ import annotations

import torch

from . import (bitnet_decode_chain, bitnet_decode_chain_steps, bitnet_decode_chain_workspace_size,
               bitnet_quantize_weights, bitnet_rms_norm, bitnet_rms_norm_w158a8_matmul,
               bitnet_w158a8_matmul)


class DecodeChain:
    def __init__(self, weights, device="cuda:0", weights_static: bool = True,
                 persistent: bool = False, quantized=None):
        """weights: list over layers of a list of 4 (W [N, K] float tensor,
        relu2) pairs in the order qkv, o, up, down (any iterable: a
        generator keeps only one layer's latent weights alive at a time).
        Weights are quantised on the device once, here.
        quantized: instead of weights, the ``layers`` of another DecodeChain
        (packed weights shared, nothing quantised again)."""
        self.device = torch.device(device)
        self.weights_static = weights_static
        if quantized is not None:
            self.layers = quantized
        else:
            self.layers = []
            for layer in weights:
                proj = []
                for W, relu2 in layer:
                    W = W.to(self.device).contiguous()
                    packed, gamma = bitnet_quantize_weights(W)
                    proj.append(dict(packed=packed, gamma=gamma, N=W.shape[0], K=W.shape[1],
                                     relu2=relu2))
                    del W
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
        self.persistent = persistent
        if persistent:
            steps = []
            for li, (proj, bufs) in enumerate(zip(self.layers, self.outs)):
                for pi, p in enumerate(proj):
                    step = dict(packed=p["packed"], gamma=p["gamma"], Y=bufs[pi], relu2=p["relu2"])
                    if pi == 0 and li > 0:  # the previous layer's normalisation, folded in
                        step.update(norm_in=True, X_normed=self.outs[li - 1][4])
                    steps.append(step)
            self._steps = bitnet_decode_chain_steps(steps)
            self._keep = steps
            self.workspace = torch.zeros(bitnet_decode_chain_workspace_size(self._steps),
                                         dtype=torch.uint8, device=self.device)

    @property
    def packed_bytes(self) -> int:
        return sum(p["packed"].numel() for layer in self.layers for p in layer)

    def _bl(self, x, p, y):
        bitnet_w158a8_matmul(x, p["packed"], p["gamma"], relu2=p["relu2"], Y=y,
                             weights_static=self.weights_static)

    def run(self, x0: torch.Tensor | None = None) -> torch.Tensor:
        if x0 is not None:
            self.x_in.copy_(x0)
        if self.persistent:
            bitnet_decode_chain(self._steps, self.x_in, self.workspace, y_norm=self.outs[-1][4])
            return self.outs[-1][4]
        for li, (proj, bufs) in enumerate(zip(self.layers, self.outs)):
            qkv, o, up, down = proj
            if li == 0:
                self._bl(self.x_in, qkv, bufs[0])
            else:  # the previous layer's normalisation, inside this call
                prev = self.outs[li - 1]
                bitnet_rms_norm_w158a8_matmul(prev[3], qkv["packed"], qkv["gamma"],
                                              X_normed=prev[4], relu2=qkv["relu2"], Y=bufs[0],
                                              weights_static=self.weights_static)
            q = bufs[0][:, : self.d]          # contiguous for one token
            self._bl(q, o, bufs[1])
            self._bl(bufs[1], up, bufs[2])
            self._bl(bufs[2], down, bufs[3])
        last = self.outs[-1]
        bitnet_rms_norm(last[3], Y=last[4])
        return last[4]

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
        return 1 if self.persistent else 4 * len(self.layers) + 1
