"""Synthetic 24-layer decoder forward: 288 W4A4 GEMM calls per forward.

The workload of the "fp4-cuda-kernel" forum post (a 24-layer transformer,
288 GEMM calls per forward pass, weights quantized once at load,
activations quantized on the fly per call), with random-init weights and
the shapes of a 2880-hidden / 7680-FFN model:

  per layer  q, k, v, o             [2880 <- 2880]
             gate0, gate1, up0, up1 [3840 <- 2880]   (gate = [gate0 | gate1])
             down0 .. down3         [ 720 <- 7680]   (down = [down0 | ... | down3])
  => 12 GEMMs per layer, 288 per forward.

Glue between the GEMMs is kept minimal and runs in torch bf16 (it is not
part of the FP4 path): attention is replaced by passing v through (a
synthetic stand-in, there is no attention kernel here), the FFN is
silu(gate) * up, and both sub-blocks are residual with a 1/sqrt(2) scale so
the activations keep their magnitude over 24 layers without norms.  The
split GEMMs write straight into column slices of one output buffer (ldc =
the full width), so no concatenation runs.  Every GEMM call goes through
the library: fp4_gemm_fused for M <= 32 (activation quantized inside the
call chain), fp4_quantize_act + fp4_gemm otherwise, DYNAMIC global scale
per call.  The whole forward is captured once into a CUDA graph and replayed
("Hardware FP4 inference for speech on Blackwell": CUDA graphs decide
whether FP4 buys speed at small batch).

The bf16 reference runs the same layer structure with torch matmuls
(cuBLAS), gate/up/down each as one GEMM over the concatenated weights.
"""
from __future__ import annotations

import math

import torch

from . import inputs, ops

HIDDEN = 2880
FFN = 7680
LAYERS = 24
# (name, N, K) of the 12 GEMMs of a layer, in call order
LAYER_GEMMS = ([("q", HIDDEN, HIDDEN), ("k", HIDDEN, HIDDEN), ("v", HIDDEN, HIDDEN),
                ("o", HIDDEN, HIDDEN)] +
               [(f"gate{i}", FFN // 2, HIDDEN) for i in range(2)] +
               [(f"up{i}", FFN // 2, HIDDEN) for i in range(2)] +
               [(f"down{i}", HIDDEN // 4, FFN) for i in range(4)])
RES = 1.0 / math.sqrt(2.0)


class SyntheticDecoder:
    """Random-init weights ~ N(0, 0.02), quantized once (NVFP4 or MXFP4)."""

    def __init__(self, device, fmt: int = ops.NVFP4, layers: int = LAYERS, seed: int = 4,
                 keep_bf16: bool = True):
        self.device = torch.device(device)
        self.fmt = fmt
        self.layers = layers
        self.wq = []      # per layer: dict name -> ops.Quantized
        self.wb = []      # per layer: dict name -> bf16 weight (reference / checks)
        for li in range(layers):
            qd, bd = {}, {}
            for gi, (name, n, k) in enumerate(LAYER_GEMMS):
                w = inputs.random_bf16(seed * 1000 + li * 16 + gi, (n, k), 0.02).to(self.device)
                qd[name] = ops.quantize_weights(w, fmt)
                if keep_bf16:
                    bd[name] = w
            if keep_bf16:
                bd["gate"] = torch.cat([bd["gate0"], bd["gate1"]])
                bd["up"] = torch.cat([bd["up0"], bd["up1"]])
                bd["down"] = torch.cat([bd[f"down{i}"] for i in range(4)])
            self.wq.append(qd)
            self.wb.append(bd)
        self.record = None   # list of (layer, name, input, output) when set to a list

    # ------------------------------------------------------------ FP4 path
    def _gemm(self, li: int, name: str, x: torch.Tensor, out: torch.Tensor) -> torch.Tensor:
        w = self.wq[li][name]
        if x.shape[0] <= 32:
            ops.gemm_fused(x, w, out=out)
        else:
            ops.gemm(ops.quantize(x, self.fmt, ops.SCALES_MMA), w, out=out)
        if self.record is not None:
            self.record.append((li, name, x.clone(), out.clone()))
        return out

    def forward_fp4(self, x: torch.Tensor) -> torch.Tensor:
        M = x.shape[0]
        dev = x.device
        bf = torch.bfloat16
        for li in range(self.layers):
            t = torch.empty((M, HIDDEN), dtype=bf, device=dev)
            self._gemm(li, "q", x, t)
            self._gemm(li, "k", x, t)
            v = self._gemm(li, "v", x, torch.empty((M, HIDDEN), dtype=bf, device=dev))
            o = self._gemm(li, "o", v, torch.empty((M, HIDDEN), dtype=bf, device=dev))
            x = (x + o) * RES
            gate = torch.empty((M, FFN), dtype=bf, device=dev)
            up = torch.empty((M, FFN), dtype=bf, device=dev)
            for i in range(2):
                self._gemm(li, f"gate{i}", x, gate[:, i * (FFN // 2):(i + 1) * (FFN // 2)])
            for i in range(2):
                self._gemm(li, f"up{i}", x, up[:, i * (FFN // 2):(i + 1) * (FFN // 2)])
            h = torch.nn.functional.silu(gate) * up
            down = torch.empty((M, HIDDEN), dtype=bf, device=dev)
            for i in range(4):
                self._gemm(li, f"down{i}", h, down[:, i * (HIDDEN // 4):(i + 1) * (HIDDEN // 4)])
            x = (x + down) * RES
        return x

    # ------------------------------------------------- bf16 torch reference
    def forward_bf16(self, x: torch.Tensor) -> torch.Tensor:
        for li in range(self.layers):
            W = self.wb[li]
            x @ W["q"].T
            x @ W["k"].T
            v = x @ W["v"].T
            x = (x + v @ W["o"].T) * RES
            h = torch.nn.functional.silu(x @ W["gate"].T) * (x @ W["up"].T)
            x = (x + h @ W["down"].T) * RES
        return x

    # ------------------------------------------------------------- graphs
    def capture(self, fn, x_static: torch.Tensor):
        """Capture fn(x_static) into a CUDA graph; returns (graph, output)."""
        s = torch.cuda.Stream(device=self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            for _ in range(2):
                fn(x_static)                                 # warm-up: workspaces, attributes
        torch.cuda.current_stream(self.device).wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            out = fn(x_static)
        return g, out

    def weight_bytes(self) -> int:
        return sum(q.codes.numel() + q.scales.numel() for d in self.wq for q in d.values())

    def gemm_flops(self, M: int) -> float:
        return 2.0 * M * self.layers * sum(n * k for _, n, k in LAYER_GEMMS)
