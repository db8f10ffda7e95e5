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
part of the FP4 path): each sub-block reads an RMS-normalized copy of the
residual stream (pre-norm, no learned gain), attention is replaced by
passing v through (a synthetic stand-in, there is no attention kernel here),
the FFN is silu(gate) * up, and both sub-blocks add back into the residual
with a 1/sqrt(2) scale.  Without the norms the FFN's product of two
projections squares the magnitude layer after layer: from the seeded
weights the bf16 forward overflows to Inf by layer 8 and then turns to NaN;
with them the residual stream stays near unit RMS over all 24 layers.  The
split GEMMs write straight into column slices of one output buffer (ldc =
the full width), so no concatenation runs.  Every GEMM call goes through
the library: fp4_gemm_fused for M <= 32 (activation quantized inside the
call chain), fp4_quantize_act + fp4_gemm otherwise, DYNAMIC global scale
per call.  The whole forward is captured once into a CUDA graph and replayed
("Hardware FP4 inference for speech on Blackwell": CUDA graphs decide
whether FP4 buys speed at small batch).

The bf16 reference runs the same layer structure with torch matmuls
(cuBLAS), gate/up/down each as one GEMM over the concatenated weights.

Both forwards run the projections that share an input as concurrent
branches of the graph (side streams forked from and joined back into the
caller's stream): q | k | v, then gate0 | gate1 | up0 | up1 (bf16: gate |
up), then down0 .. down3 (bf16: one GEMM).  At decode sizes each call is
mostly fixed latency, which the branches overlap.  Each fp4_gemm of an
n-way group chooses its launch shape for 1/n of the SMs (max_sms), so that
the group's CTAs run side by side instead of queueing.
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


def _norm(x: torch.Tensor) -> torch.Tensor:
    """Pre-norm of a sub-block's input: RMS normalization over the hidden
    dimension, no learned gain (torch glue, bf16)."""
    return torch.nn.functional.rms_norm(x, (x.shape[-1],))


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
        # side streams for the concurrent branches of a layer, and one
        # library workspace per branch (concurrent calls must not share one)
        self.side = [torch.cuda.Stream(device=self.device) for _ in range(3)]
        self.ws = [None] * 4
        self.branch = 0   # index of the branch the next _gemm call runs in
        # the SMs each GEMM of an n-way branch group chooses its launch shape
        # for (its share of the device; 0 = all, outside the groups)
        self.sms = torch.cuda.get_device_properties(self.device).multi_processor_count
        self.max_sms = 0

    def _branches(self, fns):
        """Run fns[0] on the current stream and fns[i] on side stream i-1,
        all after the work already queued, and join them back."""
        cur = torch.cuda.current_stream(self.device)
        for s in self.side[:len(fns) - 1]:
            s.wait_stream(cur)
        outs = [None] * len(fns)
        self.max_sms = self.sms // len(fns) if len(fns) > 1 else 0
        for i, fn in enumerate(fns[1:]):
            with torch.cuda.stream(self.side[i]):
                self.branch = i + 1
                outs[i + 1] = fn()
        self.branch = 0
        outs[0] = fns[0]()
        for s in self.side[:len(fns) - 1]:
            cur.wait_stream(s)
        self.max_sms = 0
        return outs

    def _ws(self, M: int, N: int, K: int) -> torch.Tensor:
        """This branch's workspace, grown outside graph capture only (the
        forward runs eagerly before it is captured)."""
        need = ops.L.fp4_workspace_bytes(M, N, K, self.fmt)
        b = self.branch
        if self.ws[b] is None or self.ws[b].numel() < need:
            if torch.cuda.is_current_stream_capturing():
                raise RuntimeError("decoder workspace must be sized before capture")
            self.ws[b] = torch.empty(max(need, 1 << 16), dtype=torch.uint8, device=self.device)
        return self.ws[b]

    # ------------------------------------------------------------ FP4 path
    def _gemm(self, li: int, name: str, x: torch.Tensor, out: torch.Tensor) -> torch.Tensor:
        w = self.wq[li][name]
        ws = self._ws(x.shape[0], w.rows, w.K)
        if x.shape[0] <= 32:
            ops.gemm_fused(x, w, out=out, ws=ws, max_sms=self.max_sms)
        else:
            ops.gemm(ops.quantize(x, self.fmt, ops.SCALES_MMA, ws=ws), w, out=out,
                     max_sms=self.max_sms)
        if self.record is not None:
            self.record.append((li, name, x.clone(), out.clone()))
        return out

    def forward_fp4(self, x: torch.Tensor) -> torch.Tensor:
        M = x.shape[0]
        dev = x.device
        bf = torch.bfloat16
        for li in range(self.layers):
            tq = torch.empty((M, HIDDEN), dtype=bf, device=dev)
            tk = torch.empty((M, HIDDEN), dtype=bf, device=dev)
            v = torch.empty((M, HIDDEN), dtype=bf, device=dev)
            xn = _norm(x)
            self._branches([lambda: self._gemm(li, "v", xn, v),
                            lambda: self._gemm(li, "q", xn, tq),
                            lambda: self._gemm(li, "k", xn, tk)])
            o = self._gemm(li, "o", v, torch.empty((M, HIDDEN), dtype=bf, device=dev))
            x = (x + o) * RES
            gate = torch.empty((M, FFN), dtype=bf, device=dev)
            up = torch.empty((M, FFN), dtype=bf, device=dev)
            half = FFN // 2
            xn = _norm(x)
            self._branches([lambda i=i, t=t, name=name: self._gemm(li, f"{name}{i}", xn,
                                                                   t[:, i * half:(i + 1) * half])
                            for name, t in (("gate", gate), ("up", up)) for i in range(2)])
            h = torch.nn.functional.silu(gate) * up
            down = torch.empty((M, HIDDEN), dtype=bf, device=dev)
            q4 = HIDDEN // 4
            self._branches([lambda i=i: self._gemm(li, f"down{i}", h, down[:, i * q4:(i + 1) * q4])
                            for i in range(4)])
            x = (x + down) * RES
        return x

    # ------------------------------------------------- bf16 torch reference
    def forward_bf16(self, x: torch.Tensor) -> torch.Tensor:
        for li in range(self.layers):
            W = self.wb[li]
            xn = _norm(x)
            v, _, _ = self._branches([lambda: xn @ W["v"].T, lambda: xn @ W["q"].T,
                                      lambda: xn @ W["k"].T])
            x = (x + v @ W["o"].T) * RES
            xn = _norm(x)
            g, u = self._branches([lambda: xn @ W["gate"].T, lambda: xn @ W["up"].T])
            h = torch.nn.functional.silu(g) * u
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
