"""One streaming denoise step of a 30-layer 5B-style video DiT on the NVFP4
W4A4 path: the device state and the launch sequence the benchmark times and
the composed-step parity test checks.

Per layer, on a 3-frame chunk of 2640 tokens (dim 3072, 24 heads x 128, FFN
14336): quantize the layer input -> QKV GEMM (N = 9216) -> kv_quant_chunk of
the 3 new frames' K and V straight out of the QKV output -> kv_dequant_window
over 12 cached frames (3 sinks + 9 window) -> quantize the attention-output
stand-in -> out-projection GEMM -> quantize -> FFN-up GEMM (N = 14336) with the
GELU (tanh form) in its epilogue -> requantize the intermediate -> FFN-down
GEMM, whose output feeds the next layer.  The W4A4 linear layers and the NVFP4
KV cache are the tailorednewshub.com LongLive-2.0 article's "Inferencia W4A4
NVFP4"; the KV cache in frame blocks rebuilt for windowed attention is the
hyper.ai summary's "方法"; 3 sinks + 9 window frames are 171host.com section
2.2.  Attention, norms and residuals are not NVFP4 work and are not run: the
attention output is a fixed seeded tensor.

Every launch goes through the C ABI (ops.py marshals pointers); no step of the
path runs in Python.
"""
from __future__ import annotations

from typing import Dict, List, Optional

import torch

from . import ops as nv
from . import workloads as wl

M = wl.CHUNK_TOKENS          # 2640
D = wl.DIM                   # 3072
F = wl.FFN                   # 14336
QKV = wl.QKV_N               # 9216
TPF = wl.TOKENS_PER_FRAME    # 880
NEW_FRAMES = wl.CHUNK_FRAMES  # 3
WINDOW = wl.SINK_FRAMES + wl.WINDOW_FRAMES  # 12
POOL = WINDOW + NEW_FRAMES   # 15 slots per layer

GEMM_SHAPES = {"qkv": (M, QKV, D), "out": (M, D, D), "up": (M, F, D), "down": (M, D, F)}
GEMM_FLOPS_LAYER = sum(2 * m * n * k for (m, n, k) in GEMM_SHAPES.values())

# what a tapped layer copies out, in launch order (see DiTStep.run)
TAP_NAMES = ("x", "qa_x", "qkv", "k_win", "v_win", "qa_attn", "o", "qa_o", "up", "qf", "down")


def _tap_like(t):
    if isinstance(t, nv.NVFP4Tensor):
        return nv.NVFP4Tensor(codes=torch.empty_like(t.codes), sf=torch.empty_like(t.sf),
                              s_t=torch.empty_like(t.s_t), rows=t.rows, cols=t.cols,
                              sf_layout=t.sf_layout)
    return torch.empty_like(t)


def _copy(dst, src):
    if isinstance(src, nv.NVFP4Tensor):
        dst.codes.copy_(src.codes)
        dst.sf.copy_(src.sf)
        dst.s_t.copy_(src.s_t)
    else:
        dst.copy_(src)


class DiTStep:
    """Device state of the denoise step (weights pre-quantized, KV pools
    prefilled with 12 seeded frames per layer) and its launch sequence."""

    def __init__(self, layers: int, device):
        self.layers = layers
        self.dev = device
        self.w: List[List[nv.NVFP4Tensor]] = []   # per layer: qkv, out, up, down
        self.cache: List[nv.KVCache] = []
        for l in range(layers):
            ws_bf16 = wl.layer_weights_cuda(l, device=device)
            self.w.append([nv.quantize(t) for t in ws_bf16])
            del ws_bf16
            c = nv.KVCache(POOL, TPF, wl.HEADS, wl.HEAD_DIM, device=device)
            # prefill the 12 cached frames (sinks + window) with seeded K/V,
            # in chunks of 8 and 4 frames
            kv = wl.kv_tensor_cuda(seed=l, tokens=WINDOW * TPF, device=device)
            for f0 in (0, 8):
                nf = min(8, WINDOW - f0)
                sl = kv[f0 * TPF:(f0 + nf) * TPF]
                c.quant_chunk(sl, sl, list(range(f0, f0 + nf)))
            self.cache.append(c)
        torch.cuda.synchronize(device)
        self.x_in = wl.activations(c=5, i=0).to(device)          # step input
        self.attn = wl.randn((M, D), 5, 1).to(device)           # attention-output stand-in
        self.qkv_out = torch.empty(M, QKV, dtype=torch.bfloat16, device=device)
        self.o_out = torch.empty(M, D, dtype=torch.bfloat16, device=device)
        self.up_out = torch.empty(M, F, dtype=torch.bfloat16, device=device)
        self.down_out = [torch.empty(M, D, dtype=torch.bfloat16, device=device) for _ in range(2)]
        self.k_win = torch.empty(WINDOW * TPF, wl.HEADS, wl.HEAD_DIM, dtype=torch.bfloat16,
                                 device=device)
        self.v_win = torch.empty_like(self.k_win)
        self.qa = nv.empty(M, D, device=device)
        self.qf = nv.empty(M, F, device=device)
        self.ws = nv.workspace(device)
        # max|C| words handed from a GEMM epilogue to the quantization of its
        # output: [0] down -> next layer's input, [1] out-proj, [2] FFN up,
        # [3..5] the Q, K, V thirds of the QKV projection (K, V -> KV chunk)
        self.amax = torch.zeros(6, dtype=torch.float32, device=device)
        self.new_slots = list(range(WINDOW, POOL))
        # sinks (slots 0-2), the 6 older window frames (slots 6-11; slots 3-5
        # hold frames that left the window), then the chunk's own 3 frames
        self.window = list(range(wl.SINK_FRAMES)) + \
            list(range(wl.SINK_FRAMES + NEW_FRAMES, WINDOW)) + self.new_slots
        assert len(self.window) == WINDOW

    def output(self) -> torch.Tensor:
        return self.down_out[(self.layers - 1) % 2]

    def layer_input(self, l: int) -> torch.Tensor:
        """The tensor layer l reads (valid while later layers have not
        overwritten it: layer l's input is layer l-1's output)."""
        return self.x_in if l == 0 else self.down_out[(l - 1) % 2]

    def make_taps(self, layers) -> Dict[int, Dict[str, object]]:
        """Buffers for run(taps=...): one copy of every intermediate of each
        listed layer."""
        src = {"x": self.x_in, "qa_x": self.qa, "qkv": self.qkv_out, "k_win": self.k_win,
               "v_win": self.v_win, "qa_attn": self.qa, "o": self.o_out, "qa_o": self.qa,
               "up": self.up_out, "qf": self.qf, "down": self.down_out[0]}
        return {l: {n: _tap_like(src[n]) for n in TAP_NAMES} for l in layers}

    def run(self, mark=None, taps: Optional[Dict[int, Dict[str, object]]] = None):
        """Enqueue one step on the current stream.

        mark(name), optional, is called before each launch group and once at
        the end with None (the bench records events there).  taps, optional:
        {layer: buffers from make_taps}; for those layers every intermediate
        is copied out right after the launch that wrote it (device-to-device
        copies on the same stream; the other layers are untouched)."""
        mk = mark or (lambda name: None)
        taps = taps or {}
        x = self.x_in
        a_x, a_o, a_u = self.amax[0:1], self.amax[1:2], self.amax[2:3]
        for l in range(self.layers):
            tap = taps.get(l)

            def tp(name, src):
                if tap is not None:
                    _copy(tap[name], src)

            wq, wo, wu, wd = self.w[l]
            tp("x", x)
            mk("quant_act")
            # layer 0's input has no producer in the step: it takes the amax pass
            nv.quantize(x, out=self.qa, ws=self.ws, amax_in=a_x if l > 0 else None)
            tp("qa_x", self.qa)
            mk("gemm_qkv")
            nv.gemm(self.qa, wq, out=self.qkv_out, ws=self.ws, c_amax=self.amax[3:6],
                    c_amax_cols=D)
            tp("qkv", self.qkv_out)
            mk("kv_quant")
            self.cache[l].quant_chunk(self.qkv_out[:, D:2 * D], self.qkv_out[:, 2 * D:],
                                      self.new_slots, ws=self.ws, k_amax_in=self.amax[4:5],
                                      v_amax_in=self.amax[5:6])
            mk("kv_dequant")
            self.cache[l].dequant_window(self.window, self.k_win, self.v_win)
            tp("k_win", self.k_win)
            tp("v_win", self.v_win)
            mk("quant_act")
            nv.quantize(self.attn, out=self.qa, ws=self.ws)
            tp("qa_attn", self.qa)
            mk("gemm_out")
            nv.gemm(self.qa, wo, out=self.o_out, ws=self.ws, c_amax=a_o)
            tp("o", self.o_out)
            mk("quant_act")
            nv.quantize(self.o_out, out=self.qa, ws=self.ws, amax_in=a_o)
            tp("qa_o", self.qa)
            mk("gemm_up")
            # FFN up-projection with its GELU in the epilogue; the stored GELU
            # output's amax feeds the intermediate requantization
            nv.gemm(self.qa, wu, out=self.up_out, ws=self.ws, c_amax=a_u,
                    act=nv.N.ACT_GELU_TANH)
            tp("up", self.up_out)
            mk("requant_ffn")
            nv.quantize(self.up_out, out=self.qf, ws=self.ws, amax_in=a_u)
            tp("qf", self.qf)
            mk("gemm_down")
            x = self.down_out[l % 2]
            # the last layer's output is not quantized within the step
            last = l == self.layers - 1
            nv.gemm(self.qf, wd, out=x, ws=self.ws, c_amax=None if last else a_x)
            tp("down", x)
        mk(None)

    # kernels launched per step: a quantize with its own amax pass 2 (layer 0's
    # input, the attention output), one fed by a GEMM's c_amax 1, gemm 1,
    # kv_quant 1 (its amax comes from the QKV GEMM), kv_dequant 1
    def launches_per_step(self) -> int:
        return self.layers * (2 + 1 + 1 + 1 + 4 * 1 + 1 + 1) + 1
