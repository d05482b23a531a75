"""Seeded synthetic inputs shaped like a 5B causal video DiT at 1280x720.

This module holds input generators only -- no step of the NVFP4 method.  The
tests feed the same tensors to the CUDA library and to the CPU oracle, and the
bench harness draws its workloads here.

Geometry (a Wan2.2-TI2V-5B-style DiT): model width 3072, 24 heads x 128,
FFN width 14336, 30 layers; one latent frame of 1280x720 video is 880 tokens;
a generation chunk is 3 latent frames (2640 tokens); the attention window is 9
local + 3 sink frames (171host.com LongLive 2.0 teardown, section 2.2), and
the KV cache is quantized in chunks of up to 8 frames (hyper.ai LongLive-2.0
summary, Method section).

Every tensor i of workload c is drawn from torch.Generator('cpu') seeded with
1000 + 100*c + i, as float32, then rounded to bfloat16 (RNE) where the
workload is bf16.  The 30-layer weights of the denoise step are drawn on the
GPU (a CUDA generator seeded per layer) because 3.8 G CPU normals would take
minutes; the tests that compare those layers copy the same tensors back.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

DIM = 3072
HEADS = 24
HEAD_DIM = 128
FFN = 14336
LAYERS = 30
TOKENS_PER_FRAME = 880
CHUNK_FRAMES = 3
CHUNK_TOKENS = CHUNK_FRAMES * TOKENS_PER_FRAME  # 2640
SINK_FRAMES = 3
WINDOW_FRAMES = 9
KV_BLOCK_FRAMES = 8
QKV_N = 3 * DIM  # 9216


def _gen(c: int, i: int) -> torch.Generator:
    return torch.Generator(device="cpu").manual_seed(1000 + 100 * c + i)


def randn(shape, c: int, i: int, std: float = 1.0, dtype=torch.bfloat16) -> torch.Tensor:
    x = torch.randn(*shape, generator=_gen(c, i), dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(dtype)


# ------------------------------------------------------------------ configs
def tiny_pair(rows: int = 256, cols: int = 256, outlier_frac: float = 0.02,
              outlier_scale: float = 50.0, c: int = 1):
    """Round trip + GEMM, tiny: A and B fp32 ~ N(0,1), 2% of entries (chosen
    without replacement) scaled by 50 as outliers."""
    out = []
    for i in range(2):
        x = torch.randn(rows, cols, generator=_gen(c, i), dtype=torch.float32)
        n_out = int(round(outlier_frac * rows * cols))
        idx = torch.randperm(rows * cols, generator=_gen(c, 10 + i))[:n_out]
        x.view(-1)[idx] *= outlier_scale
        out.append(x)
    return out[0], out[1]


def activations(rows: int = CHUNK_TOKENS, cols: int = DIM, outlier_channels: int = 8,
                outlier_scale: float = 30.0, c: int = 2, i: int = 0) -> torch.Tensor:
    """bf16 activations ~ N(0,1) with a few K-channels scaled as outliers."""
    x = torch.randn(rows, cols, generator=_gen(c, i), dtype=torch.float32)
    if outlier_channels:
        ch = torch.randperm(cols, generator=_gen(c, 50 + i))[:outlier_channels]
        x[:, ch] *= outlier_scale
    return x.to(torch.bfloat16)


def weights(rows: int, cols: int, c: int, i: int, std: float = 0.02) -> torch.Tensor:
    return randn((rows, cols), c, i, std=std)


def gelu_activations(rows: int = CHUNK_TOKENS, cols: int = FFN, c: int = 3, i: int = 3
                     ) -> torch.Tensor:
    """Down-projection input: erf-GELU of N(0,1), rounded to bf16."""
    x = torch.randn(rows, cols, generator=_gen(c, i), dtype=torch.float32)
    return torch.nn.functional.gelu(x).to(torch.bfloat16)


def kv_tensor(seed: int, tokens: int, heads: int = HEADS, head_dim: int = HEAD_DIM,
              c: int = 4) -> torch.Tensor:
    """bf16 [tokens, heads, head_dim]; head h ~ N(0, sigma_h^2), sigma_h ~ U(0.5, 4)."""
    g = _gen(c, seed)
    sigma = torch.rand(heads, generator=g, dtype=torch.float32) * 3.5 + 0.5
    x = torch.randn(tokens, heads, head_dim, generator=g, dtype=torch.float32)
    return (x * sigma[None, :, None]).to(torch.bfloat16)


@dataclass
class QKVWorkload:
    """Single DiT QKV projection: A [2640, 3072] bf16, W [9216, 3072] bf16."""
    a: torch.Tensor
    w: torch.Tensor


def qkv(c: int = 2) -> QKVWorkload:
    return QKVWorkload(a=activations(c=c, i=0), w=weights(QKV_N, DIM, c=c, i=1))


@dataclass
class FFNWorkload:
    x: torch.Tensor        # [2640, 3072]
    w_up: torch.Tensor     # [14336, 3072]
    w_down: torch.Tensor   # [3072, 14336]
    h: torch.Tensor        # standalone down-proj input GELU(N(0,1)) [2640, 14336]


def ffn(c: int = 3) -> FFNWorkload:
    return FFNWorkload(x=randn((CHUNK_TOKENS, DIM), c, 0), w_up=weights(FFN, DIM, c, 1),
                       w_down=weights(DIM, FFN, c, 2), h=gelu_activations(c=c, i=3))


def kv_window(c: int = 4):
    """K and V for one layer's full window: [10560, 24, 128] bf16 each
    (3 sink + 9 window latent frames x 880 tokens)."""
    frames = SINK_FRAMES + WINDOW_FRAMES
    t = frames * TOKENS_PER_FRAME
    return kv_tensor(0, t, c=c), kv_tensor(1, t, c=c)


def kv_tensor_cuda(seed: int, tokens: int, heads: int = HEADS, head_dim: int = HEAD_DIM,
                   device="cuda", c: int = 5) -> torch.Tensor:
    """kv_tensor's recipe drawn on the GPU (CUDA generator seeded
    1000 + 100*c + 500 + seed): used to prefill the 30 layers' caches."""
    g = torch.Generator(device=device).manual_seed(1000 + 100 * c + 500 + seed)
    sigma = torch.rand(heads, generator=g, device=device) * 3.5 + 0.5
    x = torch.randn(tokens, heads, head_dim, generator=g, device=device)
    return (x * sigma[None, :, None]).to(torch.bfloat16)


def layer_weights_cuda(layer: int, device="cuda", c: int = 5):
    """The four weight matrices of one DiT layer (QKV, out, up, down) drawn on
    the GPU from a CUDA generator seeded 1000 + 100*c + layer."""
    g = torch.Generator(device=device).manual_seed(1000 + 100 * c + layer)
    shapes = [(QKV_N, DIM), (DIM, DIM), (FFN, DIM), (DIM, FFN)]
    return [(torch.randn(*s, generator=g, device=device, dtype=torch.float32) * 0.02)
            .to(torch.bfloat16) for s in shapes]
