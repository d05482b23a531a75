"""Run one libnvfp4 kernel on one DiT-shaped case a few times, for profilers.

    python -m nvfp4_w4a4_quantized_08_b200.cases <case> [reps]

Cases (seeded synthetic inputs, shapes of one layer of the 5B-style DiT):
  gemm_qkv  gemm_out  gemm_up  gemm_down   -- nvfp4_gemm, bf16 output
  quant_act  (2640 x 3072 bf16)  quant_ffn  (2640 x 14336 bf16)   -- nvfp4_quantize
  kv  -- kv_quant_chunk of 3 new frames (K, V read from a fused QKV output)
         then kv_dequant_window over 12 slots
Each case prepares its inputs, synchronizes, then launches the kernel(s) `reps`
times, so `ncu -s <launches before> -c 1` picks one steady-state launch.
"""
from __future__ import annotations

import sys

import torch

import nvfp4_w4a4_quantized_08_b200 as nv

GEMM = {"gemm_qkv": (2640, 9216, 3072), "gemm_out": (2640, 3072, 3072),
        "gemm_up": (2640, 14336, 3072), "gemm_down": (2640, 3072, 14336)}
QUANT = {"quant_act": (2640, 3072), "quant_ffn": (2640, 14336)}


def run(case: str, reps: int = 3) -> None:
    torch.cuda.set_device(0)
    g = torch.Generator(device="cuda").manual_seed(7)
    if case in GEMM:
        M, N, K = GEMM[case]
        a = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
        w = (torch.randn(N, K, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
        qa, qw = nv.quantize(a), nv.quantize(w)
        out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        torch.cuda.synchronize()
        for _ in range(reps):
            nv.gemm(qa, qw, out=out)
    elif case in QUANT:
        x = torch.randn(*QUANT[case], device="cuda", generator=g).to(torch.bfloat16)
        q = nv.empty(*QUANT[case])
        torch.cuda.synchronize()
        for _ in range(reps):
            nv.quantize(x, out=q)
    elif case == "kv":
        cache = nv.KVCache(15, 880, 24, 128)
        qkv = torch.randn(2640, 9216, device="cuda", generator=g).to(torch.bfloat16)
        for s0 in (0, 3, 6, 9):
            cache.quant_chunk(qkv[:, 3072:6144], qkv[:, 6144:], [s0, s0 + 1, s0 + 2])
        kw = torch.empty(12 * 880, 24, 128, dtype=torch.bfloat16, device="cuda")
        vw = torch.empty_like(kw)
        torch.cuda.synchronize()
        for _ in range(reps):
            cache.quant_chunk(qkv[:, 3072:6144], qkv[:, 6144:], [12, 13, 14])
            cache.dequant_window([0, 1, 2, 6, 7, 8, 9, 10, 11, 12, 13, 14], kw, vw)
    else:
        raise SystemExit(f"unknown case {case!r}; one of {sorted([*GEMM, *QUANT, 'kv'])}")
    torch.cuda.synchronize()
    status = nv.device_status()
    if status:
        raise SystemExit(f"device status {status}")
    print(f"{case}: {reps} reps ok")


if __name__ == "__main__":
    run(sys.argv[1], int(sys.argv[2]) if len(sys.argv) > 2 else 3)
