"""Helpers shared by the GPU parity tests: move seeded inputs to the oracle's
numpy form and compare the CUDA path's outputs with the oracle's."""
from __future__ import annotations

import numpy as np
import torch

GEMM_REL_TOL = 1e-3     # |y - y_ref| <= 1e-3 * sum_k |a_k w_k|
BF16_HALF_ULP = 2.0 ** -8
GELU_SLOPE_MAX = 1.13   # max |d GELU_tanh / dy| (pinned in test_oracle_gelu.py)
TANH_APPROX_REL = 2.0 ** -11  # hardware tanh.approx.f32 relative error, with margin


def assert_gelu_gemm_close(orc, g_gpu: np.ndarray, y_ref: np.ndarray, S: np.ndarray,
                           bf16_out: bool):
    """GEMM with the GELU epilogue: |g - GELU(y_ref)| <= GELU_SLOPE_MAX * e +
    TANH_APPROX_REL * (|y_ref| + e), e the error of GELU's input: the GEMM
    bound 1e-3 * S, plus for bf16 output the rounding of y to bf16 (the GELU
    takes the bf16 product there), carried through GELU's slope; the second
    term is the hardware tanh's error (the GELU moves by 0.5 |y| |dtanh|).
    For bf16 output, half a bf16 ulp of the result on top."""
    g_gpu = g_gpu.astype(np.float64)
    g_ref = orc.gelu_tanh(y_ref)
    e = GEMM_REL_TOL * S
    if bf16_out:
        e = e + BF16_HALF_ULP * (np.abs(y_ref) + e)
    tol = GELU_SLOPE_MAX * e + TANH_APPROX_REL * (np.abs(y_ref) + e)
    if bf16_out:
        tol = tol + BF16_HALF_ULP * (np.abs(g_ref) + tol)
    err = np.abs(g_gpu - g_ref)
    bad = ~(err <= tol)
    if bad.any():
        i = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{bad.sum()} of {bad.size} outside tolerance; first {i.tolist()}: "
            f"gpu {g_gpu[tuple(i[0])]} ref {g_ref[tuple(i[0])]} y_ref {y_ref[tuple(i[0])]} "
            f"S {S[tuple(i[0])]}")


def bits(x: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns (numpy, CPU); fp32 -> float32 numpy."""
    x = x.detach().cpu().contiguous()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view(np.uint16)
    if x.dtype == torch.float32:
        return x.numpy()
    raise TypeError(x.dtype)


def np_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint8)


def assert_quant_equal(orc, gpu_q, x_np, sf_layout: int, s_t_in=None):
    """GPU NVFP4 tensor == oracle quantization of x_np, byte for byte."""
    codes, sf, st = orc.quantize(x_np, s_t=s_t_in)
    g_codes = np_u8(gpu_q.codes)
    g_st = float(gpu_q.s_t.cpu()[0])
    assert np.float32(g_st) == np.float32(st), (g_st, st)
    np.testing.assert_array_equal(g_codes, codes)
    rows, cols = x_np.shape
    ref_sf = sf.reshape(-1) if sf_layout == 0 else orc.sf_to_mma(sf, rows, cols)
    np.testing.assert_array_equal(np_u8(gpu_q.sf)[: ref_sf.size], ref_sf)
    return codes, sf, st


def sf_rowmajor(orc, gpu_q) -> np.ndarray:
    """The GPU tensor's block scales in row-major order (undoing the MMA layout)."""
    raw = np_u8(gpu_q.sf)
    nkb = gpu_q.cols // 16
    if gpu_q.sf_layout == 0:
        return raw[: gpu_q.rows * nkb].reshape(gpu_q.rows, nkb)
    r = np.arange(gpu_q.rows)[:, None]
    k = np.arange(nkb)[None, :]
    ktiles = (nkb + 3) // 4
    off = ((r // 128) * ktiles + k // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + k % 4
    return raw[off]


def assert_gemm_close(y_gpu: np.ndarray, y_ref: np.ndarray, S: np.ndarray, bf16_out: bool):
    """Per element: |y - y_ref| <= 1e-3 * S (+ half a bf16 ulp of |y_ref| for bf16 output);
    exact zero where S == 0."""
    y_gpu = y_gpu.astype(np.float64)
    tol = GEMM_REL_TOL * S
    if bf16_out:
        tol = tol + BF16_HALF_ULP * np.abs(y_ref)
    err = np.abs(y_gpu - y_ref)
    bad = ~(err <= tol)
    if bad.any():
        i = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{bad.sum()} of {bad.size} outside tolerance; first {i.tolist()}: "
            f"gpu {y_gpu[tuple(i[0])]} ref {y_ref[tuple(i[0])]} S {S[tuple(i[0])]}")
    assert np.all(y_gpu[S == 0] == 0)
