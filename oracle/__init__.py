"""CPU oracle of the NVFP4 W4A4 path (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import this package.  The product library
(``nvfp4_w4a4_quantized_08_b200``) never imports it, and this package imports
nothing from the product: the two share no code.

This module is argument marshalling around ``liboracle.so`` (built from
``nvfp4_oracle.c`` by :func:`build`); every step of the arithmetic lives in the
C source, which cites the passages of the LongLive-2.0 pages it follows.
Arrays are numpy; bfloat16 tensors travel as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

OK, ERR_ARG, ERR_NONFINITE, ERR_DOMAIN = 0, 1, 2, 3


class OracleError(RuntimeError):
    pass


# gcc flags of the oracle: IEEE binary32 with no contraction, OpenMP on outer loops
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-fexcess-precision=standard"]


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (IEEE binary32, no contraction, OpenMP)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        i64, i32, f32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
        L.orc_e2m1_value.restype = ctypes.c_double
        L.orc_e2m1_value.argtypes = [i32]
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_e4m3_value.argtypes = [i32]
        L.orc_e4m3_encode.restype = i32
        L.orc_e4m3_encode.argtypes = [f32]
        L.orc_e2m1_encode.restype = i32
        L.orc_e2m1_encode.argtypes = [f32]
        L.orc_bf16_from_f32.restype = ctypes.c_uint16
        L.orc_bf16_from_f32.argtypes = [f32]
        L.orc_block_scale.restype = i32
        L.orc_block_scale.argtypes = [f32, f32]
        L.orc_element_code.restype = i32
        L.orc_element_code.argtypes = [f32, i32, f32]
        L.orc_dequant_elem.restype = ctypes.c_uint16
        L.orc_dequant_elem.argtypes = [i32, i32, f32]
        L.orc_sf_mma_offset.restype = i64
        L.orc_sf_mma_offset.argtypes = [i64, i64, i64]
        L.orc_sf_mma_bytes.restype = i64
        L.orc_sf_mma_bytes.argtypes = [i64, i64]
        L.orc_sf_to_mma.restype = i32
        L.orc_sf_to_mma.argtypes = [vp, i64, i64, vp]
        L.orc_tensor_scale.restype = i32
        L.orc_tensor_scale.argtypes = [vp, i32, i64, i64, i64, vp, vp]
        L.orc_quantize.restype = i32
        L.orc_quantize.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, vp]
        L.orc_dequantize.restype = i32
        L.orc_dequantize.argtypes = [vp, vp, f32, i64, i64, vp]
        L.orc_dequantize_exact.restype = i32
        L.orc_dequantize_exact.argtypes = [vp, vp, f32, i64, i64, vp]
        L.orc_gemm.restype = i32
        L.orc_gemm.argtypes = [vp, vp, f32, vp, vp, f32, i64, i64, i64, vp, i64, vp, vp]
        L.orc_window_attention.restype = i32
        L.orc_window_attention.argtypes = [vp, i64, vp, i64, vp, vp, i64, i32, i32,
                                           ctypes.c_double, vp, vp]
        L.orc_gelu_tanh.restype = i32
        L.orc_gelu_tanh.argtypes = [vp, vp, i64]
        L.orc_kv_quant_chunk.restype = i32
        L.orc_kv_quant_chunk.argtypes = [vp, i64, i32, i32, i32, i32, vp, vp, vp, i32]
        L.orc_block_scale_rule.restype = i32
        L.orc_block_scale_rule.argtypes = [vp, ctypes.c_float, i32]
        L.orc_kv_dequant_window.restype = i32
        L.orc_kv_dequant_window.argtypes = [vp, vp, vp, i32, vp, i32, i32, i32, i32, vp]
        L.orc_set_threads.restype = i32
        L.orc_set_threads.argtypes = [i32]
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _check(rc: int, what: str) -> None:
    if rc != OK:
        names = {ERR_ARG: "bad argument", ERR_NONFINITE: "non-finite input",
                 ERR_DOMAIN: "tensor scale outside the recipe's domain"}
        raise OracleError(f"oracle {what}: {names.get(rc, rc)}")


def set_threads(n: int) -> int:
    """Set the OpenMP thread count (0 = leave); returns the count in use."""
    return lib().orc_set_threads(int(n))


# ---------------------------------------------------------------- formats
def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(int(code))


def e4m3_value(byte: int) -> float:
    return lib().orc_e4m3_value(int(byte))


def e4m3_encode(r: float) -> int:
    return lib().orc_e4m3_encode(float(np.float32(r)))


def e2m1_encode(y: float) -> int:
    return lib().orc_e2m1_encode(float(np.float32(y)))


def bf16_from_f32(f: float) -> int:
    return lib().orc_bf16_from_f32(float(np.float32(f)))


def block_scale(amax_b: float, s_t: float) -> int:
    return lib().orc_block_scale(float(np.float32(amax_b)), float(np.float32(s_t)))


def element_code(x: float, s_b: int, s_t: float) -> int:
    return lib().orc_element_code(float(np.float32(x)), int(s_b), float(np.float32(s_t)))


def dequant_elem(code: int, s_b: int, s_t: float) -> int:
    return lib().orc_dequant_elem(int(code), int(s_b), float(np.float32(s_t)))


def sf_mma_offset(row: int, kb: int, nkb: int) -> int:
    return lib().orc_sf_mma_offset(row, kb, nkb)


def sf_mma_bytes(rows: int, cols: int) -> int:
    return lib().orc_sf_mma_bytes(rows, cols)


def sf_to_mma(sf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    out = np.empty(sf_mma_bytes(rows, cols), dtype=np.uint8)
    _check(lib().orc_sf_to_mma(_ptr(sf), rows, cols, _ptr(out)), "sf_to_mma")
    return out


# ---------------------------------------------------------------- codec
def _dtype_code(x: np.ndarray) -> int:
    if x.dtype == np.uint16:
        return 0  # bfloat16 bit patterns
    if x.dtype == np.float32:
        return 1
    raise TypeError("oracle inputs are bf16 bits (uint16) or float32")


def tensor_scale(x: np.ndarray) -> Tuple[float, float]:
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    amax = np.zeros(1, np.float32)
    st = np.zeros(1, np.float32)
    _check(lib().orc_tensor_scale(_ptr(x), _dtype_code(x), rows, cols, cols, _ptr(amax),
                                  _ptr(st)), "tensor_scale")
    return float(amax[0]), float(st[0])


def quantize(x: np.ndarray, s_t: Optional[float] = None
             ) -> Tuple[np.ndarray, np.ndarray, float]:
    """x: [rows, cols] bf16 bits (uint16) or float32 -> (codes [rows, cols/2],
    sf [rows, cols/16] row-major E4M3 bytes, s_t)."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    codes = np.empty((rows, cols // 2), np.uint8)
    sf = np.empty((rows, cols // 16), np.uint8)
    st = np.zeros(1, np.float32)
    st_in = None if s_t is None else np.array([s_t], np.float32)
    rc = lib().orc_quantize(_ptr(x), _dtype_code(x), rows, cols, cols, _ptr(codes), _ptr(sf),
                            _ptr(st), None if st_in is None else _ptr(st_in))
    _check(rc, "quantize")
    return codes, sf, float(st[0])


def dequantize(codes: np.ndarray, sf: np.ndarray, s_t: float) -> np.ndarray:
    """-> bf16 bits [rows, cols]"""
    codes = np.ascontiguousarray(codes, np.uint8)
    sf = np.ascontiguousarray(sf, np.uint8)
    rows, half = codes.shape
    out = np.empty((rows, half * 2), np.uint16)
    _check(lib().orc_dequantize(_ptr(codes), _ptr(sf), float(s_t), rows, half * 2, _ptr(out)),
           "dequantize")
    return out


def dequantize_exact(codes: np.ndarray, sf: np.ndarray, s_t: float) -> np.ndarray:
    """-> float64 [rows, cols], the exact values v(q) * s_b * s_t"""
    codes = np.ascontiguousarray(codes, np.uint8)
    sf = np.ascontiguousarray(sf, np.uint8)
    rows, half = codes.shape
    out = np.empty((rows, half * 2), np.float64)
    _check(lib().orc_dequantize_exact(_ptr(codes), _ptr(sf), float(s_t), rows, half * 2,
                                      _ptr(out)), "dequantize_exact")
    return out


def gemm(a: Tuple[np.ndarray, np.ndarray, float], w: Tuple[np.ndarray, np.ndarray, float],
         rows: Optional[Sequence[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """FP64 reference of C = A W^T on NVFP4 operands (codes, row-major sf, s_t).
    Returns (y, S) for the requested rows of A (all rows when None)."""
    ac, asf, ast = a
    wc, wsf, wst = w
    ac = np.ascontiguousarray(ac, np.uint8)
    asf = np.ascontiguousarray(asf, np.uint8)
    wc = np.ascontiguousarray(wc, np.uint8)
    wsf = np.ascontiguousarray(wsf, np.uint8)
    M, K = ac.shape[0], ac.shape[1] * 2
    N = wc.shape[0]
    assert wc.shape[1] * 2 == K
    if rows is None:
        ids = None
        n = M
    else:
        ids = np.ascontiguousarray(np.asarray(rows, np.int64))
        n = ids.shape[0]
    y = np.empty((n, N), np.float64)
    S = np.empty((n, N), np.float64)
    rc = lib().orc_gemm(_ptr(ac), _ptr(asf), float(ast), _ptr(wc), _ptr(wsf), float(wst), M, N,
                        K, None if ids is None else _ptr(ids), n, _ptr(y), _ptr(S))
    _check(rc, "gemm")
    return y, S


def gelu_tanh(y: np.ndarray) -> np.ndarray:
    """GELU, tanh form, elementwise in binary64 (the GEMM epilogue's FFN
    activation): 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3)))."""
    y = np.ascontiguousarray(y, np.float64)
    out = np.empty_like(y)
    _check(lib().orc_gelu_tanh(_ptr(y), _ptr(out), y.size), "gelu_tanh")
    return out


def kv_quant_chunk(kv: np.ndarray, n_frames: int, tpf: int, heads: int, head_dim: int,
                   token_stride: Optional[int] = None, rule: int = 0
                   ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """kv: bf16 bits, flat buffer holding n_frames*tpf tokens at token_stride
    elements apart.  rule 0: block max onto 6; rule 1: Four Over Six.
    -> (codes [n_frames, tpf*heads*head_dim/2],
    sf [n_frames, tpf*heads*head_dim/16], s_t [n_frames])."""
    kv = np.ascontiguousarray(kv, np.uint16)
    ts = heads * head_dim if token_stride is None else token_stride
    per = tpf * heads * head_dim
    codes = np.empty((n_frames, per // 2), np.uint8)
    sf = np.empty((n_frames, per // 16), np.uint8)
    st = np.empty(n_frames, np.float32)
    rc = lib().orc_kv_quant_chunk(_ptr(kv), ts, n_frames, tpf, heads, head_dim, _ptr(codes),
                                  _ptr(sf), _ptr(st), rule)
    _check(rc, "kv_quant_chunk")
    return codes, sf, st


def block_scale_rule(block: np.ndarray, s_t: float, rule: int) -> int:
    """Scale byte of one 16-element fp32 block under `rule` (0: onto 6,
    1: Four Over Six)."""
    block = np.ascontiguousarray(block, np.float32)
    if block.size != 16:
        raise ValueError("a block has 16 elements")
    return int(lib().orc_block_scale_rule(_ptr(block), float(s_t), int(rule)))


def kv_dequant_window(pool_codes: np.ndarray, pool_sf: np.ndarray, pool_st: np.ndarray,
                      slot_ids: Sequence[int], tpf: int, heads: int, head_dim: int
                      ) -> np.ndarray:
    """-> bf16 bits [len(slot_ids)*tpf, heads, head_dim]"""
    pool_codes = np.ascontiguousarray(pool_codes, np.uint8)
    pool_sf = np.ascontiguousarray(pool_sf, np.uint8)
    pool_st = np.ascontiguousarray(pool_st, np.float32)
    ids = np.ascontiguousarray(np.asarray(slot_ids, np.int32))
    out = np.empty((len(ids) * tpf, heads, head_dim), np.uint16)
    rc = lib().orc_kv_dequant_window(_ptr(pool_codes), _ptr(pool_sf), _ptr(pool_st),
                                     pool_codes.shape[0], _ptr(ids), len(ids), tpf, heads,
                                     head_dim, _ptr(out))
    _check(rc, "kv_dequant_window")
    return out


def window_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                     rows: Optional[Sequence[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Windowed attention in binary64.  q: bf16 bits [tq, q_stride] (head h at
    columns h*head_dim...); k, v: bf16 bits [n_kv, heads, head_dim] (the window
    rebuild's output).  -> (out, E), both [n_rows, heads, head_dim]:
    out = sum_j p_j v_j, E = sum_j p_j |v_j| (the scale of the P V sum)."""
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    v = np.ascontiguousarray(v, np.uint16)
    n_kv, heads, hd = k.shape
    assert v.shape == k.shape and q.ndim == 2
    if rows is None:
        ids, n = None, q.shape[0]
    else:
        ids = np.ascontiguousarray(np.asarray(rows, np.int64))
        n = ids.shape[0]
    out = np.empty((n, heads, hd), np.float64)
    E = np.empty((n, heads, hd), np.float64)
    _check(lib().orc_window_attention(_ptr(q), q.shape[1], None if ids is None else _ptr(ids), n,
                                      _ptr(k), _ptr(v), n_kv, heads, hd, float(scale), _ptr(out),
                                      _ptr(E)), "window_attention")
    return out, E


def sink_window_frames(chunks: Sequence[Tuple[int, bool]], global_sinks: int, shot_sinks: int,
                       window: int) -> List[List[int]]:
    """Frames each chunk of a multi-shot generation attends to, in frame order.

    The two-level attention sinks (neurohive.io LongLive-2.0 article, inference
    section; tailorednewshub.com article, "Sumidero de Atención Multi-Toma"):
    the first `global_sinks` frames of the video stay for good, the first
    `shot_sinks` frames of the current shot are re-bound at each cut; with the
    local window of the last `window` frames, the chunk's own included
    (171host.com teardown, section 2.2).  chunks: (n_frames, new_shot) in
    generation order; the first chunk starts the first shot."""
    out = []
    f0 = 0
    shot = 0
    for n, new_shot in chunks:
        f1 = f0 + n
        if new_shot or f0 == 0:
            shot = f0
        frames = []
        for f in range(f1):
            in_global = f < global_sinks
            in_shot = shot <= f < shot + shot_sinks
            in_window = f >= f1 - window
            if in_global or in_shot or in_window:
                frames.append(f)
        out.append(frames)
        f0 = f1
    return out
