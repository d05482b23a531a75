"""torch-facing wrappers of the libnvfp4 entry points.

Argument marshalling only: each function passes device pointers, sizes and
``torch.cuda.current_stream()`` to the C ABI, which launches the kernels.  No
step of the NVFP4 path runs in Python or torch.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence, Tuple

import torch

from . import _native as N
from ._native import NVFP4Error  # noqa: F401  (re-export)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


_workspaces: Dict[Tuple[int, int], torch.Tensor] = {}


def workspace(device=None) -> torch.Tensor:
    """A zero-filled workspace for the current stream of `device` (cached).
    Calls that share it must stay ordered on that stream."""
    idx = None if device is None else torch.device(device).index
    dev = torch.device("cuda", torch.cuda.current_device() if idx is None else idx)
    key = (dev.index, torch.cuda.current_stream(dev).cuda_stream)
    ws = _workspaces.get(key)
    if ws is None:
        ws = torch.zeros(N.lib().nvfp4_workspace_bytes(), dtype=torch.uint8, device=dev)
        _workspaces[key] = ws
    return ws


@dataclass
class NVFP4Tensor:
    """Device buffers of an NVFP4 tensor (see nvfp4_tensor in include/nvfp4.h)."""
    codes: torch.Tensor   # uint8 [rows, cols/2]
    sf: torch.Tensor      # uint8 [nvfp4_sf_bytes]
    s_t: torch.Tensor     # float32 [1]
    rows: int
    cols: int
    sf_layout: int

    def c_struct(self) -> N.Tensor:
        return N.Tensor(self.codes.data_ptr(), self.sf.data_ptr(), self.s_t.data_ptr(),
                        self.rows, self.cols, self.sf_layout)

    @property
    def device(self):
        return self.codes.device


def codes_bytes(rows: int, cols: int) -> int:
    return int(N.lib().nvfp4_codes_bytes(rows, cols))


def sf_bytes(rows: int, cols: int, sf_layout: int) -> int:
    return int(N.lib().nvfp4_sf_bytes(rows, cols, sf_layout))


def empty(rows: int, cols: int, sf_layout: int = N.SF_MMA128x4, device="cuda") -> NVFP4Tensor:
    nb = sf_bytes(rows, cols, sf_layout)
    if nb == 0 and rows * cols > 0:
        raise NVFP4Error(N.ERR_UNSUPPORTED_SHAPE, "empty")
    return NVFP4Tensor(
        codes=torch.empty(rows, cols // 2, dtype=torch.uint8, device=device),
        sf=torch.empty(max(nb, 1), dtype=torch.uint8, device=device),
        s_t=torch.empty(1, dtype=torch.float32, device=device),
        rows=rows, cols=cols, sf_layout=sf_layout)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return N.BF16
    if t.dtype == torch.float32:
        return N.FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def quantize(x: torch.Tensor, sf_layout: int = N.SF_MMA128x4, s_t: Optional[torch.Tensor] = None,
             out: Optional[NVFP4Tensor] = None, ws: Optional[torch.Tensor] = None,
             amax_in: Optional[torch.Tensor] = None) -> NVFP4Tensor:
    """nvfp4_quantize: x is a 2-D bf16/fp32 CUDA tensor with unit column stride.

    s_t:     a one-element fp32 tensor holding the tensor scale to use, or None.
    amax_in: a one-element fp32 tensor holding max|x| as accumulated by the
             producer (``gemm(..., c_amax=)``); the amax pass is skipped and the
             word is reset to 0 when the launch ends.  Exclusive with s_t.
    """
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("quantize expects a 2-D tensor with contiguous rows")
    rows, cols = x.shape
    if out is None:
        out = empty(rows, cols, sf_layout, x.device)
    ws = workspace(x.device) if ws is None else ws
    st = out.c_struct()
    N.check(N.lib().nvfp4_quantize(x.data_ptr(), _dtype_code(x), rows, cols, x.stride(0),
                                   ctypes.byref(st), _ptr(s_t), _ptr(amax_in), ws.data_ptr(),
                                   ws.numel(), _stream()), "nvfp4_quantize")
    return out


def dequantize(t: NVFP4Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """nvfp4_dequantize -> bf16 [rows, cols]"""
    if out is None:
        out = torch.empty(t.rows, t.cols, dtype=torch.bfloat16, device=t.device)
    st = t.c_struct()
    N.check(N.lib().nvfp4_dequantize(ctypes.byref(st), out.data_ptr(), out.stride(0), _stream()),
            "nvfp4_dequantize")
    return out


def gemm(a: NVFP4Tensor, w: NVFP4Tensor, out_dtype: torch.dtype = torch.bfloat16,
         out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
         c_amax: Optional[torch.Tensor] = None, c_amax_cols: int = 0,
         act: int = N.ACT_NONE) -> torch.Tensor:
    """nvfp4_gemm: C = act(A W^T), [a.rows, w.rows] in bf16 or fp32.

    act:    N.ACT_NONE, or N.ACT_GELU_TANH (the FFN's GELU, tanh form, in the
            epilogue before the output rounding).

    c_amax: fp32 tensor that starts at 0 (or at a smaller running max); the
            kernel raises it to max|C| over the values it stores.  With
            c_amax_cols = 0 one element covers all of C; with c_amax_cols > 0
            (a multiple of 256 dividing N) element g covers columns
            [g * c_amax_cols, (g + 1) * c_amax_cols).
    """
    if c_amax is not None:
        need = 1 if c_amax_cols == 0 else max(1, w.rows // c_amax_cols)
        if c_amax.dtype != torch.float32 or c_amax.numel() < need:
            raise ValueError(f"c_amax needs {need} fp32 elements")
    if out is None:
        out = torch.empty(a.rows, w.rows, dtype=out_dtype, device=a.device)
    ws = workspace(a.device) if ws is None else ws
    sa, sw = a.c_struct(), w.c_struct()
    N.check(N.lib().nvfp4_gemm(ctypes.byref(sa), ctypes.byref(sw), out.data_ptr(),
                               _dtype_code(out), out.stride(0), act, _ptr(c_amax), c_amax_cols,
                               ws.data_ptr(), ws.numel(), _stream()), "nvfp4_gemm")
    return out


class KVCache:
    """The NVFP4 KV cache of one layer: n_slots frame slots for K and V."""

    def __init__(self, n_slots: int, tokens_per_frame: int, heads: int, head_dim: int,
                 device="cuda", scale_rule: int = N.SCALE_ONTO_6):
        """scale_rule: N.SCALE_ONTO_6 (the recipe) or N.SCALE_FOUR_OVER_SIX."""
        per = tokens_per_frame * heads * head_dim
        self.scale_rule = scale_rule
        self.n_slots, self.tpf, self.heads, self.head_dim = n_slots, tokens_per_frame, heads, head_dim
        self.k_codes = torch.zeros(n_slots, per // 2, dtype=torch.uint8, device=device)
        self.v_codes = torch.zeros_like(self.k_codes)
        self.k_sf = torch.zeros(n_slots, per // 16, dtype=torch.uint8, device=device)
        self.v_sf = torch.zeros_like(self.k_sf)
        self.k_st = torch.zeros(n_slots, dtype=torch.float32, device=device)
        self.v_st = torch.zeros_like(self.k_st)

    def c_struct(self) -> N.KvCache:
        return N.KvCache(self.k_codes.data_ptr(), self.v_codes.data_ptr(), self.k_sf.data_ptr(),
                         self.v_sf.data_ptr(), self.k_st.data_ptr(), self.v_st.data_ptr(),
                         self.n_slots, self.tpf, self.heads, self.head_dim, self.scale_rule)

    def quant_chunk(self, k: torch.Tensor, v: torch.Tensor, dst_slots: Sequence[int],
                    ws: Optional[torch.Tensor] = None, k_amax_in: Optional[torch.Tensor] = None,
                    v_amax_in: Optional[torch.Tensor] = None) -> None:
        """nvfp4_kv_quant_chunk.  k, v: bf16 views [tokens, heads*head_dim] (or
        [tokens, heads, head_dim]) with unit stride inside a token.
        k_amax_in, v_amax_in: both None (amax pass), or one-element fp32
        tensors holding max|K|, max|V| from the producer; reset to 0."""
        token_stride = k.stride(0)
        if v.stride(0) != token_stride:
            raise ValueError("k and v must share a token stride")
        slots = (ctypes.c_int32 * len(dst_slots))(*dst_slots)
        ws = workspace(k.device) if ws is None else ws
        cs = self.c_struct()
        N.check(N.lib().nvfp4_kv_quant_chunk(ctypes.byref(cs), k.data_ptr(), v.data_ptr(),
                                             token_stride, slots, len(dst_slots), _ptr(k_amax_in),
                                             _ptr(v_amax_in), ws.data_ptr(), ws.numel(),
                                             _stream()), "nvfp4_kv_quant_chunk")

    def dequant_window(self, slot_ids: Sequence[int], k_out: Optional[torch.Tensor] = None,
                       v_out: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
        """nvfp4_kv_dequant_window -> bf16 K, V [n*tokens_per_frame, heads, head_dim]"""
        n = len(slot_ids)
        shape = (n * self.tpf, self.heads, self.head_dim)
        if k_out is None:
            k_out = torch.empty(shape, dtype=torch.bfloat16, device=self.k_codes.device)
        if v_out is None:
            v_out = torch.empty(shape, dtype=torch.bfloat16, device=self.k_codes.device)
        ids = (ctypes.c_int32 * n)(*slot_ids)
        cs = self.c_struct()
        N.check(N.lib().nvfp4_kv_dequant_window(ctypes.byref(cs), ids, n, k_out.data_ptr(),
                                                v_out.data_ptr(), _stream()),
                "nvfp4_kv_dequant_window")
        return k_out, v_out

    def window_attention(self, q: torch.Tensor, slot_ids: Sequence[int],
                         scale: Optional[float] = None,
                         out: Optional[torch.Tensor] = None,
                         ws: Optional[torch.Tensor] = None) -> torch.Tensor:
        """nvfp4_window_attention: softmax(scale q k^T) v over the listed slots,
        read straight from the NVFP4 pools.  q: bf16 [tq, >= heads*head_dim]
        (row stride a multiple of 8, e.g. the Q third of a QKV output) ->
        bf16 [tq, heads*head_dim] (or `out`, same layout as q)."""
        width = self.heads * self.head_dim
        if q.dtype != torch.bfloat16 or q.dim() != 2 or q.stride(1) != 1 or q.shape[1] < width:
            raise ValueError(f"q must be a 2-D bf16 tensor of at least {width} unit-stride columns")
        if scale is None:
            scale = self.head_dim ** -0.5
        if out is None:
            out = torch.empty(q.shape[0], width, dtype=torch.bfloat16, device=q.device)
        elif (out.dtype != torch.bfloat16 or out.dim() != 2 or out.stride(1) != 1 or
              out.shape[0] != q.shape[0] or out.shape[1] < width):
            raise ValueError(f"out must be a 2-D bf16 tensor of {q.shape[0]} rows and at least "
                             f"{width} unit-stride columns")
        n = len(slot_ids)
        ids = (ctypes.c_int32 * n)(*slot_ids)
        cs = self.c_struct()
        ws = workspace(q.device) if ws is None else ws
        N.check(N.lib().nvfp4_window_attention(ctypes.byref(cs), ids, n, q.data_ptr(), q.stride(0),
                                               q.shape[0], float(scale), out.data_ptr(),
                                               out.stride(0), ws.data_ptr(), ws.numel(),
                                               _stream()),
                "nvfp4_window_attention")
        return out


class SinkPlan:
    """nvfp4_sink_plan: host-side slot planning under the two-level attention
    sinks (global sinks kept for good, shot sinks re-bound at cuts, a local
    window).  next() -> (dst_slots for KVCache.quant_chunk, window slot list
    for KVCache.dequant_window / window_attention)."""

    def __init__(self, n_slots: int, global_sinks: int = 3, shot_sinks: int = 3,
                 window: int = 9):
        self.n_slots = n_slots
        self._h = N.lib().nvfp4_sink_plan_create(n_slots, global_sinks, shot_sinks, window)
        if not self._h:
            raise N.NVFP4Error(N.ERR_INVALID_ARG, "nvfp4_sink_plan_create")

    def next(self, n_frames: int, new_shot: bool = False) -> Tuple[List[int], List[int]]:
        dst = (ctypes.c_int32 * max(1, n_frames))()
        win = (ctypes.c_int32 * self.n_slots)()
        n = ctypes.c_int32(0)
        N.check(N.lib().nvfp4_sink_plan_next(self._h, n_frames, int(bool(new_shot)), dst, win,
                                             ctypes.byref(n)), "nvfp4_sink_plan_next")
        return list(dst[:n_frames]), list(win[:n.value])

    def frame_of_slot(self, slot: int) -> int:
        return int(N.lib().nvfp4_sink_plan_frame_of_slot(self._h, slot))

    def close(self) -> None:
        if getattr(self, "_h", None):
            N.lib().nvfp4_sink_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # interpreter shutdown: the library may be gone already
            pass


def device_status(ws: Optional[torch.Tensor] = None) -> int:
    """nvfp4_get_device_status: sync the current stream, read and clear the
    workspace status word."""
    ws = workspace() if ws is None else ws
    return int(N.lib().nvfp4_get_device_status(ws.data_ptr(), _stream()))


def set_wait_limit_ns(ns: int) -> None:
    N.lib().nvfp4_set_wait_limit_ns(int(ns))
