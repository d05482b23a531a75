"""The C-ABI library on the host (no GPU work): it loads, exports every entry
point include/nvfp4.h declares, sizes its buffers, and rejects bad arguments
before any launch.  Every call below carries at least one invalid argument, so
it returns from the host-side checks and touches no device memory."""
import ctypes
import os
import re

import pytest
import torch

from nvfp4_w4a4_quantized_08_b200 import _native as N
from nvfp4_w4a4_quantized_08_b200 import build as nbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")

FAKE = 0x7F0000001000  # never dereferenced: each call fails a host check first


@pytest.fixture(scope="module")
def L():
    nbuild.build()
    return N.lib()


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(nvfp4_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(N.EXPORTS)


def test_sizes(L):
    assert L.nvfp4_codes_bytes(2640, 3072) == 2640 * 1536
    assert L.nvfp4_sf_bytes(2640, 3072, N.SF_ROWMAJOR) == 2640 * 192
    assert L.nvfp4_sf_bytes(2640, 3072, N.SF_MMA128x4) == 2688 * 192
    assert L.nvfp4_sf_bytes(5, 48, N.SF_MMA128x4) == 128 * 4
    assert L.nvfp4_codes_bytes(4, 24) == 0  # cols not a multiple of 16
    assert L.nvfp4_sf_bytes(4, 32, 7) == 0
    assert L.nvfp4_workspace_bytes() >= 32
    assert L.nvfp4_status_string(N.ERR_TIMEOUT) == b"device wait timed out"


def _tensor(rows=256, cols=256, layout=N.SF_MMA128x4, codes=FAKE, sf=FAKE, st=FAKE):
    return N.Tensor(codes, sf, st, rows, cols, layout)


def test_quantize_rejects(L):
    t = _tensor()
    ws = FAKE
    q = L.nvfp4_quantize
    assert q(None, N.BF16, 256, 256, 256, ctypes.byref(t), None, None, ws, 256,
             None) == N.ERR_INVALID_ARG
    assert q(FAKE, 9, 256, 256, 256, ctypes.byref(t), None, None, ws, 256,
             None) == N.ERR_INVALID_ARG
    # a given tensor scale and a producer amax are exclusive
    assert q(FAKE, N.BF16, 256, 256, 256, ctypes.byref(t), FAKE, FAKE, ws, 256,
             None) == N.ERR_INVALID_ARG
    assert q(FAKE, N.BF16, 256, 256, 256, ctypes.byref(t), None, FAKE + 2, ws, 256,
             None) == N.ERR_MISALIGNED
    bad = _tensor(cols=40)
    assert q(FAKE, N.BF16, 256, 40, 40, ctypes.byref(bad), None, None, ws, 256,
             None) == N.ERR_UNSUPPORTED_SHAPE
    assert q(FAKE, N.BF16, 255, 256, 256, ctypes.byref(t), None, None, ws, 256,
             None) == N.ERR_INVALID_ARG  # rows differ from out->rows
    assert q(FAKE + 2, N.BF16, 256, 256, 256, ctypes.byref(t), None, None, ws, 256,
             None) == N.ERR_MISALIGNED
    assert q(FAKE, N.BF16, 256, 256, 260, ctypes.byref(t), None, None, ws, 256,
             None) == N.ERR_MISALIGNED  # 520-byte row stride
    mis = _tensor(codes=FAKE + 8)
    assert q(FAKE, N.BF16, 256, 256, 256, ctypes.byref(mis), None, None, ws, 256,
             None) == N.ERR_MISALIGNED
    assert q(FAKE, N.BF16, 256, 256, 256, ctypes.byref(t), None, None, ws, 8, None) == N.ERR_WORKSPACE
    assert q(FAKE, N.BF16, 256, 256, 256, ctypes.byref(t), None, None, None, 256,
             None) == N.ERR_WORKSPACE
    huge = _tensor(rows=1 << 30, cols=256)
    assert q(FAKE, N.BF16, 1 << 30, 256, 256, ctypes.byref(huge), None, None, ws, 256,
             None) == N.ERR_UNSUPPORTED_SHAPE


def test_gemm_rejects(L):
    a = _tensor(rows=2640, cols=3072)
    w = _tensor(rows=9216, cols=3072)
    g = L.nvfp4_gemm
    ok_args = (FAKE, N.BF16, 9216, N.ACT_NONE, None, 0, FAKE, 256, None)
    assert g(ctypes.byref(a), ctypes.byref(_tensor(rows=9216, cols=3072, layout=N.SF_ROWMAJOR)),
             *ok_args) == N.ERR_INVALID_ARG
    assert g(ctypes.byref(a), ctypes.byref(_tensor(rows=9216, cols=2048)),
             *ok_args) == N.ERR_INVALID_ARG  # K mismatch
    assert g(ctypes.byref(_tensor(rows=2640, cols=3056)),
             ctypes.byref(_tensor(rows=9216, cols=3056)), *ok_args) == N.ERR_UNSUPPORTED_SHAPE
    # any N; a c_amax column group must divide it
    assert g(ctypes.byref(a), ctypes.byref(_tensor(rows=9200, cols=3072)),
             FAKE, N.BF16, 9216, 0, FAKE, 3072, FAKE, 256, None) == N.ERR_INVALID_ARG
    assert g(ctypes.byref(a), ctypes.byref(w), FAKE, N.BF16, 9000, 0, None, 0, FAKE, 256,
             None) == N.ERR_INVALID_ARG  # ldc < N
    assert g(ctypes.byref(a), ctypes.byref(w), FAKE, N.BF16, 9220, 0, None, 0, FAKE, 256,
             None) == N.ERR_MISALIGNED
    assert g(ctypes.byref(a), ctypes.byref(w), FAKE, 5, 9216, 0, None, 0, FAKE, 256,
             None) == N.ERR_INVALID_ARG
    assert g(ctypes.byref(a), ctypes.byref(w), FAKE, N.BF16, 9216, 0, None, 0, FAKE, 4,
             None) == N.ERR_WORKSPACE
    assert g(ctypes.byref(a), ctypes.byref(w), FAKE, N.BF16, 9216, 0, FAKE + 1, 0, FAKE, 256,
             None) == N.ERR_MISALIGNED  # c_amax
    for cols in (-256, 100, 2048, 9216 * 2):  # not a multiple of 256 dividing N
        assert g(ctypes.byref(a), ctypes.byref(w), FAKE, N.BF16, 9216, 0, FAKE, cols, FAKE, 256,
                 None) == N.ERR_INVALID_ARG
    for act in (-1, 2):  # not an nvfp4_act
        assert g(ctypes.byref(a), ctypes.byref(w), FAKE, N.BF16, 9216, act, None, 0, FAKE, 256,
                 None) == N.ERR_INVALID_ARG


def _cache(n_slots=12, tpf=880, heads=24, hd=128, rule=0):
    return N.KvCache(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, n_slots, tpf, heads, hd, rule)


def test_kv_rejects(L):
    c = _cache()
    q = L.nvfp4_kv_quant_chunk
    S = ctypes.c_int32 * 9
    slots = S(0, 1, 2, 3, 4, 5, 6, 7, 8)
    assert q(ctypes.byref(c), FAKE, FAKE, 3072, slots, 9, None, None, FAKE, 256,
             None) == N.ERR_INVALID_ARG
    assert q(ctypes.byref(c), FAKE, FAKE, 3072, slots, 0, None, None, FAKE, 256,
             None) == N.ERR_INVALID_ARG
    bad = (ctypes.c_int32 * 2)(0, 12)
    assert q(ctypes.byref(c), FAKE, FAKE, 3072, bad, 2, None, None, FAKE, 256,
             None) == N.ERR_INVALID_ARG
    rep = (ctypes.c_int32 * 2)(3, 3)
    assert q(ctypes.byref(c), FAKE, FAKE, 3072, rep, 2, None, None, FAKE, 256,
             None) == N.ERR_INVALID_ARG
    assert q(ctypes.byref(c), FAKE, FAKE, 3000, slots, 2, None, None, FAKE, 256,
             None) == N.ERR_INVALID_ARG  # token stride < heads * head_dim
    assert q(ctypes.byref(c), FAKE, FAKE, 3076, slots, 2, None, None, FAKE, 256,
             None) == N.ERR_MISALIGNED
    assert q(ctypes.byref(_cache(hd=40)), FAKE, FAKE, 3072, slots, 2, None, None, FAKE, 256,
             None) == N.ERR_UNSUPPORTED_SHAPE
    assert q(ctypes.byref(c), FAKE, FAKE, 3072, slots, 2, None, None, FAKE, 16,
             None) == N.ERR_WORKSPACE
    # scale rules: 0 (onto 6) and 1 (Four Over Six) only
    assert q(ctypes.byref(_cache(rule=2)), FAKE, FAKE, 3072, slots, 2, None, None, FAKE, 256,
             None) == N.ERR_INVALID_ARG
    # the producer's amax words come as a pair or not at all
    assert q(ctypes.byref(c), FAKE, FAKE, 3072, slots, 2, FAKE, None, FAKE, 256,
             None) == N.ERR_INVALID_ARG
    assert q(ctypes.byref(c), FAKE, FAKE, 3072, slots, 2, FAKE, FAKE + 2, FAKE, 256,
             None) == N.ERR_MISALIGNED
    d = L.nvfp4_kv_dequant_window
    ids = (ctypes.c_int32 * 3)(0, 5, 12)
    assert d(ctypes.byref(c), ids, 3, FAKE, FAKE, None) == N.ERR_INVALID_ARG
    ids = (ctypes.c_int32 * 1)(0)
    assert d(ctypes.byref(c), ids, 0, FAKE, FAKE, None) == N.ERR_INVALID_ARG
    assert d(ctypes.byref(c), ids, 1, FAKE + 4, FAKE, None) == N.ERR_MISALIGNED
    big = (ctypes.c_int32 * 257)(*([0] * 257))
    assert d(ctypes.byref(c), big, 257, FAKE, FAKE, None) == N.ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU refusal")
def test_no_gpu_means_arch_error_not_fallback(L):
    """With every argument valid but no sm_100 device, the call refuses with
    NVFP4_ERR_ARCH instead of computing anything on the host."""
    t = _tensor()
    assert L.nvfp4_quantize(FAKE, N.BF16, 256, 256, 256, ctypes.byref(t), None, None, FAKE, 256,
                            None) == N.ERR_ARCH


def test_window_attention_rejects(L):
    c = _cache()
    f = L.nvfp4_window_attention
    S = ctypes.c_int32 * 3
    ids = S(0, 1, 2)
    ok = (ids, 3, FAKE, 9216, 2640, 0.088, FAKE, 3072, FAKE, 256, None)
    # argument checks run before any device query, so a call that passes them
    # would reach the device: only failing combinations are exercised here
    assert f(ctypes.byref(c), S(0, 1, 12), 3, *ok[2:]) == N.ERR_INVALID_ARG  # slot out of range
    assert f(ctypes.byref(c), ids, 0, *ok[2:]) == N.ERR_INVALID_ARG
    assert f(ctypes.byref(c), ids, 3, FAKE, 9216, 2640, 0.0, FAKE, 3072,
             FAKE, 256, None) == N.ERR_INVALID_ARG  # scale
    assert f(ctypes.byref(c), ids, 3, FAKE, 9216, 2640, float("nan"), FAKE, 3072,
             FAKE, 256, None) == N.ERR_INVALID_ARG
    assert f(ctypes.byref(c), ids, 3, FAKE, 3000, 2640, 0.088, FAKE, 3072,
             FAKE, 256, None) == N.ERR_INVALID_ARG  # q stride below heads * head_dim
    assert f(ctypes.byref(_cache(hd=64)), ids, 3, FAKE, 9216, 2640, 0.088, FAKE, 3072,
             FAKE, 256, None) == N.ERR_UNSUPPORTED_SHAPE  # head_dim 128 only
    assert f(ctypes.byref(c), ids, 3, FAKE, 9216, 0, 0.088, FAKE, 3072,
             FAKE, 256, None) == N.ERR_UNSUPPORTED_SHAPE  # tq
    assert f(ctypes.byref(c), ids, 3, FAKE + 8, 9216, 2640, 0.088, FAKE, 3072,
             FAKE, 256, None) == N.ERR_MISALIGNED
    assert f(ctypes.byref(c), ids, 3, FAKE, 9220, 2640, 0.088, FAKE, 3072,
             FAKE, 256, None) == N.ERR_MISALIGNED
    assert f(ctypes.byref(c), ids, 3, FAKE, 9216, 2640, 0.088, FAKE, 3072,
             None, 256, None) == N.ERR_WORKSPACE
    assert f(ctypes.byref(c), ids, 3, FAKE, 9216, 2640, 0.088, FAKE, 3072,
             FAKE, 128, None) == N.ERR_WORKSPACE


def test_sink_plan_null_and_bad_arguments(L):
    S = ctypes.c_int32 * 16
    n = ctypes.c_int32(0)
    assert L.nvfp4_sink_plan_next(None, 3, 0, S(), S(), ctypes.byref(n)) == N.ERR_INVALID_ARG
    assert not L.nvfp4_sink_plan_create(15, -1, 3, 9)
    assert not L.nvfp4_sink_plan_create(15, 3, 3, 0)
    h = L.nvfp4_sink_plan_create(15, 3, 3, 9)
    assert h
    assert L.nvfp4_sink_plan_next(h, 3, 0, None, S(), ctypes.byref(n)) == N.ERR_INVALID_ARG
    assert L.nvfp4_sink_plan_frame_of_slot(None, 0) == -1
    assert L.nvfp4_sink_plan_frame_of_slot(h, 0) == -1  # nothing planned yet
    L.nvfp4_sink_plan_destroy(h)
    L.nvfp4_sink_plan_destroy(None)  # a no-op
