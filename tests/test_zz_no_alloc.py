"""nvfp4_quantize_noalloc: the quantizer for callers that cannot allocate.

Callers that run inside a memory budget owned by someone else, or hooks that
only receive their input and output buffers, cannot hand the library a device
workspace.  nvfp4_quantize_noalloc keeps the quantizer's scratch words in a
small array that belongs to the library itself.  This test calls it through
the C ABI twice in a row -- first on a tensor with a large amax, then on one
with a small amax, so leftover scratch from the first call would corrupt the
second -- and requires each output to equal, byte for byte, what
nvfp4_quantize produces with its own zeroed workspace (the quantizer's outputs
are exact, so the tolerance is zero).
"""
import ctypes

import pytest
import torch

import nvfp4_w4a4_quantized_08_b200 as nv
from nvfp4_w4a4_quantized_08_b200 import _native as N

pytestmark = pytest.mark.gpu


def _quantize_noalloc(x: torch.Tensor, layout: int) -> nv.NVFP4Tensor:
    rows, cols = x.shape
    out = nv.empty(rows, cols, layout, x.device)
    st = out.c_struct()
    dtype = N.BF16 if x.dtype == torch.bfloat16 else N.FP32
    rc = N.lib().nvfp4_quantize_noalloc(x.data_ptr(), dtype, rows, cols, x.stride(0),
                                        ctypes.byref(st), None,
                                        torch.cuda.current_stream().cuda_stream)
    assert rc == N.OK, N.status_string(rc)
    return out


def _quantize_with_workspace(x: torch.Tensor, layout: int) -> nv.NVFP4Tensor:
    ws = torch.zeros(N.lib().nvfp4_workspace_bytes(), dtype=torch.uint8, device=x.device)
    return nv.quantize(x, sf_layout=layout, ws=ws)


@pytest.mark.parametrize("layout", [N.SF_MMA128x4, N.SF_ROWMAJOR])
def test_noalloc_matches_workspace_path_two_calls(layout):
    g = torch.Generator().manual_seed(77)
    big = (torch.randn(2640, 3072, generator=g) * 40).to(torch.bfloat16).cuda()
    small = (torch.randn(300, 1040, generator=g) * 0.01).to(torch.float32).cuda()
    results = [_quantize_noalloc(big, layout), _quantize_noalloc(small, layout)]
    refs = [_quantize_with_workspace(big, layout), _quantize_with_workspace(small, layout)]
    torch.cuda.synchronize()
    for got, ref in zip(results, refs):
        assert torch.equal(got.s_t, ref.s_t)
        assert torch.equal(got.codes, ref.codes)
        assert torch.equal(got.sf, ref.sf)


def test_noalloc_rejects_bad_arguments_without_launching():
    x = torch.zeros(4, 24, dtype=torch.bfloat16, device="cuda")
    out = nv.empty(4, 32, N.SF_ROWMAJOR)
    st = out.c_struct()
    st.cols = 24  # not a multiple of 16
    rc = N.lib().nvfp4_quantize_noalloc(x.data_ptr(), N.BF16, 4, 24, 24, ctypes.byref(st), None,
                                        None)
    assert rc == N.ERR_UNSUPPORTED_SHAPE
