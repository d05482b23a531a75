"""GPU parity: nvfp4_quantize / nvfp4_dequantize against the CPU oracle,
byte for byte (codes, E4M3 scales in both layouts, tensor scale, bf16)."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_08_b200 as nv
from nvfp4_w4a4_quantized_08_b200 import workloads as wl

from _util import assert_quant_equal, bits, np_u8

pytestmark = pytest.mark.gpu

LAYOUTS = [nv.SF_ROWMAJOR, nv.SF_MMA128x4]


def _q(x_cpu, layout, **kw):
    return nv.quantize(x_cpu.cuda(), sf_layout=layout, **kw)


@pytest.mark.parametrize("layout", LAYOUTS)
def test_tiny_pair_fp32(orc, layout):
    """Round trip, tiny: A and B fp32 256x256 ~ N(0,1), 2% outliers x50."""
    a, b = wl.tiny_pair()
    for x in (a, b):
        q = _q(x, layout)
        codes, sf, st = assert_quant_equal(orc, q, bits(x), layout)
        deq = nv.dequantize(q)
        np.testing.assert_array_equal(bits(deq), orc.dequantize(codes, sf, st))
    assert nv.device_status() == 0


@pytest.mark.parametrize("layout", LAYOUTS)
def test_qkv_activations(orc, layout):
    """Activations of one 3-frame chunk: 2640 x 3072 bf16, 8 outlier channels x30."""
    x = wl.activations()
    q = _q(x, layout)
    codes, sf, st = assert_quant_equal(orc, q, bits(x), layout)
    np.testing.assert_array_equal(bits(nv.dequantize(q)), orc.dequantize(codes, sf, st))


def test_ffn_intermediate(orc):
    """FFN intermediate requant input: GELU(N(0,1)) 2640 x 14336 bf16."""
    x = wl.gelu_activations()
    q = _q(x, nv.SF_MMA128x4)
    assert_quant_equal(orc, q, bits(x), nv.SF_MMA128x4)


@pytest.mark.parametrize("rows,cols", [(1, 16), (3, 48), (127, 272), (129, 64), (300, 1040),
                                       (33, 80), (256, 4096)])
@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_ragged_shapes(orc, rows, cols, layout, dtype):
    g = torch.Generator().manual_seed(rows * 7919 + cols)
    x = (torch.randn(rows, cols, generator=g) * torch.exp(2 * torch.randn(rows, 1, generator=g)))
    x = x.to(dtype)
    q = _q(x, layout)
    codes, sf, st = assert_quant_equal(orc, q, bits(x), layout)
    np.testing.assert_array_equal(bits(nv.dequantize(q)), orc.dequantize(codes, sf, st))


@pytest.mark.parametrize("layout", LAYOUTS)
def test_row_stride(orc, layout):
    """ld > cols: quantize a column slice of a wider tensor; dequantize into a
    wider output."""
    g = torch.Generator().manual_seed(3)
    big = torch.randn(200, 520, generator=g).to(torch.bfloat16)
    view = big[:, 8:392]
    x = big.cuda()[:, 8:392]
    q = nv.quantize(x, sf_layout=layout)
    codes, sf, st = assert_quant_equal(orc, q, bits(view.contiguous()), layout)
    out = torch.full((200, 400), 7.0, dtype=torch.bfloat16, device="cuda")
    nv.dequantize(q, out=out[:, :384])
    np.testing.assert_array_equal(bits(out[:, :384]), orc.dequantize(codes, sf, st))
    assert torch.all(out[:, 384:] == 7.0)


@pytest.mark.parametrize("layout", LAYOUTS)
def test_dequantize_to_16_byte_aligned_destinations(orc, layout):
    """Destinations 16- but not 32-byte aligned (and a row stride of 8 mod 16
    elements) take the two-store path; the bytes must not change."""
    g = torch.Generator().manual_seed(13)
    x = torch.randn(130, 272, generator=g).to(torch.bfloat16)
    q = nv.quantize(x.cuda(), sf_layout=layout)
    codes, sf, st = assert_quant_equal(orc, q, bits(x), layout)
    ref = orc.dequantize(codes, sf, st)
    buf = torch.empty(130 * 272 + 8, dtype=torch.bfloat16, device="cuda")
    flat = buf[8:].view(130, 272)  # base 16 bytes past a 256-byte boundary
    nv.dequantize(q, out=flat)
    np.testing.assert_array_equal(bits(flat), ref)
    wide = torch.empty(130 * 280 + 8, dtype=torch.bfloat16, device="cuda")[8:].view(130, 280)
    nv.dequantize(q, out=wide[:, :272])  # ld = 280
    np.testing.assert_array_equal(bits(wide[:, :272]), ref)


def test_given_tensor_scale(orc):
    g = torch.Generator().manual_seed(4)
    x = (torch.randn(96, 160, generator=g) * 5).to(torch.bfloat16)
    for st in (0.001, 0.02, 1.5):
        s = torch.tensor([st], dtype=torch.float32, device="cuda")
        q = _q(x, nv.SF_MMA128x4, s_t=s)
        assert_quant_equal(orc, q, bits(x), nv.SF_MMA128x4, s_t_in=np.float32(st))


def _tie_tensor(orc):
    """Elements exactly on E2M1 rounding boundaries and one ulp either side,
    and block maxima exactly on E4M3 rounding boundaries."""
    e = -3
    s_t = 2.0 ** e
    rows = []
    # E2M1 decision points with s_b = 1.0 (block max = 6 -> r = 1), d = s_t
    for t in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0):
        for delta in (-1, 0, 1):
            v = np.nextafter(np.float32(t * s_t), np.float32(np.inf) if delta > 0 else 0.0) \
                if delta else np.float32(t * s_t)
            row = np.zeros(16, np.float32)
            row[0] = 6 * s_t
            row[1] = v
            row[2] = -v
            rows.append(row)
    # E4M3 decision points: block max = 6 * s_t * m for midpoints m
    vals = [orc.e4m3_value(c) for c in range(0x7F)]
    for c in range(1, 0x7E, 5):
        m = (vals[c] + vals[c + 1]) / 2
        row = np.zeros(16, np.float32)
        row[0] = np.float32(6 * s_t * m)
        row[3] = np.float32(-3 * s_t * m)
        rows.append(row)
    amax_row = np.zeros(16, np.float32)
    amax_row[0] = 2688 * s_t  # tensor amax -> s_t exactly 2^e
    rows.append(amax_row)
    return np.stack(rows).astype(np.float32)


def test_ties_fp32(orc):
    x = _tie_tensor(orc)
    for layout in LAYOUTS:
        q = _q(torch.from_numpy(x), layout)
        assert_quant_equal(orc, q, x, layout)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_dense_ties_power_of_two_tensor_scale(orc, dtype):
    """bf16-valued data with amax 5.25, so s_t = 5.25 / 2688 = 2^-9 exactly:
    many quotients land exactly on E2M1 and E4M3 rounding boundaries, in most
    warps of the launch (every element position of a block gets some)."""
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(1000, 4096, generator=g) * 1.5).clamp(-5.25, 5.25)
    x = x.to(torch.bfloat16).to(dtype)
    x[7, 123] = 5.25
    for layout in LAYOUTS:
        q = _q(x, layout)
        assert float(q.s_t.cpu()[0]) == 2.0 ** -9
        assert_quant_equal(orc, q, bits(x), layout)


def test_zero_and_special_values(orc):
    x = torch.zeros(130, 64)
    q = _q(x, nv.SF_MMA128x4)
    assert_quant_equal(orc, q, x.numpy(), nv.SF_MMA128x4)
    assert float(q.s_t.cpu()[0]) == 0.0 and not np_u8(q.codes).any()
    y = torch.randn(130, 64, generator=torch.Generator().manual_seed(5))
    y[5, 16:32] = 0.0
    y[6, 0] = -0.0
    y[7, :16] = -1e-9
    y[8, 3] = 1e4
    for dtype in (torch.float32, torch.bfloat16):
        yy = y.to(dtype)
        q = _q(yy, nv.SF_ROWMAJOR)
        assert_quant_equal(orc, q, bits(yy), nv.SF_ROWMAJOR)
    assert nv.device_status() == 0


def test_domain_error_is_reported(orc):
    tiny = torch.full((4, 32), 1e-33, dtype=torch.float32)
    nv.quantize(tiny.cuda())
    assert nv.device_status() == nv._native.ERR_DOMAIN
    assert nv.device_status() == 0  # read-and-clear
    bad = torch.zeros(4, 32)
    bad[1, 1] = float("nan")
    nv.quantize(bad.cuda())
    assert nv.device_status() == nv._native.ERR_DOMAIN
    # a normal call afterwards is unaffected
    x = torch.randn(4, 32)
    q = _q(x, nv.SF_ROWMAJOR)
    assert_quant_equal(orc, q, x.numpy(), nv.SF_ROWMAJOR)


def test_workspace_returns_to_zero():
    ws = torch.zeros(nv._native.lib().nvfp4_workspace_bytes(), dtype=torch.uint8, device="cuda")
    x = torch.randn(1000, 512, device="cuda").to(torch.bfloat16)
    for _ in range(3):
        nv.quantize(x, ws=ws)
    torch.cuda.synchronize()
    assert not ws.any()
    q1 = nv.quantize(x, ws=ws)
    q2 = nv.quantize(x, ws=ws)
    assert torch.equal(q1.codes, q2.codes) and torch.equal(q1.sf, q2.sf)
