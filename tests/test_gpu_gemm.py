"""GPU parity: nvfp4_gemm against the oracle's FP64 reference.

Pass criterion per output element: |y_gpu - y_ref| <= 1e-3 * sum_k |a_k w_k|,
plus half a bf16 ulp of |y_ref| for bf16 output; y_ref is the binary64 sum of
the exactly dequantized operands.  The operands themselves are checked
byte-exact against the oracle's quantization first."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_08_b200 as nv
from nvfp4_w4a4_quantized_08_b200 import workloads as wl

from _util import assert_gelu_gemm_close, assert_gemm_close, assert_quant_equal, bits

pytestmark = pytest.mark.gpu


def _operands(orc, a_cpu, w_cpu):
    qa = nv.quantize(a_cpu.cuda())
    qw = nv.quantize(w_cpu.cuda())
    oa = assert_quant_equal(orc, qa, bits(a_cpu), nv.SF_MMA128x4)
    ow = assert_quant_equal(orc, qw, bits(w_cpu), nv.SF_MMA128x4)
    return qa, qw, oa, ow


def _sample_rows(M, n_random=32, seed=0):
    rng = np.random.default_rng(seed)
    tail_start = (M // 128) * 128
    rows = set(rng.choice(M, size=min(n_random, M), replace=False).tolist())
    rows.update(range(tail_start, M))  # the whole ragged last tile
    rows.update([0, M - 1])
    return sorted(rows)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_tiny_gemm_all_elements(orc, out_dtype):
    """FP4 GEMM M = N = K = 256 on the tiny outlier pair; every element checked."""
    a, b = wl.tiny_pair()
    qa, qw, oa, ow = _operands(orc, a, b)
    y = nv.gemm(qa, qw, out_dtype=out_dtype)
    y_ref, S = orc.gemm(oa, ow)
    assert_gemm_close(y.float().cpu().numpy(), y_ref, S, out_dtype == torch.bfloat16)
    assert nv.device_status() == 0


@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (100, 256, 128), (128, 512, 192),
                                   (129, 256, 320), (300, 768, 1024), (77, 256, 4096),
                                   (513, 1024, 256),
                                   # N tails: a last tile without its second 128 W rows
                                   # (384, 640), with them partly padding (200), tiny N
                                   (100, 384, 128), (300, 200, 256), (129, 16, 64),
                                   (513, 640, 192), (1, 48, 64),
                                   # K not a multiple of 64: a last half K step
                                   (100, 256, 32), (300, 256, 96), (129, 384, 160),
                                   (1, 200, 288)])
def test_small_shapes(orc, M, N, K):
    g = torch.Generator().manual_seed(M * 31 + N * 7 + K)
    a = (torch.randn(M, K, generator=g) * 2).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    qa, qw, oa, ow = _operands(orc, a, w)
    y = nv.gemm(qa, qw, out_dtype=torch.float32)
    y_ref, S = orc.gemm(oa, ow)
    assert_gemm_close(y.cpu().numpy(), y_ref, S, False)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_output_row_stride_and_alignment(orc, out_dtype):
    """C written into a wider buffer (ldc = N + 8: rows 16- but not 32-byte
    aligned, the 128-bit store path) and into one whose base is 16 bytes past
    a 32-byte boundary; the columns outside [0, N) stay untouched."""
    M, N, K = 200, 512, 256
    g = torch.Generator().manual_seed(9)
    a = (torch.randn(M, K, generator=g) * 2).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    qa, qw, oa, ow = _operands(orc, a, w)
    y_ref, S = orc.gemm(oa, ow)
    wide = torch.full((M, N + 8), 3.0, dtype=out_dtype, device="cuda")
    nv.gemm(qa, qw, out=wide[:, :N])
    assert_gemm_close(wide[:, :N].float().cpu().numpy(), y_ref, S, out_dtype == torch.bfloat16)
    assert torch.all(wide[:, N:] == 3.0)
    shift = 16 // torch.tensor([], dtype=out_dtype).element_size()
    buf = torch.zeros(M * N + shift, dtype=out_dtype, device="cuda")
    y = buf[shift:].view(M, N)
    nv.gemm(qa, qw, out=y)
    assert_gemm_close(y.float().cpu().numpy(), y_ref, S, out_dtype == torch.bfloat16)
    assert nv.device_status() == 0


def test_qkv_projection(orc):
    """QKV projection: M=2640 (3 frames x 880 tokens), N=9216, K=3072; 32
    random rows plus the whole 80-row tail tile, all columns."""
    wk = wl.qkv()
    qa, qw, oa, ow = _operands(orc, wk.a, wk.w)
    y = nv.gemm(qa, qw, out_dtype=torch.bfloat16)
    rows = _sample_rows(wk.a.shape[0])
    y_ref, S = orc.gemm(oa, ow, rows=rows)
    assert_gemm_close(y[rows].float().cpu().numpy(), y_ref, S, True)


def test_ffn_pair(orc):
    """FFN up (M=2640, N=14336, K=3072) and down (M=2640, N=3072, K=14336) with the
    standalone GELU(N(0,1)) down-projection input."""
    f = wl.ffn()
    qx, qu, ox, ou = _operands(orc, f.x, f.w_up)
    y_up = nv.gemm(qx, qu, out_dtype=torch.float32)
    rows = _sample_rows(f.x.shape[0], n_random=16, seed=1)
    y_ref, S = orc.gemm(ox, ou, rows=rows)
    assert_gemm_close(y_up[rows].cpu().numpy(), y_ref, S, False)
    qh, qd, oh, od = _operands(orc, f.h, f.w_down)
    y_dn = nv.gemm(qh, qd, out_dtype=torch.bfloat16)
    rows = _sample_rows(f.h.shape[0], n_random=16, seed=2)
    y_ref, S = orc.gemm(oh, od, rows=rows)
    assert_gemm_close(y_dn[rows].float().cpu().numpy(), y_ref, S, True)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (129, 512, 320), (300, 768, 1024),
                                   (129, 384, 320)])
def test_gelu_epilogue(orc, M, N, K, out_dtype):
    """act = GELU (tanh form) in the epilogue, every element against the
    oracle's binary64 GELU of its binary64 GEMM, over inputs that put outputs
    on both sides of zero and far out in the tails."""
    g = torch.Generator().manual_seed(M + 3 * N + 5 * K)
    a = (torch.randn(M, K, generator=g) * 2).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.1).to(torch.bfloat16)
    qa, qw, oa, ow = _operands(orc, a, w)
    y = nv.gemm(qa, qw, out_dtype=out_dtype, act=nv.ACT_GELU_TANH)
    y_ref, S = orc.gemm(oa, ow)
    assert (y_ref < -3).any() and (y_ref > 3).any()
    assert_gelu_gemm_close(orc, y.float().cpu().numpy(), y_ref, S, out_dtype == torch.bfloat16)
    assert nv.device_status() == 0


def test_ffn_up_with_gelu(orc):
    """FFN up-projection M=2640, N=14336, K=3072 with the GELU epilogue, bf16
    output, sampled rows (all columns, the ragged last tile included)."""
    f = wl.ffn()
    qx, qu, ox, ou = _operands(orc, f.x, f.w_up)
    h = nv.gemm(qx, qu, out_dtype=torch.bfloat16, act=nv.ACT_GELU_TANH)
    rows = _sample_rows(f.x.shape[0], n_random=12, seed=3)
    y_ref, S = orc.gemm(ox, ou, rows=rows)
    assert_gelu_gemm_close(orc, h[rows].float().cpu().numpy(), y_ref, S, True)
    assert nv.device_status() == 0


def test_timeout_path_reports_and_recovers(orc):
    """A wait limit of 0 ns with a single output tile and K = 65536 (256 K
    slabs): the epilogue warps wait for the tile's accumulator for the whole
    main loop (about 100 us), far longer than the two suspended polls
    (at most 20 us each) a wait makes before it checks its deadline, so the
    wait runs out.  The kernel must record NVFP4_ERR_TIMEOUT, drain its
    copies, MMAs and stores, free tensor memory and return; each timed-out
    call is followed by a call with the normal limit that must be correct."""
    g = torch.Generator().manual_seed(8)
    K = 65536
    a = torch.randn(128, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(256, K, generator=g) * 0.1).to(torch.bfloat16)
    qa, qw, oa, ow = _operands(orc, a, w)
    y_ref, S = orc.gemm(oa, ow)
    seen = []
    for _ in range(3):
        try:
            nv.set_wait_limit_ns(0)
            nv.gemm(qa, qw, out_dtype=torch.float32)
            seen.append(nv.device_status())
        finally:
            nv.set_wait_limit_ns(2_000_000_000)
        y = nv.gemm(qa, qw, out_dtype=torch.float32)
        assert nv.device_status() == 0
        assert_gemm_close(y.cpu().numpy(), y_ref, S, False)
    assert all(st in (0, nv._native.ERR_TIMEOUT) for st in seen), seen
    assert nv._native.ERR_TIMEOUT in seen, seen


@pytest.mark.parametrize("M,N,K,out_dtype", [(300, 384, 256, torch.bfloat16),
                                             (129, 200, 128, torch.float32),
                                             (100, 640, 192, torch.bfloat16)])
def test_n_tail_amax_and_padding(orc, M, N, K, out_dtype):
    """A GEMM whose N is not a multiple of the 256-column tile: every stored
    element within the bound, the c_amax word equal to max|C| over the stored
    values only (the tile's columns past N hold no output), and the columns of
    a wider output buffer past N left untouched."""
    g = torch.Generator().manual_seed(M + 7 * N + 11 * K)
    a = (torch.randn(M, K, generator=g) * 2).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    qa, qw, oa, ow = _operands(orc, a, w)
    ldc = (N + 63) // 64 * 64 + 64
    buf = torch.full((M, ldc), 7.0, dtype=out_dtype, device="cuda")
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    y = nv.gemm(qa, qw, out=buf[:, :N], c_amax=amax)
    y_ref, S = orc.gemm(oa, ow)
    assert_gemm_close(y.float().cpu().numpy(), y_ref, S, out_dtype == torch.bfloat16)
    assert float(amax.cpu()[0]) == float(y.float().abs().max().cpu())
    assert bool((buf[:, N:] == 7.0).all())
    assert nv.device_status() == 0

