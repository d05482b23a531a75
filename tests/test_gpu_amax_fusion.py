"""GPU: the tensor amax handed from a GEMM epilogue to the next quantization.

The recipe's tensor scale is s_t = amax(x) / (6 * 448): the FP32 tensor-level
scale of the two-level NVFP4 scaling (tailorednewshub.com LongLive-2.0 article,
section "Entrenamiento NVFP4"), with the amax mapped onto the largest E2M1
value times the largest E4M3 value.  When x is
the output of an nvfp4_gemm, the GEMM can accumulate max|x| over the values it
stores (c_amax) and nvfp4_quantize can take that word (amax_in) instead of
running its own amax pass.  These tests check that the hand-off changes no
byte: c_amax is exactly max|C| of what was stored, and the quantization fed
from it is identical to the one that measured the amax itself (and to the
oracle)."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_08_b200 as nv

from _util import assert_quant_equal, bits

pytestmark = pytest.mark.gpu


def _operands(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    a = (torch.randn(M, K, generator=g) * 2).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    return nv.quantize(a.cuda()), nv.quantize(w.cuda())


def _amax_word():
    return torch.zeros(1, dtype=torch.float32, device="cuda")


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (300, 768, 1024), (2640, 3072, 3072)])
def test_c_amax_is_max_abs_of_stored_output(M, N, K, out_dtype):
    qa, qw = _operands(M, N, K, seed=M + N + K)
    c_amax = _amax_word()
    y = nv.gemm(qa, qw, out_dtype=out_dtype, c_amax=c_amax)
    torch.cuda.synchronize()
    # exact: the max of the stored values is one of them, no arithmetic involved
    assert c_amax.item() == y.float().abs().max().item()
    assert nv.device_status() == 0


def test_c_amax_keeps_a_larger_running_value_and_accumulates():
    qa, qw = _operands(256, 512, 256, seed=3)
    y = nv.gemm(qa, qw, out_dtype=torch.float32)
    m = y.abs().max().item()
    word = torch.full((1,), 4 * m, dtype=torch.float32, device="cuda")
    nv.gemm(qa, qw, out_dtype=torch.float32, c_amax=word)
    assert word.item() == 4 * m
    # two GEMMs into one word: the max over both outputs
    qb, qv = _operands(130, 256, 512, seed=4)
    word.zero_()
    y1 = nv.gemm(qa, qw, out_dtype=torch.bfloat16, c_amax=word)
    y2 = nv.gemm(qb, qv, out_dtype=torch.bfloat16, c_amax=word)
    assert word.item() == max(y1.float().abs().max().item(), y2.float().abs().max().item())


@pytest.mark.parametrize("layout", [nv.SF_ROWMAJOR, nv.SF_MMA128x4])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_from_amax_in_matches_own_amax_pass(orc, layout, dtype):
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(777, 1040, generator=g) * 3).to(dtype)
    xd = x.cuda()
    ref = nv.quantize(xd, sf_layout=layout)
    word = torch.full((1,), xd.float().abs().max().item(), dtype=torch.float32, device="cuda")
    q = nv.quantize(xd, sf_layout=layout, amax_in=word)
    torch.cuda.synchronize()
    assert word.item() == 0.0  # consumed and reset
    assert torch.equal(q.codes, ref.codes) and torch.equal(q.sf, ref.sf)
    assert torch.equal(q.s_t, ref.s_t)
    assert_quant_equal(orc, q, bits(x), layout)
    assert nv.device_status() == 0


def test_gemm_to_quantize_chain(orc):
    """C = A W^T with c_amax, then quantize C from it: same bytes as quantizing
    C with the amax pass, and as the oracle's quantization of C."""
    qa, qw = _operands(517, 1024, 768, seed=21)
    word = _amax_word()
    y = nv.gemm(qa, qw, out_dtype=torch.bfloat16, c_amax=word)
    q = nv.quantize(y, amax_in=word)
    ref = nv.quantize(y)
    torch.cuda.synchronize()
    assert word.item() == 0.0
    assert torch.equal(q.codes, ref.codes) and torch.equal(q.sf, ref.sf)
    assert_quant_equal(orc, q, bits(y), nv.SF_MMA128x4)
    # the word is ready for the next producer: a second round trip agrees again
    nv.gemm(qa, qw, out_dtype=torch.bfloat16, out=y, c_amax=word)
    q2 = nv.quantize(y, amax_in=word)
    assert torch.equal(q2.codes, ref.codes) and torch.equal(q2.s_t, ref.s_t)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_gelu_epilogue_amax_and_requant(orc, out_dtype):
    """FFN up-projection with the GELU epilogue feeding the intermediate
    requantization: c_amax is exactly max|C| of the stored GELU values, and the
    quantization fed from it is the one the oracle makes of those values."""
    qa, qw = _operands(390, 1024, 512, seed=51)
    word = _amax_word()
    h = nv.gemm(qa, qw, out_dtype=out_dtype, c_amax=word, act=nv.ACT_GELU_TANH)
    torch.cuda.synchronize()
    assert word.item() == h.float().abs().max().item()
    assert h.float().min().item() > -0.171  # GELU's floor
    q = nv.quantize(h, amax_in=word)
    assert word.item() == 0.0
    assert_quant_equal(orc, q, bits(h), nv.SF_MMA128x4)
    assert nv.device_status() == 0


def test_amax_in_out_of_domain_is_reported_and_reset():
    x = torch.ones(64, 64, device="cuda", dtype=torch.bfloat16)
    word = torch.full((1,), 1e38, dtype=torch.float32, device="cuda")  # s_t > 2^100
    nv.quantize(x, amax_in=word)
    assert nv.device_status() == nv._native.ERR_DOMAIN
    assert word.item() == 0.0
    zero = nv.quantize(x, amax_in=word)  # amax 0: s_t = 0, every code +0
    torch.cuda.synchronize()
    assert zero.s_t.item() == 0.0 and not zero.codes.any()
    assert nv.device_status() == 0
    assert np.isfinite(word.item())


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_c_amax_per_column_group(out_dtype):
    """c_amax_cols = 256, 512, N: word g is max|C| over its own columns only."""
    qa, qw = _operands(300, 1536, 512, seed=31)
    for cols in (256, 512, 1536):
        words = torch.zeros(1536 // cols, dtype=torch.float32, device="cuda")
        y = nv.gemm(qa, qw, out_dtype=out_dtype, c_amax=words, c_amax_cols=cols)
        torch.cuda.synchronize()
        ref = y.float().abs().reshape(300, 1536 // cols, cols).amax(dim=(0, 2))
        assert torch.equal(words, ref), (cols, words, ref)


def test_kv_chunk_from_qkv_gemm_amax(orc):
    """QKV projection with one amax word per Q/K/V third; the K and V words
    feed kv_quant_chunk, which then writes the same bytes as with its own
    amax pass, and leaves both words at 0."""
    tpf, heads, hd = 16, 4, 64
    d = heads * hd
    qa, qw = _operands(3 * tpf, 3 * d, 256, seed=41)
    words = torch.zeros(3, dtype=torch.float32, device="cuda")
    qkv = nv.gemm(qa, qw, out_dtype=torch.bfloat16, c_amax=words, c_amax_cols=d)
    torch.cuda.synchronize()
    assert words[1].item() == qkv[:, d:2 * d].float().abs().max().item()
    assert words[2].item() == qkv[:, 2 * d:].float().abs().max().item()
    fused = nv.KVCache(4, tpf, heads, hd)
    plain = nv.KVCache(4, tpf, heads, hd)
    fused.quant_chunk(qkv[:, d:2 * d], qkv[:, 2 * d:], [3, 0, 2], k_amax_in=words[1:2],
                      v_amax_in=words[2:3])
    plain.quant_chunk(qkv[:, d:2 * d], qkv[:, 2 * d:], [3, 0, 2])
    torch.cuda.synchronize()
    assert words[1].item() == 0.0 and words[2].item() == 0.0
    for name in ("k_codes", "v_codes", "k_sf", "v_sf", "k_st", "v_st"):
        assert torch.equal(getattr(fused, name), getattr(plain, name)), name
    assert nv.device_status() == 0
