"""GPU parity: the NVFP4 KV-cache chunk codec (kv_quant_chunk /
kv_dequant_window) against the CPU oracle, byte for byte."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_08_b200 as nv
from nvfp4_w4a4_quantized_08_b200 import workloads as wl

from _util import bits, np_u8

pytestmark = pytest.mark.gpu


def _check_slots(orc, cache, kv_bits_chunks, tpf, heads, hd):
    """kv_bits_chunks: list of (slots, k_bits, v_bits, n_frames) written in order."""
    per = tpf * heads * hd
    for slots, kb, vb, nf in kv_bits_chunks:
        for plane, (src, codes_pool, sf_pool, st_pool) in enumerate(
                [(kb, cache.k_codes, cache.k_sf, cache.k_st),
                 (vb, cache.v_codes, cache.v_sf, cache.v_st)]):
            c, s, t = orc.kv_quant_chunk(src, nf, tpf, heads, hd)
            gc = np_u8(codes_pool)
            gs = np_u8(sf_pool)
            gt = st_pool.cpu().numpy()
            for f, slot in enumerate(slots):
                np.testing.assert_array_equal(gc[slot], c[f])
                np.testing.assert_array_equal(gs[slot], s[f])
                assert np.float32(gt[slot]) == np.float32(t[f])
    assert per % 16 == 0


def test_window_codec_one_layer(orc):
    """One layer's cache: K, V [10560, 24, 128] (3 sink + 9 window frames of 880
    tokens), quantized in chunks of 8 and 4 frames, then the 12-slot window
    (sinks first) rebuilt to bf16."""
    tpf, heads, hd = wl.TOKENS_PER_FRAME, wl.HEADS, wl.HEAD_DIM
    k, v = wl.kv_window()
    cache = nv.KVCache(16, tpf, heads, hd)
    kg, vg = k.cuda(), v.cuda()
    # pool slots: frames 0..7 -> slots 4..11, frames 8..11 -> slots 0..3
    chunks = [(list(range(4, 12)), 0, 8), ([0, 1, 2, 3], 8, 4)]
    written = []
    for slots, f0, nf in chunks:
        t0, t1 = f0 * tpf, (f0 + nf) * tpf
        cache.quant_chunk(kg[t0:t1], vg[t0:t1], slots)
        written.append((slots, bits(k[t0:t1]).reshape(-1), bits(v[t0:t1]).reshape(-1), nf))
    assert nv.device_status() == 0
    _check_slots(orc, cache, written, tpf, heads, hd)
    window = [4, 5, 6] + [7, 8, 9, 10, 11, 0, 1, 2, 3]
    ko, vo = cache.dequant_window(window)
    pool_c = np_u8(cache.k_codes)
    pool_s = np_u8(cache.k_sf)
    pool_t = cache.k_st.cpu().numpy()
    ref_k = orc.kv_dequant_window(pool_c, pool_s, pool_t, window, tpf, heads, hd)
    np.testing.assert_array_equal(bits(ko), ref_k)
    ref_v = orc.kv_dequant_window(np_u8(cache.v_codes), np_u8(cache.v_sf),
                                  cache.v_st.cpu().numpy(), window, tpf, heads, hd)
    np.testing.assert_array_equal(bits(vo), ref_v)


def test_chunk_from_fused_qkv_output(orc):
    """K and V read straight out of a [tokens, 3*dim] QKV output (token stride 9216)."""
    tpf, heads, hd = 880, 24, 128
    g = torch.Generator().manual_seed(11)
    qkv = (torch.randn(3 * tpf, 3 * heads * hd, generator=g) * 2).to(torch.bfloat16)
    cache = nv.KVCache(5, tpf, heads, hd)
    q = qkv.cuda()
    d = heads * hd
    cache.quant_chunk(q[:, d:2 * d], q[:, 2 * d:], [4, 0, 2])
    kb = bits(qkv[:, d:2 * d].contiguous()).reshape(-1)
    vb = bits(qkv[:, 2 * d:].contiguous()).reshape(-1)
    _check_slots(orc, cache, [([4, 0, 2], kb, vb, 3)], tpf, heads, hd)


@pytest.mark.parametrize("tpf,heads,hd,nf", [(7, 3, 16, 1), (5, 2, 48, 8), (13, 4, 64, 3),
                                             (1, 1, 16, 5), (33, 5, 32, 2)])
def test_small_geometries(orc, tpf, heads, hd, nf):
    g = torch.Generator().manual_seed(tpf * 100 + hd)
    k = (torch.randn(nf * tpf, heads, hd, generator=g) * 3).to(torch.bfloat16)
    v = (torch.randn(nf * tpf, heads, hd, generator=g) * 0.1).to(torch.bfloat16)
    cache = nv.KVCache(10, tpf, heads, hd)
    slots = list(range(9, 9 - nf, -1))
    cache.quant_chunk(k.cuda(), v.cuda(), slots)
    _check_slots(orc, cache, [(slots, bits(k).reshape(-1), bits(v).reshape(-1), nf)], tpf, heads,
                 hd)
    window = [slots[0], slots[-1], slots[0]]  # repeats allowed
    ko, vo = cache.dequant_window(window)
    ref = orc.kv_dequant_window(np_u8(cache.k_codes), np_u8(cache.k_sf), cache.k_st.cpu().numpy(),
                                window, tpf, heads, hd)
    np.testing.assert_array_equal(bits(ko), ref)


def test_window_into_16_byte_aligned_outputs(orc):
    tpf, heads, hd = 9, 2, 32
    g = torch.Generator().manual_seed(17)
    k = (torch.randn(3 * tpf, heads, hd, generator=g)).to(torch.bfloat16)
    cache = nv.KVCache(4, tpf, heads, hd)
    cache.quant_chunk(k.cuda(), k.cuda(), [3, 1, 0])
    n = 3 * tpf * heads * hd
    kb = torch.empty(n + 8, dtype=torch.bfloat16, device="cuda")[8:].view(3 * tpf, heads, hd)
    vb = torch.empty(n + 8, dtype=torch.bfloat16, device="cuda")[8:].view(3 * tpf, heads, hd)
    window = [0, 3, 1]
    cache.dequant_window(window, kb, vb)
    ref = orc.kv_dequant_window(np_u8(cache.k_codes), np_u8(cache.k_sf), cache.k_st.cpu().numpy(),
                                window, tpf, heads, hd)
    np.testing.assert_array_equal(bits(kb), ref)
    np.testing.assert_array_equal(bits(vb), ref)


def test_bad_slots_rejected_on_host():
    cache = nv.KVCache(4, 8, 2, 16)
    k = torch.zeros(16, 2, 16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.NVFP4Error):
        cache.quant_chunk(k, k, [0, 4])  # out of range
    with pytest.raises(nv.NVFP4Error):
        cache.quant_chunk(k, k, [1, 1])  # repeated
    with pytest.raises(nv.NVFP4Error):
        cache.dequant_window([0, -1])


@pytest.mark.parametrize("token_stride_extra", [0, 64])
def test_four_over_six_chunk_matches_oracle(orc, token_stride_extra):
    """Four Over Six chunks: codes, scales and s_t byte-identical to the
    oracle's rule, some block scales different from the onto-6 rule, and the
    window rebuild of those slots identical to the oracle's."""
    tpf, heads, hd, nf = 40, 6, 64, 3
    g = torch.Generator().manual_seed(23)
    sig = torch.tensor([0.5, 1.0, 2.0, 3.0, 4.0, 0.7]).view(1, heads, 1)
    kv = (torch.randn(nf * tpf, heads, hd, generator=g) * sig).to(torch.bfloat16)
    width = heads * hd + token_stride_extra
    buf = torch.zeros(nf * tpf, width, dtype=torch.bfloat16)
    buf[:, :heads * hd] = kv.reshape(nf * tpf, -1)
    cache = nv.KVCache(5, tpf, heads, hd, scale_rule=nv.SCALE_FOUR_OVER_SIX)
    d = buf.cuda()
    cache.quant_chunk(d[:, :heads * hd], d[:, :heads * hd], [4, 1, 2])
    bits_flat = bits(buf).reshape(-1)
    codes, sf, st = orc.kv_quant_chunk(bits_flat, nf, tpf, heads, hd, token_stride=width, rule=1)
    _, sf6, _ = orc.kv_quant_chunk(bits_flat, nf, tpf, heads, hd, token_stride=width, rule=0)
    assert np.any(sf != sf6)
    for f, slot in enumerate([4, 1, 2]):
        np.testing.assert_array_equal(np_u8(cache.k_codes[slot]), codes[f])
        np.testing.assert_array_equal(np_u8(cache.k_sf[slot]), sf[f])
        np.testing.assert_array_equal(np_u8(cache.v_codes[slot]), codes[f])
        assert float(cache.k_st[slot].item()) == float(st[f])
    window = [2, 4, 1]
    ko, _ = cache.dequant_window(window)
    ref = orc.kv_dequant_window(np_u8(cache.k_codes), np_u8(cache.k_sf),
                                cache.k_st.cpu().numpy(), window, tpf, heads, hd)
    np.testing.assert_array_equal(bits(ko), ref)
    assert nv.device_status() == 0


def _f32_steps_errors(blocks, s_t):
    """Approximate (binary64) squared errors of each block under onto-6 and
    onto-4, from the recipe's binary32 steps; used only to pick test blocks."""
    import ml_dtypes
    f32 = np.float32
    amax_b = np.max(np.abs(blocks), axis=1).astype(f32)
    out = []
    for top in (6.0, 4.0):
        r = amax_b / (f32(top) * f32(s_t))
        sb = np.minimum(r, f32(448)).astype(ml_dtypes.float8_e4m3fn)
        sbv = sb.astype(f32)
        d = (sbv * f32(s_t))[:, None]
        with np.errstate(divide="ignore", invalid="ignore"):
            y = np.clip(blocks / d, -6, 6)
        q = y.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
        q[sbv == 0] = 0
        recon = np.abs(q) * sbv.astype(np.float64)[:, None] * float(s_t)
        out.append((sb.view(np.uint8), ((np.abs(blocks) - recon) ** 2).sum(axis=1)))
    return amax_b, out


def test_four_over_six_near_ties_match_oracle(orc):
    """Blocks whose two errors are within the binary32 screening margin (so
    the kernel decides them in binary64), plus exact ties, plus ordinary
    blocks: the chunk's scales and codes equal the oracle's."""
    rng = np.random.default_rng(77)
    s_t = np.float32(8.0) / np.float32(2688.0)
    pool = rng.normal(0, 1, (40000, 16)) * rng.choice([0.3, 1.0, 2.5], (40000, 1))
    pool = torch.from_numpy(np.clip(pool, -7.5, 7.5).astype(np.float32)).to(torch.bfloat16)
    blocks = pool.float().numpy()
    amax_b, ((s6, e6), (s4, e4)) = _f32_steps_errors(blocks, s_t)
    near = np.nonzero((s4 != s6) & (np.abs(e4 - e6) <= 2.0 ** -12 * amax_b.astype(np.float64) ** 2))[0]
    assert near.size >= 20
    tie = np.zeros((2, 16), np.float32)
    tie[0, :] = 3.0  # both rules code it exactly
    tie[1, ::2] = 1.5
    top = np.zeros((1, 16), np.float32)
    top[0, 0] = 8.0  # the chunk's amax: s_t = 8 / 2688
    chosen = np.concatenate([top, tie, blocks[near[:96]], blocks[:64]])
    chunk = torch.from_numpy(chosen).to(torch.bfloat16)  # [tpf, heads=1, head_dim=16]
    tpf = chunk.shape[0]
    cache = nv.KVCache(2, tpf, 1, 16, scale_rule=nv.SCALE_FOUR_OVER_SIX)
    d = chunk.reshape(tpf, 16).cuda()
    cache.quant_chunk(d, d, [1])
    codes, sf, st = orc.kv_quant_chunk(bits(chunk).reshape(-1), 1, tpf, 1, 16, rule=1)
    assert float(st[0]) == float(s_t)
    np.testing.assert_array_equal(np_u8(cache.k_sf[1]), sf[0])
    np.testing.assert_array_equal(np_u8(cache.k_codes[1]), codes[0])
    assert nv.device_status() == 0
