"""GPU parity: nvfp4_window_attention (attention straight from the NVFP4 KV
cache) against the oracle's binary64 attention.

K and V are quantized into the cache on the GPU (kv_quant_chunk) and by the
oracle from the same seeded bf16 inputs; the GPU pools are first checked equal
to the oracle's byte for byte, and the oracle's own pools are rebuilt to bf16
(its window rebuild) and fed to its attention.

Bound per output element, E = sum_j p_j |v_j| (the scale of the P V sum):
  |o - o_ref| <= 2^-6 E + 2^-8 |o_ref|.
The kernel rounds each probability to bf16 before P V while the normaliser
sums the unrounded ones (<= 2^-8 E); scores are fp32 sums of 128 exact
products (relative 2^-17 of sum |q k|, a logit error of at most ~2^-12, which
moves the output by ~2^-11 E); the fp32 accumulations over up to ~10^4 tokens
add ~2^-10 E each to the numerator and the normaliser; the output is rounded to
bf16 (2^-8 |o|).  2^-6 E covers the sum with a factor ~2 to spare; an indexing
or masking error moves outputs by O(E)."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_08_b200 as nv
from nvfp4_w4a4_quantized_08_b200 import workloads as wl

from _util import bits, np_u8

pytestmark = pytest.mark.gpu

HD = 128


def _build(orc, n_slots, tpf, heads, chunks, seed):
    """chunks: list of (slot list, n_frames) written in order.  Returns the GPU
    cache and the oracle's pools (codes, sf, st per plane)."""
    cache = nv.KVCache(n_slots, tpf, heads, HD)
    per = tpf * heads * HD
    pools = {p: [np.zeros((n_slots, per // 2), np.uint8), np.zeros((n_slots, per // 16), np.uint8),
                 np.zeros(n_slots, np.float32)] for p in ("k", "v")}
    for ci, (slots, nf) in enumerate(chunks):
        k = wl.kv_tensor(seed + 2 * ci, nf * tpf, heads, HD)
        v = wl.kv_tensor(seed + 2 * ci + 1, nf * tpf, heads, HD)
        cache.quant_chunk(k.cuda(), v.cuda(), slots)
        for p, x in (("k", k), ("v", v)):
            c, s, t = orc.kv_quant_chunk(bits(x).reshape(-1), nf, tpf, heads, HD)
            for f, slot in enumerate(slots):
                pools[p][0][slot], pools[p][1][slot], pools[p][2][slot] = c[f], s[f], t[f]
    for p, (cp, sp, tp) in (("k", (cache.k_codes, cache.k_sf, cache.k_st)),
                            ("v", (cache.v_codes, cache.v_sf, cache.v_st))):
        np.testing.assert_array_equal(np_u8(cp), pools[p][0])
        np.testing.assert_array_equal(np_u8(sp), pools[p][1])
        np.testing.assert_array_equal(tp.cpu().numpy(), pools[p][2])
    return cache, pools


def _oracle(orc, pools, window, tpf, heads, q_bits, scale, rows=None):
    k = orc.kv_dequant_window(*pools["k"], window, tpf, heads, HD)
    v = orc.kv_dequant_window(*pools["v"], window, tpf, heads, HD)
    return orc.window_attention(q_bits, k, v, scale, rows=rows)


def _assert_close(o_gpu, o_ref, E):
    o_gpu = o_gpu.astype(np.float64)
    tol = 2.0 ** -6 * E + 2.0 ** -8 * np.abs(o_ref)
    err = np.abs(o_gpu - o_ref)
    bad = ~(err <= tol)
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{bad.sum()} of {bad.size} outside tolerance; first {i}: "
                             f"gpu {o_gpu[i]} ref {o_ref[i]} E {E[i]}")


def _q(tq, heads, seed, std=1.0):
    return wl.randn((tq, heads * HD), 6, seed, std=std)


@pytest.mark.parametrize("tq", [1, 100, 130])
def test_small_window_ragged(orc, tq):
    """3 slots of 80 tokens (240 keys: three full 64-token tiles and a 48-token
    tail that straddles slots), 2 heads, tq = 1, 100 and 130 queries."""
    tpf, heads = 80, 2
    cache, pools = _build(orc, 4, tpf, heads, [([3, 0, 1], 3)], seed=10)
    window = [1, 3, 0]
    q = _q(tq, heads, seed=tq)
    out = cache.window_attention(q.cuda(), window)
    ref, E = _oracle(orc, pools, window, tpf, heads, bits(q), HD ** -0.5)
    _assert_close(out.float().cpu().numpy().reshape(tq, heads, HD), ref, E)
    assert nv.device_status() == 0


def test_repeated_slots_strided_q_and_scale(orc):
    """A slot listed twice, Q read out of a wider (QKV-like) buffer, the output
    written into a wider buffer whose other columns stay untouched, and a
    non-default softmax scale."""
    tpf, heads = 48, 3
    cache, pools = _build(orc, 3, tpf, heads, [([0, 1, 2], 3)], seed=20)
    window = [2, 0, 2, 1]
    tq = 70
    q = _q(tq, heads, seed=5, std=2.0)
    qkv = torch.zeros(tq, 3 * heads * HD, dtype=torch.bfloat16)
    qkv[:, :heads * HD] = q
    wide = torch.full((tq, heads * HD + 16), 5.0, dtype=torch.bfloat16, device="cuda")
    cache.window_attention(qkv.cuda()[:, :heads * HD], window, scale=0.05,
                           out=wide[:, :heads * HD])
    ref, E = _oracle(orc, pools, window, tpf, heads, bits(q), 0.05)
    _assert_close(wide[:, :heads * HD].float().cpu().numpy().reshape(tq, heads, HD), ref, E)
    assert torch.all(wide[:, heads * HD:] == 5.0)


def test_dit_window_sampled_rows(orc):
    """The step's shape: 2640 queries (3 frames), 24 heads, a 12-slot window of
    880-token frames (3 sinks + 6 cached + the 3 new frames: 10560 keys),
    quantized in chunks of 8 and 4 frames; sampled query rows, all heads."""
    tpf, heads = wl.TOKENS_PER_FRAME, wl.HEADS
    cache, pools = _build(orc, 15, tpf, heads,
                          [(list(range(0, 8)), 8), ([8, 9, 10, 11], 4), ([12, 13, 14], 3)],
                          seed=30)
    window = [0, 1, 2] + [6, 7, 8, 9, 10, 11] + [12, 13, 14]
    tq = 3 * tpf
    q = _q(tq, heads, seed=7)
    out = cache.window_attention(q.cuda(), window)
    rows = [0, 1, 63, 64, 1000, 2047, 2560, 2600, tq - 1]
    ref, E = _oracle(orc, pools, window, tpf, heads, bits(q), HD ** -0.5, rows=rows)
    _assert_close(out[rows].float().cpu().numpy().reshape(len(rows), heads, HD), ref, E)
    assert nv.device_status() == 0
