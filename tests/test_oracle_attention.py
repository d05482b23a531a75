"""Pins of the oracle's windowed attention (no GPU).

out = softmax(scale * q k^T) v over the window's tokens, every query seeing
every token (the chunk attends to its sink and window frames and to itself:
hyper.ai LongLive-2.0 summary, section "方法"; 171host.com teardown, section
2.2), in binary64 on bf16 inputs.  Pinned against torch's float64
scaled_dot_product_attention (a library routine), and against closed forms that
a dropped term, a wrong sign, a transposed operand or a wrong head/token index
would break: constant values give that constant, one key gives its value, a
vanishing scale gives the mean of the values, reordering the keys changes
nothing, and each head only sees its own slice.
"""
import numpy as np
import torch

import ml_dtypes


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)


def _val(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _case(tq=5, n_kv=37, heads=3, hd=16, seed=0):
    g = np.random.default_rng(seed)
    q = _bf16_bits(g.standard_normal((tq, heads * hd)) * 1.5)
    k = _bf16_bits(g.standard_normal((n_kv, heads, hd)))
    v = _bf16_bits(g.standard_normal((n_kv, heads, hd)) * 2)
    return q, k, v


def test_matches_torch_sdpa_float64(orc):
    q, k, v = _case()
    tq, (n_kv, heads, hd) = q.shape[0], k.shape
    scale = 0.3
    out, E = orc.window_attention(q, k, v, scale)
    qt = torch.from_numpy(_val(q).reshape(tq, heads, hd)).permute(1, 0, 2)
    kt = torch.from_numpy(_val(k)).permute(1, 0, 2)
    vt = torch.from_numpy(_val(v)).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    np.testing.assert_allclose(out, ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)
    assert np.all(E >= np.abs(out) - 1e-12)


def test_closed_forms(orc):
    q, k, v = _case(seed=1)
    n_kv, heads, hd = k.shape
    const = _bf16_bits(np.full((n_kv, heads, hd), -0.75))
    out, E = orc.window_attention(q, k, const, 0.5)
    np.testing.assert_allclose(out, -0.75, rtol=1e-14)
    np.testing.assert_allclose(E, 0.75, rtol=1e-14)
    one, _ = orc.window_attention(q, k[:1], v[:1], 0.5)
    np.testing.assert_allclose(one, np.broadcast_to(_val(v[:1]), one.shape), rtol=1e-15)
    tiny, _ = orc.window_attention(q, k, v, 1e-30)
    np.testing.assert_allclose(tiny, np.broadcast_to(_val(v).mean(axis=0), tiny.shape),
                               rtol=1e-12, atol=1e-14)


def test_key_order_and_heads(orc):
    q, k, v = _case(seed=2)
    perm = np.random.default_rng(3).permutation(k.shape[0])
    a, _ = orc.window_attention(q, k, v, 0.4)
    b, _ = orc.window_attention(q, k[perm], v[perm], 0.4)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
    # head 1 alone, with the other heads' data replaced, gives the same head-1 output
    k2, v2 = k.copy(), v.copy()
    k2[:, [0, 2]] = _bf16_bits(np.ones_like(_val(k[:, [0, 2]])))
    v2[:, [0, 2]] = _bf16_bits(np.zeros_like(_val(v[:, [0, 2]])))
    c, _ = orc.window_attention(q, k2, v2, 0.4)
    np.testing.assert_array_equal(c[:, 1], a[:, 1])
    assert not np.allclose(c[:, 0], a[:, 0])


def test_row_subset_and_stride(orc):
    q, k, v = _case(tq=9, seed=4)
    wide = np.zeros((q.shape[0], q.shape[1] + 24), np.uint16)
    wide[:, :q.shape[1]] = q
    full, _ = orc.window_attention(q, k, v, 0.25)
    part, _ = orc.window_attention(wide, k, v, 0.25, rows=[8, 0, 3])
    np.testing.assert_array_equal(part, full[[8, 0, 3]])
