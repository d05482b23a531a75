"""The window attention's parity bound, checked on the CPU against a model of
the kernel's arithmetic (no GPU).

The model follows the kernel step by step in binary32: scores as fp32 sums of
bf16 products, scaled to base 2, a running row max and sum over 64-token tiles
(online softmax with exp2), probabilities rounded to bf16 before P V, fp32
accumulation, the output normalised and rounded to bf16.  Against the oracle's
binary64 attention it must stay inside the bound the GPU test uses,
|o - o_ref| <= 2^-6 E + 2^-8 |o_ref| with E = sum_j p_j |v_j|, and it should use
a visible part of it (the bound is not vacuous)."""
import numpy as np
import torch

TILE = 64


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16) \
        .to(torch.float32).numpy()


def _bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _model(q, k, v, scale):
    """q [tq, d], k, v [n_kv, d] (bf16-valued float32) -> bf16-valued output."""
    f32 = np.float32
    scale_log2 = f32(scale * np.log2(np.e))
    tq, d = q.shape
    m = np.full(tq, -np.inf, f32)
    l = np.zeros(tq, f32)
    o = np.zeros((tq, d), f32)
    for t0 in range(0, k.shape[0], TILE):
        kt, vt = k[t0:t0 + TILE], v[t0:t0 + TILE]
        s = (q @ kt.T).astype(f32) * scale_log2
        mn = np.maximum(m, s.max(axis=1))
        corr = np.exp2(m - mn).astype(f32)
        p = np.exp2(s - mn[:, None]).astype(f32)
        l = l * corr + p.sum(axis=1, dtype=f32)
        o = o * corr[:, None] + (_bf16(p) @ vt).astype(f32)
        m = mn
    return _bf16(o / l[:, None])


def test_bound_holds_with_margin(orc):
    rng = np.random.default_rng(5)
    heads, d, tq, n_kv = 3, 128, 48, 10 * TILE + 37
    sigma = rng.uniform(0.5, 4.0, heads)
    q = _bf16(rng.standard_normal((tq, heads, d)))
    k = _bf16(rng.standard_normal((n_kv, heads, d)) * sigma[None, :, None])
    v = _bf16(rng.standard_normal((n_kv, heads, d)) * sigma[None, :, None])
    scale = d ** -0.5
    ref, E = orc.window_attention(_bits(q.reshape(tq, heads * d)), _bits(k), _bits(v), scale)
    worst = 0.0
    for h in range(heads):
        out = _model(q[:, h], k[:, h], v[:, h], scale)
        tol = 2.0 ** -6 * E[:, h] + 2.0 ** -8 * np.abs(ref[:, h])
        ratio = np.abs(out - ref[:, h]) / tol
        assert np.all(ratio <= 1.0)
        worst = max(worst, float(ratio.max()))
    assert worst > 1.0 / 64  # the bound is of the error's size, not far above it
