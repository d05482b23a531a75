"""Pins of the oracle's Four Over Six KV scale rule (no GPU).

The pages name the KV cache's adaptive scale choice "Four Over Six"
(tailorednewshub.com LongLive-2.0 article, section "Inferencia W4A4 NVFP4")
without a formula.  The reading the oracle implements: per 16-element block,
map the block maximum onto 6 (the standard rule) or onto 4, quantize with each,
keep the scale whose squared error against the exactly decoded values is
smaller, 6 on a tie.  These tests restate each step independently (numpy
binary32 and ml_dtypes for the recipe's roundings, exact rationals for the
errors) and check invariants the rule must satisfy.
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

F32 = np.float32


def _scale_onto(amax_b, s_t, top):
    if s_t == 0:
        return 0
    r = F32(amax_b) / (F32(top) * F32(s_t))
    return int(np.array(min(r, F32(448.0)), F32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8))


def _e4m3(b):
    return float(np.array(b, np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64))


def _e2m1(q):
    return float(np.array(q & 7, np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64))


def _codes(block, sb, s_t):
    if sb == 0:
        return np.zeros(16, np.uint8)
    d = F32(_e4m3(sb)) * F32(s_t)
    y = block.astype(F32) / d
    return np.clip(y, -6, 6).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


def _exact_sq_error(block, codes, sb, s_t):
    sbv, st = Fraction(_e4m3(sb)), Fraction(float(s_t))
    e = Fraction(0)
    for x, q in zip(block, codes):
        diff = Fraction(abs(float(x))) - Fraction(_e2m1(int(q))) * sbv * st
        e += diff * diff
    return e


def _independent_rule(block, s_t):
    amax_b = np.max(np.abs(block))
    s6, s4 = _scale_onto(amax_b, s_t, 6), _scale_onto(amax_b, s_t, 4)
    e6 = _exact_sq_error(block, _codes(block, s6, s_t), s6, s_t)
    e4 = _exact_sq_error(block, _codes(block, s4, s_t), s4, s_t)
    return (s4 if e4 < e6 else s6), s4, s6, e4, e6


def test_worked_block_maps_onto_four(orc):
    """s_t = 2^-3 and a block of E2M1 values with maximum 4: onto 6 the scale
    is E4M3(4 / 0.75) = 5.5 and the codes are inexact; onto 4 it is 8, so
    d = 1 and every value is coded exactly.  The rule takes 4."""
    s_t = 0.125
    block = np.array([4, 3, -2, 1.5, 1, 0.5, -4, 0, 2, -3, 1, 0.5, 1.5, -1, 3, 4], F32)
    b6 = orc.block_scale_rule(block, s_t, 0)
    b4 = orc.block_scale_rule(block, s_t, 1)
    assert _e4m3(b6) == 5.5 and _e4m3(b4) == 8.0
    assert _exact_sq_error(block, _codes(block, b4, s_t), b4, s_t) == 0
    assert _exact_sq_error(block, _codes(block, b6, s_t), b6, s_t) > 0


def test_block_at_the_tensor_max_keeps_six(orc):
    """amax_b = amax: onto 4 wants 2688/4 = 672 > 448, which saturates; the
    saturated scale decodes the maximum as 448 * 4 / 672 of itself, so the
    rule keeps 6 (scale 448)."""
    amax = 7.0
    s_t = F32(amax) / F32(2688.0)
    block = np.array([amax] + [1.0] * 15, F32)
    b = orc.block_scale_rule(block, s_t, 1)
    assert _e4m3(b) == 448.0


def test_rule_matches_independent_restatement(orc):
    rng = np.random.default_rng(3)
    mismatches, close = 0, 0
    for i in range(600):
        kind = i % 3
        if kind == 0:
            block = rng.normal(0, 1, 16)
        elif kind == 1:
            block = rng.normal(0, 1, 16) * np.where(rng.random(16) < 0.1, 20, 1)
        else:
            block = rng.uniform(-1, 1, 16) ** 3
        # bf16 values, as the KV cache holds
        block = torch.from_numpy(block.astype(F32)).to(torch.bfloat16).float().numpy()
        s_t = F32(rng.uniform(0.5, 3.0)) / F32(2688.0) * F32(np.max(np.abs(block)) / 2.0 + 1e-3)
        want, s4, s6, e4, e6 = _independent_rule(block, s_t)
        got = orc.block_scale_rule(block, s_t, 1)
        if e4 != e6 and abs(e4 - e6) <= Fraction(1, 10**9) * max(e4, e6):
            close += 1  # binary64 evaluation may round either way here
            assert got in (s4, s6)
            continue
        mismatches += got != want
    assert mismatches == 0
    assert close < 6


def test_kv_chunk_rule_never_increases_block_error(orc):
    """Four Over Six changes some block scales of a KV chunk, keeps s_t, and
    never makes a block's squared error larger than the standard rule's."""
    g = torch.Generator().manual_seed(8)
    tpf, heads, hd = 6, 3, 32
    kv = (torch.randn(2 * tpf, heads, hd, generator=g) *
          torch.tensor([0.5, 2.0, 4.0]).view(1, 3, 1)).to(torch.bfloat16)
    bits = kv.view(torch.int16).numpy().view(np.uint16).reshape(-1)
    c0, s0, t0 = orc.kv_quant_chunk(bits, 2, tpf, heads, hd, rule=0)
    c1, s1, t1 = orc.kv_quant_chunk(bits, 2, tpf, heads, hd, rule=1)
    np.testing.assert_array_equal(t0, t1)
    assert np.any(s0 != s1)
    x = kv.float().numpy().reshape(-1, 16)
    st = float(t0[0])
    q0 = np.stack([c0.reshape(-1) & 0xF, c0.reshape(-1) >> 4], -1).reshape(-1, 16)
    q1 = np.stack([c1.reshape(-1) & 0xF, c1.reshape(-1) >> 4], -1).reshape(-1, 16)
    for b in np.nonzero(s0.reshape(-1) != s1.reshape(-1))[0][:60]:
        e0 = _exact_sq_error(x[b], q0[b], int(s0.reshape(-1)[b]), st)
        e1 = _exact_sq_error(x[b], q1[b], int(s1.reshape(-1)[b]), st)
        assert e1 < e0
    # the codes under either rule are the plain recipe's codes for that block scale
    for b in range(0, x.shape[0], 7):
        np.testing.assert_array_equal(q1[b], _codes(x[b], int(s1.reshape(-1)[b]), st))


def test_exact_tie_keeps_six(orc):
    """A block coded without error by both scales: with s_t = 1/16 and maximum
    0.75, onto 6 gives s_b = 2 (grid {0, .5, 1, 1.5, 2, 3, 4, 6} / 8) and onto 4
    gives s_b = 3 (grid {0, .75, 1.5, 2.25, 3, 4.5, 6, 9} / 16); the values
    0.75, 0.375 and 0.1875 lie on both, so both squared errors are exactly 0
    and the rule keeps 6."""
    block = np.zeros(16, np.float32)
    block[[0, 3, 7, 12]] = [0.75, 0.375, -0.1875, 0.375]
    s_t = 1.0 / 16
    six = orc.block_scale_rule(block, s_t, 0)
    assert orc.e4m3_value(six) == 2.0
    assert orc.block_scale_rule(block, s_t, 1) == six
    # the onto-4 scale really is different and exact too
    s4 = int(np.array(0.75 / (4 * s_t), np.float32).astype(ml_dtypes.float8_e4m3fn)
             .view(np.uint8))
    assert orc.e4m3_value(s4) == 3.0
    for x in block:
        for s in (2.0, 3.0):
            q = abs(float(x)) / (s * s_t)
            assert q in (0, 0.5, 1, 1.5, 2, 3, 4, 6)
