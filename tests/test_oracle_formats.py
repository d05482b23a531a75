"""Pins of the oracle's format primitives against independent libraries and
the format definitions (no GPU).

E2M1 and E4M3 are checked against ml_dtypes / torch's float8 and float4
conversions, which implement the OCP microscaling formats independently of
this repository; bfloat16 rounding against torch.  The E2M1 layout itself
(2 exponent bits, 1 mantissa bit) is the one the neurohive.io LongLive-2.0
article states in its NVFP4 paragraph (tests/golden/page_facts.json).
"""
import json
import os

import ml_dtypes
import numpy as np
import pytest
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def test_e2m1_layout_matches_pages(orc):
    facts = json.load(open(GOLD))
    fmt = facts["element_format"]["value"]
    assert fmt["exponent_bits"] + fmt["mantissa_bits"] + 1 == 4
    # 2^(exponent_bits) binades x 2^(mantissa_bits) steps = 8 magnitudes
    mags = sorted({abs(orc.e2m1_value(c)) for c in range(16)})
    assert len(mags) == 2 ** fmt["exponent_bits"] * 2 ** fmt["mantissa_bits"]


def test_e2m1_decode_all_codes(orc):
    ref = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    got = np.array([orc.e2m1_value(c) for c in range(16)])
    np.testing.assert_array_equal(got, ref)
    # sign of the two zeros
    assert np.signbit(got[8]) and not np.signbit(got[0])


def test_e4m3_decode_all_bytes(orc):
    ref_t = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = ref_t.to(torch.float64).numpy()
    ref2 = np.arange(256, dtype=np.uint16).astype(np.uint8).view(ml_dtypes.float8_e4m3fn)
    ref2 = ref2.astype(np.float64)
    got = np.array([orc.e4m3_value(b) for b in range(256)])
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    np.testing.assert_array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    np.testing.assert_array_equal(got[~nan], ref2[~nan])
    # format landmarks: largest finite 448, smallest subnormal 2^-9, smallest normal 2^-6
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6
    # non-negative finite values strictly increase with the code
    assert np.all(np.diff(got[:0x7F]) > 0)


def _e4m3_grid():
    vals = np.array([np.float64(np.arange(256, dtype=np.uint16).astype(np.uint8)
                                .view(ml_dtypes.float8_e4m3fn).astype(np.float64)[c])
                     for c in range(0x7F)])
    mids = (vals[:-1] + vals[1:]) / 2  # exact ties (representable in float32)
    pts = [vals, mids]
    f = mids.astype(np.float32)
    pts.append(np.nextafter(f, np.float32(np.inf)).astype(np.float64))
    pts.append(np.nextafter(f, np.float32(0)).astype(np.float64))
    rng = np.random.default_rng(7)
    pts.append(np.exp2(rng.uniform(-12, 9, 4000)))
    return np.concatenate(pts).astype(np.float32)


def test_e4m3_encode_matches_library(orc):
    r = _e4m3_grid()
    r = r[r <= 448.0]
    ref = r.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    got = np.array([orc.e4m3_encode(v) for v in r], dtype=np.uint8)
    np.testing.assert_array_equal(got, ref)


def test_e4m3_encode_ties_and_saturation(orc):
    # tie between 0 and the smallest subnormal 2^-9 goes to the even code 0
    assert orc.e4m3_encode(2.0 ** -10) == 0x00
    assert orc.e4m3_encode(np.nextafter(np.float32(2.0 ** -10), np.float32(1))) == 0x01
    # 448 is the largest finite value; anything above saturates to it
    for v in (448.0, 449.0, 464.0, 480.0, 1e6, 3e38):
        assert orc.e4m3_encode(v) == 0x7E
    # tie 1.0625 between 1.0 (0x38, even) and 1.125 (0x39): to 0x38
    assert orc.e4m3_encode(1.0625) == 0x38
    # tie 1.1875 between 1.125 (0x39) and 1.25 (0x3A, even): to 0x3A
    assert orc.e4m3_encode(1.1875) == 0x3A


def test_e2m1_encode_matches_library(orc):
    mags = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    ties = np.array([.25, .75, 1.25, 1.75, 2.5, 3.5, 5], np.float32)
    pts = [mags, ties, np.nextafter(ties, np.float32(9)), np.nextafter(ties, np.float32(0)),
           np.array([6.5, 7, 100, 3e38], np.float32)]
    rng = np.random.default_rng(3)
    pts.append(rng.uniform(0, 7, 5000).astype(np.float32))
    y = np.concatenate(pts)
    y = np.concatenate([y, -y])
    ref = y.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    got = np.array([orc.e2m1_encode(v) for v in y], dtype=np.uint8)
    np.testing.assert_array_equal(got, ref)


def test_e2m1_encode_tie_table(orc):
    # round half to even code: the expected codes follow from the code parity
    expect = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for y, c in expect.items():
        assert orc.e2m1_encode(y) == c
        assert orc.e2m1_encode(-y) == c | 8
    assert orc.e2m1_encode(-0.0) == 8 and orc.e2m1_encode(0.0) == 0
    assert orc.e2m1_encode(-0.1) == 8  # negative values that round to zero keep the sign


def test_bf16_rounding_matches_torch(orc):
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        np.exp2(rng.uniform(-130, 127, 20000)).astype(np.float32),
    ])
    # exact ties: bf16 value + half an ulp
    base = rng.standard_normal(5000).astype(np.float32)
    bb = (base.view(np.uint32) & 0xFFFF0000) | 0x8000
    x = np.concatenate([x, bb.view(np.float32), -x])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.bf16_from_f32(v) for v in x], dtype=np.uint16)
    np.testing.assert_array_equal(got, ref)


def test_sf_mma_layout_is_a_permutation(orc):
    # within one 128 x 4 tile the 512 (row, block) pairs fill offsets 0..511
    offs = sorted(orc.sf_mma_offset(r, c, 4) for r in range(128) for c in range(4))
    assert offs == list(range(512))
    # landmarks of the 32 x 16-byte arrangement
    assert orc.sf_mma_offset(1, 0, 4) == 16
    assert orc.sf_mma_offset(32, 0, 4) == 4
    assert orc.sf_mma_offset(127, 3, 4) == 31 * 16 + 3 * 4 + 3
    # tiles: row-tile major, then block-tile (nkb = 12 -> 3 block tiles)
    assert orc.sf_mma_offset(0, 4, 12) == 512
    assert orc.sf_mma_offset(128, 0, 12) == 3 * 512
    # padded sizes
    assert orc.sf_mma_bytes(2640, 3072) == 2688 * 192
    assert orc.sf_mma_bytes(1, 16) == 128 * 4
