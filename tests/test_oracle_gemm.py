"""Pins of the oracle's FP64 GEMM reference (no GPU).

The reference is y[m,n] = sum_k a[m,k] w[n,k] over the exactly dequantized
NVFP4 operands (tailorednewshub.com LongLive-2.0 article, section 'Inferencia
W4A4 NVFP4': BF16 GEMMs become FP4 GEMMs).  It is checked against numpy's
matmul of the same exact operands, against closed forms built from
representable codes, and for sensitivity to a transposed operand.
"""
import ml_dtypes
import numpy as np
import pytest

F32 = np.float32


def _q(orc, x):
    return orc.quantize(np.ascontiguousarray(x, F32))


@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (5, 7, 64), (33, 20, 128), (3, 130, 48)])
def test_gemm_matches_numpy(orc, M, N, K):
    rng = np.random.default_rng(M * 1000 + N * 10 + K)
    a = _q(orc, rng.standard_normal((M, K)) * 2)
    w = _q(orc, rng.standard_normal((N, K)) * 0.02)
    y, S = orc.gemm(a, w)
    A = orc.dequantize_exact(*a)
    W = orc.dequantize_exact(*w)
    np.testing.assert_allclose(y, A @ W.T, rtol=0, atol=1e-12 * (np.abs(A) @ np.abs(W).T).max())
    np.testing.assert_allclose(S, np.abs(A) @ np.abs(W).T, rtol=1e-14)
    # row sampling returns the same rows
    rows = [M - 1, 0]
    y2, S2 = orc.gemm(a, w, rows=rows)
    np.testing.assert_array_equal(y2, y[rows])
    np.testing.assert_array_equal(S2, S[rows])


def test_gemm_closed_forms(orc):
    K = 64
    # all-ones operands: codes of 1.0 (code 2) with block scale 1 and s_t = 1
    ones_codes = np.full((4, K // 2), 0x22, np.uint8)
    sf_one = np.full((4, K // 16), 0x38, np.uint8)  # E4M3 1.0
    y, S = orc.gemm((ones_codes, sf_one, 1.0), (ones_codes[:3], sf_one[:3], 1.0))
    assert np.all(y == K) and np.all(S == K)
    # scales multiply through: s_tA * s_tW * K * s_bA * s_bW
    sfa = np.full((4, K // 16), 0x40, np.uint8)  # 2.0
    sfw = np.full((3, K // 16), 0x30, np.uint8)  # 0.5
    y, _ = orc.gemm((ones_codes, sfa, 0.25), (ones_codes[:3], sfw, 8.0))
    assert np.all(y == K * 2.0 * 0.5 * 0.25 * 8.0)
    # identity-like W: row n has a single 1.0 at column n -> y = A[:, :N]
    N = 16
    wc = np.zeros((N, K // 2), np.uint8)
    for n in range(N):
        wc[n, n // 2] = 0x2 << (4 * (n % 2))
    wsf = np.full((N, K // 16), 0x38, np.uint8)
    rng = np.random.default_rng(0)
    a = _q(orc, rng.standard_normal((6, K)))
    y, _ = orc.gemm(a, (wc, wsf, 1.0))
    np.testing.assert_array_equal(y, orc.dequantize_exact(*a)[:, :N])
    # a single negative code flips the sign of exactly one term
    wc2 = wc.copy()
    wc2[3, 1] = 0xA << 4  # column 3 -> -1.0
    y2, _ = orc.gemm(a, (wc2, wsf, 1.0))
    np.testing.assert_array_equal(y2[:, 3], -y[:, 3])


def test_gemm_detects_transposed_operand(orc):
    rng = np.random.default_rng(4)
    K = 32
    a = _q(orc, rng.standard_normal((K, K)))
    w = _q(orc, rng.standard_normal((K, K)))
    y, _ = orc.gemm(a, w)
    A = orc.dequantize_exact(*a)
    W = orc.dequantize_exact(*w)
    assert np.allclose(y, A @ W.T)
    assert not np.allclose(y, A @ W)


def test_gemm_scale_layout_conversion(orc):
    """The tensor-core scale layout is a pure permutation of the row-major
    scales: reading every (row, block) back through the offset function
    recovers them, and padding bytes are zero."""
    rng = np.random.default_rng(2)
    rows, cols = 200, 192
    sf = rng.integers(1, 0x7F, size=(rows, cols // 16)).astype(np.uint8)
    tiled = orc.sf_to_mma(sf, rows, cols)
    back = np.array([[tiled[orc.sf_mma_offset(r, k, cols // 16)] for k in range(cols // 16)]
                     for r in range(rows)], np.uint8)
    np.testing.assert_array_equal(back, sf)
    assert int(tiled.astype(np.int64).sum()) == int(sf.astype(np.int64).sum())
