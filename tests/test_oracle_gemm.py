"""Pins for the oracle's quantized GEMM (CPU only).

The shared weight pass computes Y = X W^T for all rows of the batch (OpenJet
page, section 只搬一次权重). The oracle is checked against:
* numpy's matmul over weights dequantised by the independent ``gguf`` library
  (brute force on small, non-square shapes, so a transposed operand fails);
* one-hot activations (y = the weight column, read through the library);
* a closed form for all-zero quants (y = -sum_j dmin*m_j*sum_{k in j} x_k);
* row invariance (row r of an M-row product equals the 1-row product, bitwise);
* additivity over disjoint activation supports;
* its own row-subset entry point.
"""
import numpy as np
import pytest

import synth
from conftest import SEED

gguf = pytest.importorskip("gguf")
from gguf import quants  # noqa: E402


def _lib_dequant(fmt, W, N, K):
    t = gguf.GGMLQuantizationType.Q4_K if fmt == 4 else gguf.GGMLQuantizationType.Q6_K
    bs = 144 if fmt == 4 else 210
    return quants.dequantize(np.ascontiguousarray(W).reshape(-1, bs), t).astype(np.float64).reshape(N, K)


def _bf16_f64(x):
    import oracle
    return oracle.bf16_array_to_f64(x)


@pytest.mark.parametrize("fmt,N,K,M", [(4, 37, 768, 3), (4, 256, 1024, 1), (6, 19, 512, 5), (4, 9, 256, 16)])
def test_gemm_against_library_matmul(orc, fmt, N, K, M):
    W = (synth.q4k_matrix_np if fmt == 4 else synth.q6k_matrix_np)(SEED, 3, N, K)
    X = synth.bf16_normal_np(SEED, 3, (M, K))
    Y, A = orc.gemm(fmt, W, N, K, X)
    wl = _lib_dequant(fmt, W, N, K)
    x = _bf16_f64(X)
    ref = x @ wl.T
    # the library's float32 dequantisation differs from the exact weights by a few ulps
    tol = 8 * 2.0 ** -23 * (np.abs(x) @ np.abs(wl).T) + 1e-12
    assert (np.abs(Y - ref) <= tol).all()
    assert np.allclose(A, np.abs(x) @ np.abs(wl).T, rtol=1e-5)


def test_gemm_one_hot_reads_weight_column(orc):
    N, K = 40, 512
    W = synth.q4k_matrix_np(SEED, 4, N, K)
    wl = _lib_dequant(4, W, N, K)
    for k in (0, 1, 31, 32, 100, 255, 256, 300, 511):
        X = np.zeros((1, K), np.uint16)
        X[0, k] = 0x3F80  # bf16 1.0
        Y, _ = orc.gemm(4, W, N, K, X)
        assert np.allclose(Y[0], wl[:, k], rtol=4 * 2.0 ** -23, atol=1e-9)


def test_gemm_zero_quants_closed_form(orc):
    """All q = 0: w = -dmin*m_j, so y = -sum_j dmin*m_j*S_j with S_j the sub-block sums of x."""
    g = np.random.default_rng(5)
    N, K = 6, 512
    W = np.zeros((N, K // 256 * 144), np.uint8)
    expect_terms = []
    for n in range(N):
        row = []
        for b in range(K // 256):
            sc = g.integers(0, 64, 8).astype(np.uint8)
            m = g.integers(0, 64, 8).astype(np.uint8)
            dmin = np.float16(abs(g.standard_normal()) * 0.01)
            blk = orc.q4k_encode(np.zeros(256, np.uint8), sc, m, 0x3C00, int(dmin.view(np.uint16)))
            W[n, b * 144:(b + 1) * 144] = blk
            row.append((float(dmin), m.astype(np.float64)))
        expect_terms.append(row)
    X = synth.bf16_normal_np(SEED, 5, (2, K))
    x = _bf16_f64(X)
    Y, _ = orc.gemm(4, W, N, K, X)
    for r in range(2):
        for n in range(N):
            s = 0.0
            for b, (dmin, m) in enumerate(expect_terms[n]):
                S = x[r, b * 256:(b + 1) * 256].reshape(8, 32).sum(1)
                s -= dmin * (m * S).sum()
            assert abs(Y[r, n] - s) <= 1e-12 * (1 + abs(s))


def test_gemm_row_invariance_bitwise(orc):
    N, K, M = 64, 1024, 12
    W = synth.q4k_matrix_np(SEED, 6, N, K)
    X = synth.bf16_normal_np(SEED, 6, (M, K))
    Y, _ = orc.gemm(4, W, N, K, X)
    for r in range(M):
        Yr, _ = orc.gemm(4, W, N, K, X[r:r + 1])
        assert np.array_equal(Yr[0], Y[r])


def test_gemm_additive_over_disjoint_supports(orc):
    N, K = 32, 768
    W = synth.q6k_matrix_np(SEED, 7, N, K)
    X = synth.bf16_normal_np(SEED, 7, (1, K))
    X1, X2 = X.copy(), X.copy()
    X1[0, ::2] = 0
    X2[0, 1::2] = 0
    Y, A = orc.gemm(6, W, N, K, X)
    Y1, _ = orc.gemm(6, W, N, K, X1)
    Y2, _ = orc.gemm(6, W, N, K, X2)
    assert np.allclose(Y, Y1 + Y2, rtol=0, atol=1e-12 * A.max())


def test_gemm_rows_subset_matches_full(orc):
    N, K, M = 50, 512, 4
    W = synth.q4k_matrix_np(SEED, 8, N, K)
    X = synth.bf16_normal_np(SEED, 8, (M, K))
    Y, A = orc.gemm(4, W, N, K, X)
    rows = [0, 7, 49, 13]
    Ys, As = orc.gemm_rows(4, W, K, rows, X)
    assert np.array_equal(Ys, Y[:, rows]) and np.array_equal(As, A[:, rows])
