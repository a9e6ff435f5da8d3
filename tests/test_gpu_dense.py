"""GPU parity of the prefill-chunk GEMM (tcgen05, fp16 operands) against the fp64 oracle.

The dense path rounds every dequantized weight to fp16: for Q4_K
w = fp16(d*sc)*q + fp16(-dmin*m) in one fused multiply-add, for Q6_K
fp16(d*sc)*(q-32). So per output
    |y - y_ref| <= 2^-10 * B + 1e-3 * A,
with A = sum_k |w x| (the decode GEMM's tolerance scale, covering the fp32
accumulation) and B = sum_k (|d sc q| + |dmin m|) |x| for Q4_K (B = A for
Q6_K). B is computed by the oracle itself on a copy of the weights whose
d is made positive and dmin negative, against |x|.
"""
import numpy as np
import pytest
import torch

import synth
from conftest import SEED

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import quantized_agent_decode_b200 as q
    from quantized_agent_decode_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return q


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _abs_terms_q4(W, N, K):
    """Q4_K bytes with d -> |d| and dmin -> -|dmin|: its product with |x| is B."""
    Wb = np.array(W, np.uint8, copy=True).reshape(N, K // 256, 144)
    hdr = Wb[:, :, 0:4].copy().view(np.uint16)  # d, dmin as fp16 bits
    hdr[..., 0] &= 0x7FFF
    hdr[..., 1] |= 0x8000
    Wb[:, :, 0:4] = hdr.view(np.uint8)
    return Wb.reshape(N, -1)


def _bound(orc, fmt, W, N, K, X, rows=None):
    Xa = X & np.uint16(0x7FFF)
    if fmt == 6:
        if rows is None:
            return orc.gemm(6, W, N, K, X)[1]
        return orc.gemm_rows(6, W, K, rows, X)[1]
    Wp = _abs_terms_q4(W, N, K)
    if rows is None:
        return orc.gemm(4, Wp, N, K, Xa)[0]
    return orc.gemm_rows(4, Wp, K, rows, Xa)[0]


def _check(Y, Yr, A, B):
    err = np.abs(Y - Yr)
    ratio = err / (2.0 ** -10 * B + 1e-3 * A + 1e-30)
    assert ratio.max() <= 1.0, f"max err / tol = {ratio.max():.3g}"


DENSE_CASES = [
    (4, 256, 512, 300),    # two activation tiles, ragged second one
    (4, 320, 768, 5),      # ragged weight tiles (2.5 x 128 rows), few rows
    (4, 128, 256, 256),    # exactly one tile, one block
    (4, 130, 1024, 1),     # a single activation row, 2 weight tiles (second has 2 rows)
    (4, 512, 2048, 513),   # 4 x 3 tiles, 8 blocks
    (6, 256, 512, 260),
    (6, 136, 4352, 17),    # the Q6_K block count is odd (17 blocks)
    (6, 384, 1024, 513),
]


@pytest.mark.parametrize("fmt,N,K,M", DENSE_CASES)
def test_dense_gemm_parity(q, orc, fmt, N, K, M):
    W = (synth.q4k_matrix_np if fmt == 4 else synth.q6k_matrix_np)(SEED, 500 + N, N, K)
    X = synth.bf16_normal_np(SEED, 500 + M, (M, K))
    Wd = torch.from_numpy(W).cuda()
    if fmt == 6:
        Wd = q.q6k_pack(Wd, N, K)
    Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    Y = torch.full((M, N), float("nan"), device="cuda")  # overwritten
    (q.q4k_gemm_dense if fmt == 4 else q.q6k_gemm_dense)(Wd, N, K, Xd, M, Y)
    torch.cuda.synchronize()
    assert q.dense_status() == 0
    Yr, A = orc.gemm(fmt, W, N, K, X)
    _check(Y.cpu().double().numpy(), Yr, A, _bound(orc, fmt, W, N, K, X))


def _full_size(q, orc, fmt, N, K, M, seed):
    g = synth.torch_gen(SEED, "cuda", seed)
    Wg = (synth.q4k_matrix_torch if fmt == 4 else synth.q6k_matrix_torch)(g, N, K, "cuda")
    Xd = synth.bf16_normal_torch(g, (M, K), "cuda")
    Wd = Wg if fmt == 4 else q.q6k_pack(Wg, N, K)
    Y = torch.full((M, N), float("nan"), device="cuda")
    (q.q4k_gemm_dense if fmt == 4 else q.q6k_gemm_dense)(Wd, N, K, Xd, M, Y)
    torch.cuda.synchronize()
    assert q.dense_status() == 0
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 129, N // 2, N - 129, N - 128, N - 1],
                                     rng.integers(0, N, 23)])).astype(np.int32)
    W = Wg.cpu().numpy()
    X = _bits(Xd)
    Yr, A = orc.gemm_rows(fmt, W, K, rows, X)
    _check(Y.cpu().double().numpy()[:, rows], Yr, A, _bound(orc, fmt, W, N, K, X, rows))
    assert np.isfinite(Y.cpu().numpy()).all()


def test_dense_gemm_prefill_chunk_gate_up(q, orc):
    """2048 prompt rows + 12 decode rows through the gate|up matrix (N=34816, K=5120),
    every output row checked on 32 sampled weight rows (tile edges included)."""
    _full_size(q, orc, 4, 34816, 5120, 2060, 71)


def test_dense_gemm_prefill_chunk_down(q, orc):
    """The same chunk through the Q6_K-like down projection (N=5120, K=17408)."""
    _full_size(q, orc, 6, 5120, 17408, 2060, 72)
