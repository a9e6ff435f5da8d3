"""GPU parity of the prefill-chunk GEMM (tcgen05, fp16 operands) against the fp64 oracle.

The dense path forms every weight in fp32 (w = d*sc*q - dmin*m for Q4_K by one
fused multiply-add of exact terms, d*sc*(q-32) exactly for Q6_K) and rounds it
to fp16 once, so each operand is within (2^-11 + 2^-24) |w| of its weight; the
activations enter exactly (bf16 -> fp16 under a per-row power-of-two scale) and
the products accumulate in fp32. The bound is the decode GEMM's, per output:
    |y - y_ref| <= 1e-3 * A,    A = sum_k |w x|.
Q6_K cases run with the synthetic scales (0..63) and with signed scales over
the whole int8 range, as real checkpoints carry them.
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


def _check(Y, Yr, A):
    err = np.abs(Y - Yr)
    ratio = err / (1e-3 * A + 1e-30)
    assert ratio.max() <= 1.0, f"max err / tol = {ratio.max():.3g}"


DENSE_CASES = [
    (4, 256, 512, 300, False),    # two activation tiles, ragged second one
    (4, 320, 768, 5, False),      # ragged weight tiles (2.5 x 128 rows), few rows
    (4, 128, 256, 256, False),    # exactly one tile, one block
    (4, 130, 1024, 1, False),     # a single activation row, 2 weight tiles (second has 2 rows)
    (4, 512, 2048, 513, False),   # 4 x 3 tiles, 8 blocks
    (6, 256, 512, 260, False),
    (6, 136, 4352, 17, False),    # the Q6_K block count is odd (17 blocks)
    (6, 384, 1024, 513, False),
    (6, 256, 1024, 300, True),    # signed int8 sub-block scales
    (6, 136, 4352, 17, True),
    # 32 tiles of 26 blocks on a 148-SM part: the schedule splits them over all CTAs
    # (stream-K, ~5.6 units per CTA, 3-5 CTAs per tile added into a zeroed output)
    (6, 2048, 6656, 300, True),
    (4, 2048, 6656, 300, False),
]


def _weights(fmt, seed, N, K, signed):
    if fmt == 4:
        return synth.q4k_matrix_np(SEED, seed, N, K)
    return synth.q6k_matrix_np(SEED, seed, N, K, signed=signed)


@pytest.mark.parametrize("fmt,N,K,M,signed", DENSE_CASES)
def test_dense_gemm_parity(q, orc, fmt, N, K, M, signed):
    W = _weights(fmt, 500 + N, N, K, signed)
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
    _check(Y.cpu().double().numpy(), Yr, A)


def _full_size(q, orc, fmt, N, K, M, seed, signed=False):
    g = synth.torch_gen(SEED, "cuda", seed)
    Wg = synth.q4k_matrix_torch(g, N, K, "cuda") if fmt == 4 else synth.q6k_matrix_torch(g, N, K, "cuda", signed)
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
    _check(Y.cpu().double().numpy()[:, rows], Yr, A)
    assert np.isfinite(Y.cpu().numpy()).all()


def test_dense_gemm_prefill_chunk_gate_up(q, orc):
    """2048 prompt rows + 12 decode rows through the gate|up matrix (N=34816, K=5120),
    every output row checked on 32 sampled weight rows (tile edges included)."""
    _full_size(q, orc, 4, 34816, 5120, 2060, 71)


def test_dense_gemm_prefill_chunk_down(q, orc):
    """The same chunk through the Q6_K-like down projection (N=5120, K=17408)."""
    _full_size(q, orc, 6, 5120, 17408, 2060, 72)


def test_dense_gemm_prefill_chunk_down_signed_scales(q, orc):
    """The down projection with signed int8 sub-block scales over the whole range."""
    _full_size(q, orc, 6, 5120, 17408, 2060, 73, signed=True)
