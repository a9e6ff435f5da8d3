"""Bounded pipeline waits that run out.

Every shared-memory pipeline wait of the GEMM kernels gives up after a bound
(about 2 s); the kernel then takes its early exit: it records a status word,
stops issuing work, waits for the copies and tensor-core products it has
already issued, frees its tensor memory and returns. The test hook
qad_debug_stall makes the producer of CTA 0 stop issuing copies part-way, so
that CTA's consumers wait for data nothing will deliver (no fault, no trap:
the wait simply never completes).

Checked for the skinny and the dense GEMM and the prefill attention: the call
returns within seconds, the status word reports the timed-out wait, and the
device is still usable: the same launch right after, with the hook off,
matches the oracle and reports no timeout. That second launch also allocates
tensor memory again, which it could not if the aborted CTA had kept its
columns.
"""
import time

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


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _stalled(q, kernel, at, run):
    """run() with CTA 0's producer stopping at step `at`; returns the seconds it took."""
    q.debug_stall(kernel, at)
    try:
        t0 = time.monotonic()
        run()
        torch.cuda.synchronize()
        return time.monotonic() - t0
    finally:
        q.debug_stall(kernel, -1)


def test_skinny_gemm_wait_timeout_then_recovers(q, orc):
    # 136 weight tiles x 4 blocks = 544 units: CTA 0 owns units 0, 1, 2 on a 148-SM part
    N, K, M = 17408, 1024, 4
    W = synth.q4k_matrix_np(SEED, 1300, N, K)
    X = synth.bf16_normal_np(SEED, 1301, (M, K))
    Wd, Xd = torch.from_numpy(W).cuda(), _bf16(X)
    Y = torch.zeros(M, N, device="cuda")
    q.device_status(reset=True)
    took = _stalled(q, 0, 1, lambda: q.q4k_gemm(Wd, N, K, Xd, M, Y))
    status = q.device_status(reset=True)
    assert status != 0, "a wait on a copy that was never issued did not time out"
    assert took < 30.0, f"the stalled GEMM took {took:.1f} s to return"
    # the device is usable: the same GEMM is correct and reports no timeout
    Y.zero_()
    q.q4k_gemm(Wd, N, K, Xd, M, Y)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    Yr, A = orc.gemm(4, W, N, K, X)
    ratio = np.abs(Y.cpu().double().numpy() - Yr) / (1e-3 * A + 1e-30)
    assert ratio.max() <= 1.0, f"max err / tol = {ratio.max():.3g}"


def test_dense_gemm_wait_timeout_then_recovers(q, orc):
    # 2 weight tiles x 2 activation tiles x 2 blocks = 8 units over 8 CTAs (stream-K):
    # CTA 0 owns the first block of tile 0, k-steps 0 .. 3
    N, K, M = 256, 512, 300
    W = synth.q4k_matrix_np(SEED, 1310, N, K)
    X = synth.bf16_normal_np(SEED, 1311, (M, K))
    Wd, Xd = torch.from_numpy(W).cuda(), _bf16(X)
    Y = torch.zeros(M, N, device="cuda")
    q.dense_status(reset=True)
    took = _stalled(q, 1, 2, lambda: q.q4k_gemm_dense(Wd, N, K, Xd, M, Y))
    status = q.dense_status(reset=True)
    assert status != 0, "a wait on a copy that was never issued did not time out"
    assert took < 30.0, f"the stalled GEMM took {took:.1f} s to return"
    Y.fill_(float("nan"))
    q.q4k_gemm_dense(Wd, N, K, Xd, M, Y)
    torch.cuda.synchronize()
    assert q.dense_status() == 0
    Yr, A = orc.gemm(4, W, N, K, X)
    ratio = np.abs(Y.cpu().double().numpy() - Yr) / (1e-3 * A + 1e-30)
    assert ratio.max() <= 1.0, f"max err / tol = {ratio.max():.3g}"


def test_prefill_attention_wait_timeout_then_recovers(q, orc):
    # 130 rows x 4 query heads per kv-head = 520 query vectors: 3 CTA pairs per kv-head;
    # CTA (0, 0) takes the last pair, whose keys end at 300 + 130: 7 tiles of 64 keys
    len_, C, n_qh, n_kvh = 300, 130, 16, 4
    cap = len_ + C + 3
    Q = synth.bf16_normal_np(SEED, 1320, (C, n_qh, 128))
    Kc = synth.bf16_normal_np(SEED, 1321, (n_kvh, cap, 128))
    Vc = synth.bf16_normal_np(SEED, 1322, (n_kvh, cap, 128))
    Qd, Kd, Vd = _bf16(Q), _bf16(Kc), _bf16(Vc)
    O = torch.zeros(C, n_qh, 128, dtype=torch.bfloat16, device="cuda")
    q.prefill_status(reset=True)
    took = _stalled(q, 2, 3, lambda: q.prefill_attn(Qd, Kd, Vd, len_, C, cap, n_qh, n_kvh, 128, O))
    status = q.prefill_status(reset=True)
    assert status != 0, "a wait on a tile that was never loaded did not time out"
    assert took < 30.0, f"the stalled attention took {took:.1f} s to return"
    O.zero_()
    q.prefill_attn(Qd, Kd, Vd, len_, C, cap, n_qh, n_kvh, 128, O)
    torch.cuda.synchronize()
    assert q.prefill_status() == 0
    O_ref, B = orc.decode_attn(Q, Kc[None], Vc[None], np.array([len_], np.int32), np.array([0, C], np.int32),
                               n_qh, n_kvh, 128, cap)
    o = orc.bf16_array_to_f64(O.cpu().view(torch.int16).numpy().view(np.uint16)).reshape(O_ref.shape)
    ratio = np.abs(o - O_ref) / (2e-3 * B + np.abs(O_ref) * 2.0 ** -9 + 1e-30)
    assert ratio.max() <= 1.0, f"max err / tol = {ratio.max():.3g}"
