"""The allocation-free GEMM entry point (qad_q4k_gemm_noalloc) for callers that
cannot allocate device memory at call time: servers that reserve all of HBM
up front, code that must avoid cudaFree's device-wide synchronisation, plain C
integrations holding only caller-owned buffers. Its scratch is the library's
fixed device array instead of a caller workspace.

Checked through the C ABI on two calls in a row (different shapes, so the
second call runs on the first call's leftover scratch) against both the fp64
oracle and the workspace entry point qad_q4k_gemm, within the GEMM tolerance
used everywhere else: |y - y_ref| <= 1e-3 * sum_k |w x| per output; the
accumulate form is checked on a pre-filled Y, and a warm call must leave the
device's free memory unchanged. This file is collected last so a failure here
leaves every other test already run.
"""
import ctypes as C

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


def _call_noalloc(q, W, N, K, X, M, Y, accumulate=0):
    L = q.lib()
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.qad_q4k_gemm_noalloc(C.c_void_p(W.data_ptr()), N, K, C.c_void_p(X.data_ptr()), M,
                                  C.c_void_p(Y.data_ptr()), accumulate, s)


def test_noalloc_gemm_matches_workspace_entry_point_twice(q, orc):
    cases = [(4096, 5120, 12), (300, 17408, 5)]
    for i, (N, K, M) in enumerate(cases):
        W = synth.q4k_matrix_np(SEED, 900 + i, N, K)
        X = synth.bf16_normal_np(SEED, 900 + i, (M, K))
        Wd = torch.from_numpy(W).cuda()
        Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
        Y_ref = torch.zeros(M, N, device="cuda")
        q.q4k_gemm(Wd, N, K, Xd, M, Y_ref)
        Y = torch.full((M, N), float("nan"), device="cuda")  # overwritten, not accumulated
        rc = _call_noalloc(q, Wd, N, K, Xd, M, Y)
        assert rc == 0, q.lib().qad_last_error()
        torch.cuda.synchronize()
        Yr, A = orc.gemm(4, W, N, K, X)
        got = Y.cpu().double().numpy()
        assert (np.abs(got - Yr) <= 1e-3 * A).all(), (np.abs(got - Yr) / (1e-3 * A)).max()
        diff = np.abs(got - Y_ref.cpu().double().numpy())
        assert (diff <= 2e-3 * A).all(), (diff / (2e-3 * A)).max()
    assert q.device_status() == 0


def test_noalloc_gemm_accumulates_and_allocates_nothing(q, orc):
    """accumulate=1 adds W x to a pre-filled Y; a warm call changes no device memory."""
    N, K, M = 520, 3072, 9
    W = synth.q4k_matrix_np(SEED, 910, N, K)
    X = synth.bf16_normal_np(SEED, 911, (M, K))
    Wd = torch.from_numpy(W).cuda()
    Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    Y0 = torch.randn(M, N, device="cuda")
    Y = Y0.clone()
    assert _call_noalloc(q, Wd, N, K, Xd, M, Y) == 0  # warm-up (overwrite form)
    torch.cuda.synchronize()
    Y.copy_(Y0)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    assert _call_noalloc(q, Wd, N, K, Xd, M, Y, accumulate=1) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"
    Yr, A = orc.gemm(4, W, N, K, X)
    base = Y0.cpu().double().numpy()
    err = np.abs(Y.cpu().double().numpy() - (base + Yr))
    assert (err <= 1e-3 * A + 4 * 2.0 ** -24 * np.abs(base)).all()
    assert q.device_status() == 0


def test_noalloc_gemm_rejects_oversized_scratch(q):
    L = q.lib()
    limit = L.qad_q4k_gemm_noalloc_scratch_bytes()
    assert limit == 1 << 20
    K = 30720  # one block past the 30464 the fixed array holds, whatever the row count
    W = torch.zeros(1, K // 256 * 144, dtype=torch.uint8, device="cuda")
    X = torch.zeros(16, K, dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros(16, 1, device="cuda")
    for M in (1, 16):
        assert q.gemm_ws_bytes(K, M) > limit >= q.gemm_ws_bytes(30464, M)
        rc = _call_noalloc(q, W, 1, K, X, M, Y)
        assert rc == -2 and b"scratch" in L.qad_last_error()
