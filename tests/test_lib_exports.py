"""The C-ABI library builds for sm_100a, loads without a GPU and exports every
symbol include/qad.h declares; host-only entry points run here (CPU only)."""
import ctypes as C
import os
import re

import numpy as np
import pytest
import torch

import synth
from conftest import ROOT, SEED, golden


@pytest.fixture(scope="module")
def qlib():
    from quantized_agent_decode_b200 import build
    build.build()
    import quantized_agent_decode_b200 as q
    return q


def _declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(inc, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(qad_[a-z0-9_]+)\s*\(", text):
            names.add(m.group(1))
    return names


def test_header_declares_the_boundary():
    names = _declared_functions()
    for need in ("qad_q4k_gemm", "qad_q6k_gemm", "qad_decode_attn", "qad_decode_step", "qad_pack_rows",
                 "qad_q4k_unpack", "qad_model_create", "qad_decode_step_host"):
        assert need in names


def test_every_declared_symbol_is_exported(qlib):
    L = C.CDLL(qlib.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(L, n)]
    assert not missing, missing
    # and the binding declares a signature for each of them
    assert not (_declared_functions() - set(qlib.SIGNATURES)), _declared_functions() - set(qlib.SIGNATURES)


def test_build_targets_sm100a_only():
    from quantized_agent_decode_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def _prototype_arg_counts():
    """Number of parameters of every qad_* prototype in include/*.h."""
    counts = {}
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if not fn.endswith(".h"):
            continue
        text = re.sub(r"/\*.*?\*/", "", open(os.path.join(inc, fn)).read(), flags=re.S)
        for m in re.finditer(r"\b(qad_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text):
            args = m.group(2).strip()
            counts[m.group(1)] = 0 if args in ("", "void") else args.count(",") + 1
    return counts


def test_binding_signatures_match_header(qlib):
    """Every ctypes signature in the binding has as many parameters as its C prototype."""
    counts = _prototype_arg_counts()
    for name, (_, argtypes) in qlib.SIGNATURES.items():
        assert name in counts, name
        assert len(argtypes) == counts[name], (name, len(argtypes), counts[name])


def test_version_and_error_text(qlib):
    L = qlib.lib()
    assert L.qad_version() >= 100
    # a host-side argument check fails without touching the GPU
    rc = L.qad_q4k_gemm(None, 1, 256, None, 1, None, 0, None, 0, None)
    assert rc == -1 and b"qad_q4k_gemm" in L.qad_last_error()
    assert L.qad_gemm_ws_bytes(255, 1) == 0 and L.qad_gemm_ws_bytes(256, 17) == 0
    assert L.qad_gemm_ws_bytes(5120, 12) > 0


def test_dense_gemm_argument_checks(qlib):
    """The prefill-chunk GEMM validates its arguments on the host before any launch."""
    L = qlib.lib()
    fake = C.c_void_p(0x10000)  # aligned, never dereferenced: every call below fails its checks first
    assert L.qad_q4k_gemm_dense(None, 128, 256, fake, 4, fake, fake, 1 << 20, None) == -1
    assert L.qad_q4k_gemm_dense(fake, 128, 300, fake, 4, fake, fake, 1 << 20, None) == -2
    assert b"K % 256" in L.qad_last_error()
    assert L.qad_q6k_gemm_dense(fake, 128, 256, C.c_void_p(0x10008), 4, fake, fake, 1 << 20, None) == -1
    need = L.qad_dense_gemm_ws_bytes(512, 300)
    assert need == 512 * 512 * 2 + 512 * 4  # M padded to two 256-row tiles, plus the row scales
    assert L.qad_q4k_gemm_dense(fake, 128, 512, fake, 300, fake, fake, need - 1, None) == -3
    assert L.qad_dense_gemm_ws_bytes(100, 4) == 0 and L.qad_dense_gemm_ws_bytes(256, 0) == 0


def test_pack_rows_matches_oracle(qlib, orc):
    gd = golden("pack_rows.json")
    H = 64
    rows_np = [synth.bf16_normal_np(SEED, 60 + a, (n, H)) for a, n in enumerate(gd["n_rows"])]
    rows_t = [torch.from_numpy(r.view(np.int16)).view(torch.bfloat16) for r in rows_np]
    X, ra, rp, ars = qlib.pack_rows(rows_t, gd["lens"], H)
    oX, ora, orp, oars = orc.pack_rows(rows_np, gd["lens"], H)
    assert np.array_equal(X.view(torch.int16).numpy().view(np.uint16), oX)
    assert ra.tolist() == ora.tolist() == gd["row_agent"]
    assert rp.tolist() == orp.tolist() == gd["row_pos"]
    assert ars.tolist() == oars.tolist() == gd["agent_row_start"]


def test_pack_rows_rejects_overflow_and_negative(qlib):
    H = 8
    rows = [torch.zeros(9, H, dtype=torch.bfloat16), torch.zeros(9, H, dtype=torch.bfloat16)]
    with pytest.raises(qlib.QadError):
        qlib.pack_rows(rows, [0, 0], H, max_rows=16)
    with pytest.raises(qlib.QadError):
        qlib.pack_rows([torch.zeros(1, H, dtype=torch.bfloat16)], [-1], H)
    X, ra, rp, ars = qlib.pack_rows([torch.zeros(0, H, dtype=torch.bfloat16)] * 3, [1, 2, 3], H)
    assert X.shape[0] == 0 and ars.tolist() == [0, 0, 0, 0]


def test_compute_calls_fail_loudly_without_gpu(qlib):
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(qlib.QadError):
        qlib.q4k_gemm(torch.zeros(1, 144, dtype=torch.uint8), 1, 256, torch.zeros(1, 256, dtype=torch.bfloat16),
                      1, torch.zeros(1, 1))


def test_q8_and_mixed_argument_checks_and_cache_sizes(qlib):
    """Host-side checks of the q8_0 and mixed-step entry points (no launch reached),
    and the cache sizes they expect."""
    L = qlib.lib()
    fake = C.c_void_p(0x10000)  # aligned, never dereferenced: every call below fails its checks first
    assert L.qad_q8_0_quantize(fake, 0, 48, fake, fake, None) == -2          # n % 32
    assert L.qad_q8_0_quantize(None, 0, 64, fake, fake, None) == -1
    assert L.qad_q8_0_quantize(C.c_void_p(0x10004), 0, 64, fake, fake, None) == -1  # x not 16-byte aligned
    args = [fake] * 7 + [4, 3, 100, 48, 8]
    assert L.qad_decode_attn_q8(*args, 64, 0.1, fake, fake, 1 << 20, None) == -2  # hd != 128
    assert L.qad_decode_attn_q8(*args, 128, 0.1, fake, fake, 16, None) == -3     # workspace
    assert L.qad_mixed_step(None, fake, 2, fake, 1, 2, fake, 0, 0, 8, fake, fake, 1 << 20, None) == -1
    # bf16: 2 bytes per value; q8_0: 1 byte per value, then fp16 scales per 32 at a 256-byte boundary
    A, kvh, cap = 4, 8, 1027
    assert qlib.kv_cache_bytes(qlib.KV_BF16, A, kvh, cap) == A * kvh * cap * 128 * 2
    codes = A * kvh * cap * 128
    assert qlib.kv_cache_bytes(qlib.KV_Q8_0, A, kvh, cap) == (codes + 255) // 256 * 256 + A * kvh * cap * 4 * 2
    assert qlib.kv_cache_bytes(7, A, kvh, cap) == 0 and qlib.kv_cache_bytes(qlib.KV_Q8_0, A, kvh, cap, hd=64) == 0


def test_debug_stall_rejects_unknown_kernel(qlib):
    """The wait-timeout test hook validates its kernel index before any CUDA call."""
    with pytest.raises(qlib.QadError):
        qlib.debug_stall(7, 0)
    with pytest.raises(qlib.QadError):
        qlib.debug_stall(-1, 0)
