"""GPU parity of the prefill-chunk causal attention against the fp64 oracle.

Row j of the chunk (position len + j) attends keys 0 .. len + j: the oracle's
decode attention with one agent whose rows are the whole chunk. The GPU path
forms S = Q K^T from exact bf16 products, rounds each probability once to fp16
(relative error <= 2^-11) and converts V to fp16 exactly, so per element the
decode attention's bound holds:
    |o - o_ref| <= 2e-3 * B + half a bf16 ulp of o_ref (2^-9 |o_ref|),
with B = sum_t p_t |v_t| from the oracle.
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


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _check(orc, o_bits, O_ref, B):
    o = orc.bf16_array_to_f64(o_bits).reshape(O_ref.shape)
    tol = 2e-3 * B + np.abs(O_ref) * 2.0 ** -9 + 1e-30
    ratio = np.abs(o - O_ref) / tol
    assert ratio.max() <= 1.0, f"max err / tol = {ratio.max():.3g}"


CASES = [  # (len, C, n_qh, n_kvh)
    (37, 100, 48, 8),    # ragged chunk, GQA 6:1 as in the stack
    (0, 130, 8, 2),      # empty prior cache (first chunk of a prompt)
    (513, 64, 6, 1),     # one kv-head
    (5, 1, 48, 8),       # a single row (the decode case)
    (100, 300, 12, 4),   # several key tiles before the diagonal
    (70, 257, 16, 16),   # no grouping, query tiles ending mid-row
]


@pytest.mark.parametrize("len_,C,n_qh,n_kvh", CASES)
def test_prefill_attn_parity(q, orc, len_, C, n_qh, n_kvh):
    """Cache slots past the chunk hold NaN: a kernel must neither read them into
    a visible product nor let them leak through a zero probability."""
    cap = len_ + C + 131
    Q = synth.bf16_normal_np(SEED, 700 + C, (C, n_qh, 128))
    Kc = synth.bf16_normal_np(SEED, 701 + C, (n_kvh, cap, 128))
    Vc = synth.bf16_normal_np(SEED, 702 + C, (n_kvh, cap, 128))
    Kc[:, len_ + C:] = 0x7FC0
    Vc[:, len_ + C:] = 0x7FC0
    O = torch.zeros(C, n_qh, 128, dtype=torch.bfloat16, device="cuda")
    q.prefill_attn(_dev(Q), _dev(Kc), _dev(Vc), len_, C, cap, n_qh, n_kvh, 128, O)
    torch.cuda.synchronize()
    assert q.prefill_status() == 0
    O_ref, B = orc.decode_attn(Q, Kc[None], Vc[None], np.array([len_], np.int32), np.array([0, C], np.int32),
                               n_qh, n_kvh, 128, cap)
    _check(orc, _bits(O), O_ref, B)


def _scaled(bits, f):
    """bf16 bits of f times the values (N(0,1) draws scaled to large magnitudes)."""
    import oracle as o
    return o.f64_array_to_bf16(o.bf16_array_to_f64(bits) * f)


@pytest.mark.parametrize("len_,C,scale", [(300, 200, 1.5e4), (0, 130, 3e3), (1000, 64, 5e2)])
def test_prefill_attn_large_scores(q, orc, len_, C, scale):
    """q, k, v of order 1e3..1e4 (as a deep synthetic stack produces): scaled
    scores reach ~1e9 in the log2 domain, where fp32 spacing is ~100; the
    softmax must stay finite and equal to the oracle's (close to a hard max)."""
    n_qh, n_kvh = 16, 4
    cap = len_ + C + 3
    Q = _scaled(synth.bf16_normal_np(SEED, 720 + C, (C, n_qh, 128)), scale)
    Kc = _scaled(synth.bf16_normal_np(SEED, 721 + C, (n_kvh, cap, 128)), scale)
    Vc = _scaled(synth.bf16_normal_np(SEED, 722 + C, (n_kvh, cap, 128)), min(scale, 1e4))
    O = torch.zeros(C, n_qh, 128, dtype=torch.bfloat16, device="cuda")
    q.prefill_attn(_dev(Q), _dev(Kc), _dev(Vc), len_, C, cap, n_qh, n_kvh, 128, O)
    torch.cuda.synchronize()
    assert q.prefill_status() == 0
    o = _bits(O)
    assert np.isfinite(orc.bf16_array_to_f64(o)).all()
    O_ref, B = orc.decode_attn(Q, Kc[None], Vc[None], np.array([len_], np.int32), np.array([0, C], np.int32),
                               n_qh, n_kvh, 128, cap)
    _check(orc, o, O_ref, B)


def test_prefill_attn_chunk_after_23k_tokens(q, orc):
    """A 2048-row chunk after 23000 cached tokens (48/8 heads), sampled rows against the
    oracle row by row (row j is a one-row agent with len + j cached tokens)."""
    len_, C, n_qh, n_kvh = 23000, 2048, 48, 8
    cap = len_ + C
    g = synth.torch_gen(SEED, "cuda", 90)
    Qd = synth.bf16_normal_torch(g, (C, n_qh, 128), "cuda")
    Kd = synth.bf16_normal_torch(g, (n_kvh, cap, 128), "cuda")
    Vd = synth.bf16_normal_torch(g, (n_kvh, cap, 128), "cuda")
    O = torch.zeros(C, n_qh, 128, dtype=torch.bfloat16, device="cuda")
    q.prefill_attn(Qd, Kd, Vd, len_, C, cap, n_qh, n_kvh, 128, O)
    torch.cuda.synchronize()
    assert q.prefill_status() == 0
    Q, Kc, Vc, Ob = _bits(Qd), _bits(Kd), _bits(Vd), _bits(O)
    for j in (0, 1, 63, 64, 1023, 2046, 2047):
        O_ref, B = orc.decode_attn(Q[j:j + 1], Kc[None], Vc[None], np.array([len_ + j], np.int32),
                                   np.array([0, 1], np.int32), n_qh, n_kvh, 128, cap)
        _check(orc, Ob[j:j + 1], O_ref, B)
