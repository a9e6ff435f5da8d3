"""GPU parity of the q8_0 KV-cache path through the C ABI: the quantiser
(bit-exact against the oracle) and the decode attention over q8_0 caches
(within 2e-3 * sum p|v| of the fp64 oracle over the same codes and scales).

The attention's rounding budget: keys enter exactly (int8 codes times the
block scale in fp32), V is rounded once to fp16 (<= 2^-11 relative) and the
probabilities are fp16 (<= 2^-11 relative), so |o - o_ref| <= ~2^-10 * B plus
fp32 accumulation, under the 2e-3 * B bar; rounding the output to bf16 adds at
most half a bf16 ulp (2^-8 relative).
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


def _check_attn(O_gpu_bits, O_ref, B, orc):
    """The fp32 result within 2e-3 * B of the oracle, then rounded to bf16: at
    most half a bf16 ulp more (2^-8 relative, the 8-bit significand)."""
    o = orc.bf16_array_to_f64(O_gpu_bits)
    ref_b = orc.bf16_array_to_f64(orc.f64_array_to_bf16(O_ref))
    ulp_half = np.abs(O_ref) * 2.0 ** -8
    bound = 2e-3 * B + ulp_half + 1e-30
    assert (np.abs(o - O_ref) <= bound).all(), np.max(np.abs(o - O_ref) / bound)
    # per (row, head): the fp32 result within 2e-3 relative (2-norm), plus the bf16 rounding of the output
    num = np.linalg.norm(o - O_ref, axis=-1)
    den = np.linalg.norm(O_ref, axis=-1)
    assert (num <= 2e-3 * den + np.linalg.norm(ulp_half, axis=-1) + 1e-30).all(), (num / den).max()
    # and most outputs round to the same bf16 value as the oracle's
    assert (o == ref_b).mean() > 0.8


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_q8_0_quantize_bit_exact(q, orc, dtype):
    rng = np.random.default_rng(21)
    n_blocks = 5000
    x = (rng.standard_normal((n_blocks, 32)) * 10.0 ** rng.integers(-5, 4, (n_blocks, 1))).astype(np.float32)
    x[0] = 0.0
    x[1] = np.arange(32) - 15.5                      # rounding ties once scaled
    x[2] = np.round(rng.standard_normal(32) * 50)
    x[2, 7] = -127.0                                 # d = 1 exactly
    x[3] = 1e-6 * (np.arange(32) - 16)               # fp16-subnormal scale
    if dtype == "bf16":
        xb = synth.bf16_bits_np(x)
        x = orc.bf16_array_to_f64(xb).astype(np.float32)
        xd = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
    else:
        xd = torch.from_numpy(x).cuda()
    qg, dg = q.q8_0_quantize(xd)
    torch.cuda.synchronize()
    qr, dr = orc.q8_0_quantize(x)
    assert np.array_equal(qg.cpu().numpy(), qr.reshape(-1))
    assert np.array_equal(dg.cpu().numpy().view(np.uint16), dr.reshape(-1))


def test_q8_0_quantize_rejects_bad_arguments(q):
    x = torch.zeros(48, device="cuda")
    with pytest.raises(q.QadError):
        q.q8_0_quantize(x)                           # 48 % 32 != 0


def _q8_inputs(lens, n_rows, n_qh, n_kvh, seed, qscale=1.0, cap_extra=5):
    A = len(lens)
    cap = max(l + n for l, n in zip(lens, n_rows)) + cap_extra
    ars = np.concatenate([[0], np.cumsum(n_rows)]).astype(np.int32)
    M = int(ars[-1])
    g = synth.torch_gen(SEED, "cpu", 600 + seed)
    Kq, Kd = synth.q8_planes_torch(g, A * n_kvh * cap, 128, "cpu")
    Vq, Vd = synth.q8_planes_torch(g, A * n_kvh * cap, 128, "cpu")
    Q = synth.bf16_normal_np(SEED, 700 + seed, (max(M, 1), n_qh, 128), scale=qscale)[:M]
    sh, shd = (A, n_kvh, cap, 128), (A, n_kvh, cap, 4)
    planes = [Kq.numpy().reshape(sh), Kd.numpy().view(np.uint16).reshape(shd),
              Vq.numpy().reshape(sh), Vd.numpy().view(np.uint16).reshape(shd)]
    return Q, planes, np.array(lens, np.int32), ars, cap


def _run_q8(q, Q, planes, lens, ars, n_qh, n_kvh, cap):
    M = int(ars[-1])
    max_rows = int(max(np.diff(ars).max(), 1))
    dev = [torch.from_numpy(np.ascontiguousarray(p).view(np.int8 if p.dtype == np.int8 else np.int16)).cuda()
           for p in planes]
    Qd = torch.from_numpy(np.ascontiguousarray(Q).view(np.int16)).view(torch.bfloat16).cuda() if M else \
        torch.zeros(1, n_qh, 128, dtype=torch.bfloat16, device="cuda")
    O = torch.zeros(max(M, 1), n_qh, 128, dtype=torch.bfloat16, device="cuda")
    q.decode_attn_q8(Qd, *dev, torch.from_numpy(lens).cuda(), torch.from_numpy(ars).cuda(), len(lens), max_rows,
                     cap, n_qh, n_kvh, 128, O)
    torch.cuda.synchronize()
    return _bits(O)[:M]


@pytest.mark.parametrize("lens,n_rows,n_qh,n_kvh", [
    ([40, 0, 7, 129], [3, 3, 3, 3], 48, 8),
    ([5, 300], [1, 4], 6, 2),
    ([0, 1, 2], [3, 0, 2], 6, 2),
    ([1100, 16, 2047], [3, 3, 2], 48, 8),   # several splits, tile tails
    ([17], [16], 8, 2),                      # 16 rows of one agent: 4 row groups
])
def test_attn_q8_parity(q, orc, lens, n_rows, n_qh, n_kvh):
    Q, planes, lens, ars, cap = _q8_inputs(lens, n_rows, n_qh, n_kvh, seed=len(lens) + n_qh + sum(n_rows))
    O_ref, B = orc.decode_attn_q8(Q, *planes, lens, ars, n_qh, n_kvh, 128, cap)
    _check_attn(_run_q8(q, Q, planes, lens, ars, n_qh, n_kvh, cap), O_ref, B, orc)


def test_attn_q8_peaked_scores(q, orc):
    """q scaled x4: softmax dominated by a few keys (large corrections between tiles)."""
    Q, planes, lens, ars, cap = _q8_inputs([700, 90], [3, 3], 48, 8, seed=7, qscale=4.0)
    O_ref, B = orc.decode_attn_q8(Q, *planes, lens, ars, 48, 8, 128, cap)
    _check_attn(_run_q8(q, Q, planes, lens, ars, 48, 8, cap), O_ref, B, orc)


def test_attn_q8_full_size_23k_context(q, orc):
    """4 agents x 23000 cached tokens, 3 rows each, 48 q-heads / 8 kv-heads, every output."""
    n_qh, n_kvh, A, L = 48, 8, 4, 23000
    cap = L + 3
    g = synth.torch_gen(SEED, "cuda", 3)
    Kq, Kd = synth.q8_planes_torch(g, A * n_kvh * cap, 128, "cuda")
    Vq, Vd = synth.q8_planes_torch(g, A * n_kvh * cap, 128, "cuda")
    Qd = synth.bf16_normal_torch(g, (12, n_qh, 128), "cuda")
    lens = np.full(A, L, np.int32)
    ars = np.arange(0, 13, 3, dtype=np.int32)
    O = torch.zeros(12, n_qh, 128, dtype=torch.bfloat16, device="cuda")
    q.decode_attn_q8(Qd, Kq, Kd.view(torch.int16), Vq, Vd.view(torch.int16), torch.from_numpy(lens).cuda(),
                     torch.from_numpy(ars).cuda(), A, 3, cap, n_qh, n_kvh, 128, O)
    torch.cuda.synchronize()
    sh, shd = (A, n_kvh, cap, 128), (A, n_kvh, cap, 4)
    O_ref, B = orc.decode_attn_q8(_bits(Qd), Kq.cpu().numpy().reshape(sh), _bits(Kd).reshape(shd),
                                  Vq.cpu().numpy().reshape(sh), _bits(Vd).reshape(shd), lens, ars, n_qh, n_kvh,
                                  128, cap)
    _check_attn(_bits(O), O_ref, B, orc)
