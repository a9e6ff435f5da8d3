"""Pins of the oracle's fp16 rounding, q8_0 quantiser and q8_0-cache attention."""
import numpy as np
import pytest

import synth
from conftest import SEED


def test_double_to_half_matches_ieee_rounding(orc):
    rng = np.random.default_rng(11)
    # every fp16 value, the midpoints between neighbours (ties) and random magnitudes
    h = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = (h[:-1] + h[1:]) / 2
    xs = np.concatenate([h, mids, -mids[::97], rng.standard_normal(2000) * 10.0 ** rng.integers(-9, 5, 2000),
                         [65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -25, 2.0 ** -24 * 1.5, 0.0, -0.0]])
    for x in xs:
        want = np.array([x], np.float64).astype(np.float16).view(np.uint16)[0]
        assert orc.double_to_half(x) == want, (x, orc.double_to_half(x), want)


def test_q8_0_hand_cases(orc):
    x = np.zeros((3, 32), np.float32)
    x[0, :31] = np.arange(31) - 16      # integers, amax 127 -> d = 1, q = x
    x[0, 31] = 127
    x[2, :] = 0.5 * np.arange(-16, 16)  # amax 8: d = 8/127
    x[2, 0] = -127                      # amax 127 again: d = 1, ties round away from zero
    x[2, 1], x[2, 2] = 2.5, -2.5
    q, d = orc.q8_0_quantize(x)
    assert d[0, 0] == 0x3C00 and q[0].tolist() == x[0].astype(int).tolist()
    assert d[1, 0] == 0 and not q[1].any()  # an all-zero block
    assert d[2, 0] == 0x3C00 and q[2, 1] == 3 and q[2, 2] == -3 and q[2, 0] == -127
    assert q[2, 3] == -7 and q[2, 31] == 8  # -6.5 -> -7, 7.5 -> 8 (half away from zero)


def test_q8_0_error_bound(orc):
    x = (np.random.default_rng(12).standard_normal((64, 128)) * 3).astype(np.float32)
    q, d = orc.q8_0_quantize(x)
    dh = d.view(np.float16).astype(np.float64)
    amax = np.abs(x.reshape(64, 4, 32)).max(axis=2)
    deq = dh[:, :, None] * q.reshape(64, 4, 32)
    err = np.abs(deq - x.reshape(64, 4, 32))
    df = amax / 127.0
    # half a step of the fp32 scale, plus the fp16 rounding of the scale times |q|
    assert (err <= df[:, :, None] * 0.5 * (1 + 1e-6) + np.abs(dh - df)[:, :, None] * 127 + 1e-12).all()
    assert np.abs(q).max() <= 127


def test_q8_attention_equals_bf16_attention_on_exact_values(orc):
    """Power-of-two scales make every dequantised value exact in bf16, so the q8_0 attention
    must equal the bf16 attention over those values."""
    A, n_kvh, n_qh, hd = 2, 2, 6, 128
    lens, n_rows = [9, 30], [3, 2]
    cap = 40
    rng = np.random.default_rng(13)
    Kq = rng.integers(-127, 128, (A, n_kvh, cap, hd)).astype(np.int8)
    Vq = rng.integers(-127, 128, (A, n_kvh, cap, hd)).astype(np.int8)
    pw = 2.0 ** rng.integers(-9, -3, (A, n_kvh, cap, hd // 32))
    Kd = pw.astype(np.float16).view(np.uint16)
    Vd = (pw * 2).astype(np.float16).view(np.uint16)
    Kb = orc.f64_array_to_bf16(np.repeat(pw, 32, axis=3) * Kq)
    Vb = orc.f64_array_to_bf16(np.repeat(pw * 2, 32, axis=3) * Vq)
    ars = np.array([0, 3, 5], np.int32)
    Q = synth.bf16_normal_np(SEED, 30, (5, n_qh, hd))
    O8, B8 = orc.decode_attn_q8(Q, Kq, Kd, Vq, Vd, lens, ars, n_qh, n_kvh, hd, cap)
    O, B = orc.decode_attn(Q, Kb, Vb, lens, ars, n_qh, n_kvh, hd, cap)
    assert np.array_equal(O8, O) and np.array_equal(B8, B)


def test_q8_0_matches_gguf_quantiser(orc):
    """The gguf package's Q8_0 quantiser (numpy, float32) is an independent
    implementation of the same block format."""
    gguf = pytest.importorskip("gguf")
    rng = np.random.default_rng(14)
    x = (rng.standard_normal((300, 32)) * 10.0 ** rng.integers(-4, 4, (300, 1))).astype(np.float32)
    x[0] = 0.0
    x[1, :] = np.arange(32) - 15.5          # halves: ties at every value once scaled
    x[2, :] = np.round(rng.standard_normal(32) * 50).astype(np.float32)
    x[2, 5] = 127.0                          # d = 1 exactly
    x[3, :] = 1e-6 * (np.arange(32) - 16)    # scale in the fp16 subnormal range
    q, d = orc.q8_0_quantize(x)
    ref = gguf.quants.quantize(x.reshape(-1), gguf.GGMLQuantizationType.Q8_0).reshape(300, 34)
    assert np.array_equal(d[:, 0], ref[:, :2].copy().view(np.uint16)[:, 0])
    assert np.array_equal(q, ref[:, 2:].view(np.int8))


def test_q8_decode_layer_appends_and_attends(orc):
    """The q8_0 layer: everything before the append equals the bf16 layer; the
    appended codes are the gguf Q8_0 blocks of the fp32 projection; the
    attention output matches torch SDPA over the dequantised cache."""
    gguf = pytest.importorskip("gguf")
    import torch
    import torch.nn.functional as F
    H, I, n_qh, n_kvh, hd = 256, 512, 4, 2, 128
    nq, nkv = n_qh * hd, n_kvh * hd
    lens = np.array([6, 0, 11], np.int32)
    ars = np.array([0, 3, 5, 6], np.int32)
    M, A, cap = 6, 3, 20
    Wqkv = synth.q4k_matrix_np(SEED, 50, nq + 2 * nkv, H)
    Wo = synth.q4k_matrix_np(SEED, 51, H, nq)
    Wgu = synth.q4k_matrix_np(SEED, 52, 2 * I, H)
    Wd = synth.q6k_matrix_np(SEED, 53, H, I)
    rng = np.random.default_rng(15)
    Kq = rng.integers(-127, 128, (A, n_kvh, cap, hd)).astype(np.int8)
    Vq = rng.integers(-127, 128, (A, n_kvh, cap, hd)).astype(np.int8)
    Kd = (np.abs(rng.standard_normal((A, n_kvh, cap, hd // 32))) * 0.02 + 1e-3).astype(np.float16).view(np.uint16)
    Vd = (np.abs(rng.standard_normal((A, n_kvh, cap, hd // 32))) * 0.02 + 1e-3).astype(np.float16).view(np.uint16)
    h0 = orc.bf16_array_to_f64(synth.bf16_normal_np(SEED, 56, (M, H)))
    h8, hb = h0.copy(), h0.copy()
    K8, V8 = (Kq.copy(), Kd.copy()), (Vq.copy(), Vd.copy())
    i8 = orc.decode_layer(Wqkv, Wo, Wgu, Wd, H, I, n_qh, n_kvh, hd, h8, ars, lens, K8, V8, cap, want=True)
    Kb = synth.bf16_normal_np(SEED, 54, (A, n_kvh, cap, hd))
    Vb = synth.bf16_normal_np(SEED, 55, (A, n_kvh, cap, hd))
    ib = orc.decode_layer(Wqkv, Wo, Wgu, Wd, H, I, n_qh, n_kvh, hd, hb, ars, lens, Kb, Vb, cap, want=True)
    assert np.array_equal(i8["x1"], ib["x1"]) and np.array_equal(i8["qkv"], ib["qkv"])

    def gq8(v):
        blk = gguf.quants.quantize(v.astype(np.float32).reshape(-1), gguf.GGMLQuantizationType.Q8_0).reshape(-1, 34)
        return blk[:, 2:].view(np.int8).reshape(-1), blk[:, :2].copy().view(np.uint16).reshape(-1)
    for r in range(M):
        a = int(np.searchsorted(ars, r, side="right") - 1)
        pos = lens[a] + r - ars[a]
        for g in range(n_kvh):
            for plane, off in ((K8, nq), (V8, nq + nkv)):
                q, d = gq8(i8["qkv"][r, off + g * hd: off + (g + 1) * hd])
                assert np.array_equal(plane[0][a, g, pos], q) and np.array_equal(plane[1][a, g, pos], d)
    # attention over the dequantised cache, restated with torch SDPA
    deq = lambda P: np.repeat(P[1].view(np.float16).astype(np.float64), 32, axis=3) * P[0]  # noqa: E731
    Kf, Vf = torch.from_numpy(deq(K8)), torch.from_numpy(deq(V8))
    Q = torch.from_numpy(orc.bf16_array_to_f64(orc.f64_array_to_bf16(i8["qkv"][:, :nq]))).reshape(M, n_qh, hd)
    G = n_qh // n_kvh
    o = torch.zeros(M, n_qh, hd, dtype=torch.float64)
    for a in range(A):
        r0, r1 = int(ars[a]), int(ars[a + 1])
        if r1 == r0:
            continue
        nk = int(lens[a]) + r1 - r0
        mask = torch.arange(nk)[None, :] <= (torch.arange(r1 - r0) + int(lens[a]))[:, None]
        o[r0:r1] = F.scaled_dot_product_attention(Q[r0:r1].permute(1, 0, 2), Kf[a, :, :nk].repeat_interleave(G, 0),
                                                  Vf[a, :, :nk].repeat_interleave(G, 0),
                                                  attn_mask=mask).permute(1, 0, 2)
    o = o.reshape(M, nq).numpy()
    got = orc.bf16_array_to_f64(i8["attn"])
    assert np.abs(got - o).max() <= 2.0 ** -8 * np.abs(o).max()


def test_q8_attention_matches_numpy_restatement(orc):
    """The q8_0 attention against numpy on tiny random caches: dequantise
    (fp16 scale x int8 code), scores, max-subtracted softmax, weighted sum."""
    A, n_kvh, n_qh, hd, cap = 2, 1, 3, 128, 12
    lens, ars = np.array([4, 9], np.int32), np.array([0, 2, 3], np.int32)
    rng = np.random.default_rng(16)
    Kq = rng.integers(-127, 128, (A, n_kvh, cap, hd)).astype(np.int8)
    Vq = rng.integers(-127, 128, (A, n_kvh, cap, hd)).astype(np.int8)
    Kd = (rng.random((A, n_kvh, cap, hd // 32)) * 0.02 + 0.001).astype(np.float16).view(np.uint16)
    Vd = (rng.random((A, n_kvh, cap, hd // 32)) * 0.02 + 0.001).astype(np.float16).view(np.uint16)
    Q = synth.bf16_normal_np(SEED, 31, (3, n_qh, hd))
    O, _ = orc.decode_attn_q8(Q, Kq, Kd, Vq, Vd, lens, ars, n_qh, n_kvh, hd, cap)
    K = np.repeat(Kd.view(np.float16).astype(np.float64), 32, axis=3) * Kq
    V = np.repeat(Vd.view(np.float16).astype(np.float64), 32, axis=3) * Vq
    q = orc.bf16_array_to_f64(Q)
    for r in range(3):
        a = 0 if r < 2 else 1
        nk = lens[a] + (r - ars[a]) + 1
        for h in range(n_qh):
            s = K[a, 0, :nk] @ q[r, h] / np.sqrt(hd)
            p = np.exp(s - s.max())
            ref = (p / p.sum()) @ V[a, 0, :nk]
            assert np.allclose(O[r, h], ref, rtol=1e-12, atol=1e-12)
