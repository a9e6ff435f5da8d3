"""Pins of the oracle's fp16 rounding, q8_0 quantiser and q8_0-cache attention."""
import numpy as np

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
