"""Pins for the oracle's Q4_K and Q6_K block codecs (CPU only).

* Hand-derived worked examples (tests/golden/q4k_worked.json, q6k_worked.json).
* The installed ``gguf`` package's numpy dequantiser (an independent library
  implementation of the same GGUF block formats) on random blocks.
* Exhaustive encode -> decode round trips over every 6-bit scale/min value in
  every sub-block slot and every quant value in every position, and
  decode -> encode on random bytes (the packing is a bijection).
"""
import numpy as np
import pytest

import synth
from conftest import SEED, golden

gguf = pytest.importorskip("gguf")
from gguf import quants  # noqa: E402


def _block_from_bytes(n, set_bytes):
    b = np.zeros(n, np.uint8)
    for k, v in set_bytes.items():
        b[int(k)] = v
    return b


@pytest.mark.parametrize("case", golden("q4k_worked.json")["cases"], ids=lambda c: c["name"])
def test_q4k_worked_examples(orc, case):
    blk = _block_from_bytes(144, case["set_bytes"])
    w = orc.dequant(4, blk, 1, 256)[0]
    for i, v in case["expect"].items():
        assert w[int(i)] == v, (i, case["why"])
    if case.get("zero_elsewhere"):
        mask = np.ones(256, bool)
        mask[[int(i) for i in case["expect"]]] = False
        assert (w[mask] == 0).all()
    # the library reproduces the same hand values
    lw = quants.dequantize(blk, gguf.GGMLQuantizationType.Q4_K).astype(np.float64)
    for i, v in case["expect"].items():
        assert lw[int(i)] == v


@pytest.mark.parametrize("case", golden("q6k_worked.json")["cases"], ids=lambda c: c["name"])
def test_q6k_worked_examples(orc, case):
    blk = _block_from_bytes(210, case["set_bytes"])
    w = orc.dequant(6, blk, 1, 256)[0]
    for i, v in case["expect"].items():
        assert w[int(i)] == v, (i, case["why"])
    lw = quants.dequantize(blk, gguf.GGMLQuantizationType.Q6_K).astype(np.float64)
    for i, v in case["expect"].items():
        assert lw[int(i)] == v


def _f32_bound(terms):
    # gguf computes in float32: a few roundings of products bounded by `terms`
    return 4 * 2.0 ** -23 * terms + 1e-30


def test_q4k_matches_gguf_on_random_blocks(orc):
    W = synth.q4k_matrix_np(SEED, 1, 64, 1024)  # 256 blocks
    ours = orc.dequant(4, W, 64, 1024).reshape(-1, 256)
    lib = quants.dequantize(W.reshape(-1, 144), gguf.GGMLQuantizationType.Q4_K).astype(np.float64)
    # |d*sc*q| + |dmin*m| bounds each float32 rounding in the library's formula
    terms = np.zeros_like(ours)
    for b in range(ours.shape[0]):
        q, sc, m, d, dmin = orc.q4k_decode(W.reshape(-1, 144)[b])
        dd, dm = orc.half_to_double(d), orc.half_to_double(dmin)
        terms[b] = np.abs(dd * np.repeat(sc, 32) * q) + np.abs(dm * np.repeat(m, 32))
    assert (np.abs(ours - lib.reshape(ours.shape)) <= _f32_bound(terms)).all()


def test_q6k_matches_gguf_on_random_blocks(orc):
    W = synth.q6k_matrix_np(SEED, 1, 64, 1024)
    ours = orc.dequant(6, W, 64, 1024).reshape(-1, 256)
    lib = quants.dequantize(W.reshape(-1, 210), gguf.GGMLQuantizationType.Q6_K).astype(np.float64)
    assert (np.abs(ours - lib.reshape(ours.shape)) <= _f32_bound(np.abs(ours))).all()


def test_q6k_negative_scales_match_gguf(orc):
    g = np.random.default_rng(3)
    blk = g.integers(0, 256, size=(32, 210), dtype=np.uint8)
    blk[:, 208:210] = np.frombuffer(np.float16([0.01] * 32).tobytes(), np.uint8).reshape(32, 2)
    ours = orc.dequant(6, blk, 32, 256)
    lib = quants.dequantize(blk, gguf.GGMLQuantizationType.Q6_K).astype(np.float64).reshape(32, 256)
    assert (np.abs(ours - lib) <= _f32_bound(np.abs(ours))).all()


def test_q4k_roundtrip_every_scale_and_min_in_every_slot(orc):
    q = np.zeros(256, np.uint8)
    for j in range(8):
        for s in range(64):
            sc = np.full(8, 5, np.uint8)
            m = np.full(8, 9, np.uint8)
            sc[j] = s
            for mv in range(64):
                m[j] = mv
                blk = orc.q4k_encode(q, sc, m, 0x1234, 0x4321)
                q2, sc2, m2, d2, dm2 = orc.q4k_decode(blk)
                assert (sc2 == sc).all() and (m2 == m).all() and d2 == 0x1234 and dm2 == 0x4321


def test_q4k_roundtrip_every_quant_in_every_position(orc):
    sc = np.arange(8, dtype=np.uint8)
    m = np.arange(8, dtype=np.uint8) * 7
    for v in range(16):
        q = np.full(256, (v + 5) % 16, np.uint8)
        for pos in range(256):
            q2 = q.copy()
            q2[pos] = v
            blk = orc.q4k_encode(q2, sc, m, 0, 0)
            assert (orc.q4k_decode(blk)[0] == q2).all()


def test_q4k_bytes_roundtrip_is_bijection(orc):
    g = np.random.default_rng(11)
    for _ in range(2000):
        blk = g.integers(0, 256, 144, dtype=np.uint8)
        q, sc, m, d, dmin = orc.q4k_decode(blk)
        assert (orc.q4k_encode(q, sc, m, d, dmin) == blk).all()


def test_q6k_roundtrip(orc):
    g = np.random.default_rng(12)
    for _ in range(2000):
        blk = g.integers(0, 256, 210, dtype=np.uint8)
        q, sc, d = orc.q6k_decode(blk)
        assert q.max() < 64
        assert (orc.q6k_encode(q, sc, d) == blk).all()
    for v in range(64):
        for pos in range(0, 256, 7):
            q = np.full(256, 63 - v, np.uint8)
            q[pos] = v
            blk = orc.q6k_encode(q, np.arange(16, dtype=np.int8), 0x3C00)
            assert (orc.q6k_decode(blk)[0] == q).all()


def test_synth_q4k_fields_are_uniform(orc):
    """The generator's uniform bytes decode to uniform quants, scales and mins."""
    W = synth.q4k_matrix_np(SEED, 2, 256, 1024).reshape(-1, 144)
    qs, scs, ms = [], [], []
    for b in W:
        q, sc, m, _, _ = orc.q4k_decode(b)
        qs.append(q), scs.append(sc), ms.append(m)
    qh = np.bincount(np.concatenate(qs), minlength=16)
    sh = np.bincount(np.concatenate(scs), minlength=64)
    mh = np.bincount(np.concatenate(ms), minlength=64)
    for h in (qh, sh, mh):
        exp = h.sum() / len(h)
        chi2 = ((h - exp) ** 2 / exp).sum()
        assert chi2 < 3 * len(h)
    d = np.array([orc.half_to_double(int(v)) for v in W[:, 0:2].copy().view(np.uint16).ravel()])
    assert (d >= 0).all() and 0.005 < d.mean() < 0.011  # E|N(0,1)|*0.01 = 0.00798
