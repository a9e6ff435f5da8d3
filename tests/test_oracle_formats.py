"""Pins for the oracle's number-format conversions (CPU only).

fp16 and bf16 decoding are checked over every bit pattern against numpy's and
torch's own conversions; bf16 rounding from fp64 is checked against
hand-derived cases (tests/golden/bf16_rounding.json) and, on values that are
exact in float32, against torch's float32 -> bfloat16 conversion.
"""
import numpy as np
import pytest
import torch

from conftest import golden


def test_half_to_double_all_patterns(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.half_to_double(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_bf16_to_double_all_patterns(orc):
    bits = np.arange(65536, dtype=np.int32).astype(np.int16)
    ref = torch.from_numpy(bits).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([orc.bf16_to_double(int(b) & 0xFFFF) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_double_to_bf16_golden(orc):
    for c in golden("bf16_rounding.json")["cases"]:
        x = float(np.ldexp(np.float64(c["m"]), c["e"]))
        assert c["m"] * 2.0 ** c["e"] == x  # the input is exact in fp64
        assert orc.double_to_bf16(x) == int(c["bits"], 16), c["why"]


def test_double_to_bf16_matches_torch_on_float32_values(orc):
    g = np.random.default_rng(7)
    vals = np.concatenate([
        g.standard_normal(20000).astype(np.float32),
        (g.standard_normal(2000) * 1e30).astype(np.float32),
        (g.standard_normal(2000) * 1e-38).astype(np.float32),  # subnormal range
        np.float32([0.0, -0.0, 65504.0, 3.0e38, -3.4e38]),
    ])
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.double_to_bf16(float(v)) for v in vals], np.uint16)
    assert (got == ref).all()


@pytest.mark.parametrize("x,bits", [(float("inf"), 0x7F80), (float("-inf"), 0xFF80), (-0.0, 0x8000)])
def test_double_to_bf16_specials(orc, x, bits):
    assert orc.double_to_bf16(x) == bits
