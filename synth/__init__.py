"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and bench.py.

This module only draws random numbers and lays them into the byte layouts the
two implementations consume. It holds none of the decode-step arithmetic: no
dequantisation, no dot products, no softmax, no normalisation.

Distributions (the workloads named for the multi-agent decode step):

* Q4_K super-blocks (144 bytes = 256 weights): ``d`` and ``dmin`` are
  fp16(|N(0,1)| * 0.01); the other 140 bytes (12 bytes of packed 6-bit
  scales/mins, 128 bytes of 4-bit quants) are uniform random bytes. The packing
  of the 16 six-bit fields into the 12 scale bytes uses every bit exactly once
  and each quant byte holds two whole nibbles, so uniform bytes are exactly
  "quants uniform in 0..15, scales and mins uniform in 0..63".
* Q6_K-like blocks (210 bytes = 256 weights): the 128 low-nibble bytes and the
  64 high-bit bytes are uniform random bytes (every 6-bit quant uniform in
  0..63), the 16 int8 sub-block scales are uniform in 0..63 (or, with
  ``signed=True``, uniform over the whole int8 range -128..127, as quantisers
  of real checkpoints produce) and ``d`` is fp16(|N(0,1)| * 0.01).
* Activations, queries, keys and values: bf16(N(0,1)) (round to nearest even).

Two back ends draw the same distributions: numpy on the host (small cases the
oracle checks in full) and torch on any device (the full-size workloads, drawn
directly in device memory). The two back ends produce different streams for the
same seed; a test always feeds one buffer to both implementations.
"""
from __future__ import annotations

import numpy as np
import torch

Q4K_BLOCK_BYTES = 144
Q6K_BLOCK_BYTES = 210
QK = 256

# Byte offsets inside a block (storage layout only; no arithmetic).
Q4K_D_OFF, Q4K_DMIN_OFF = 0, 2
Q6K_SCALES_OFF, Q6K_D_OFF = 192, 208


def np_rng(seed: int, *stream: int) -> np.random.Generator:
    """Independent numpy generator for (seed, stream...)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), *map(int, stream)])))


def torch_gen(seed: int, device, *stream: int) -> torch.Generator:
    """torch generator on ``device`` seeded from (seed, stream...)."""
    s = np.random.SeedSequence([int(seed), *map(int, stream)]).generate_state(1, np.uint64)[0]
    g = torch.Generator(device=device)
    g.manual_seed(int(s) & ((1 << 63) - 1))
    return g


def _fp16_bits_np(a: np.ndarray) -> np.ndarray:
    return np.asarray(a, np.float64).astype(np.float16).view(np.uint16)


def bf16_bits_np(a: np.ndarray) -> np.ndarray:
    """Round float values to bf16 (nearest even) and return the raw uint16 bits."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- host (numpy)

def q4k_matrix_np(seed: int, tag: int, n_rows: int, k: int) -> np.ndarray:
    """uint8 [n_rows, k/256*144]: row n's super-blocks are contiguous."""
    assert k % QK == 0
    nb = n_rows * (k // QK)
    g = np_rng(seed, 4, tag)
    blk = g.integers(0, 256, size=(nb, Q4K_BLOCK_BYTES), dtype=np.uint8)
    d = _fp16_bits_np(np.abs(g.standard_normal(nb)) * 0.01)
    dmin = _fp16_bits_np(np.abs(g.standard_normal(nb)) * 0.01)
    blk[:, Q4K_D_OFF:Q4K_D_OFF + 2] = d.view(np.uint8).reshape(nb, 2)
    blk[:, Q4K_DMIN_OFF:Q4K_DMIN_OFF + 2] = dmin.view(np.uint8).reshape(nb, 2)
    return blk.reshape(n_rows, (k // QK) * Q4K_BLOCK_BYTES)


def q6k_matrix_np(seed: int, tag: int, n_rows: int, k: int, signed: bool = False) -> np.ndarray:
    """uint8 [n_rows, k/256*210]: row n's blocks are contiguous."""
    assert k % QK == 0
    nb = n_rows * (k // QK)
    g = np_rng(seed, 6, tag)
    blk = g.integers(0, 256, size=(nb, Q6K_BLOCK_BYTES), dtype=np.uint8)
    blk[:, Q6K_SCALES_OFF:Q6K_SCALES_OFF + 16] = g.integers(0, 256 if signed else 64, size=(nb, 16), dtype=np.uint8)
    d = _fp16_bits_np(np.abs(g.standard_normal(nb)) * 0.01)
    blk[:, Q6K_D_OFF:Q6K_D_OFF + 2] = d.view(np.uint8).reshape(nb, 2)
    return blk.reshape(n_rows, (k // QK) * Q6K_BLOCK_BYTES)


def bf16_normal_np(seed: int, tag: int, shape, scale: float = 1.0) -> np.ndarray:
    """uint16 bf16 bits of N(0,1)*scale, rounded to nearest even."""
    g = np_rng(seed, 16, tag)
    return bf16_bits_np(g.standard_normal(shape) * scale)


# ---------------------------------------------------------------- device (torch)

def q4k_matrix_torch(gen: torch.Generator, n_rows: int, k: int, device) -> torch.Tensor:
    """uint8 [n_rows, k/256*144] drawn in ``device`` memory."""
    assert k % QK == 0
    nb = n_rows * (k // QK)
    blk = torch.randint(0, 256, (nb, Q4K_BLOCK_BYTES), dtype=torch.uint8, device=device, generator=gen)
    for off in (Q4K_D_OFF, Q4K_DMIN_OFF):
        v = (torch.randn(nb, device=device, generator=gen).abs_() * 0.01).to(torch.float16)
        blk[:, off:off + 2] = v.view(torch.uint8).view(nb, 2)
    return blk.view(n_rows, (k // QK) * Q4K_BLOCK_BYTES)


def q6k_matrix_torch(gen: torch.Generator, n_rows: int, k: int, device, signed: bool = False) -> torch.Tensor:
    """uint8 [n_rows, k/256*210] drawn in ``device`` memory."""
    assert k % QK == 0
    nb = n_rows * (k // QK)
    blk = torch.randint(0, 256, (nb, Q6K_BLOCK_BYTES), dtype=torch.uint8, device=device, generator=gen)
    blk[:, Q6K_SCALES_OFF:Q6K_SCALES_OFF + 16] = torch.randint(
        0, 256 if signed else 64, (nb, 16), dtype=torch.uint8, device=device, generator=gen)
    v = (torch.randn(nb, device=device, generator=gen).abs_() * 0.01).to(torch.float16)
    blk[:, Q6K_D_OFF:Q6K_D_OFF + 2] = v.view(torch.uint8).view(nb, 2)
    return blk.view(n_rows, (k // QK) * Q6K_BLOCK_BYTES)


def bf16_normal_torch(gen: torch.Generator, shape, device, scale: float = 1.0) -> torch.Tensor:
    """bf16 N(0,1)*scale drawn in ``device`` memory (float32 draw, nearest-even to bf16)."""
    t = torch.randn(shape, device=device, generator=gen)
    if scale != 1.0:
        t.mul_(scale)
    return t.to(torch.bfloat16)


def q8_planes_torch(gen: torch.Generator, n_rows: int, hd: int, device):
    """A q8_0-shaped cache of n_rows rows drawn in ``device`` memory: int8 codes
    [n_rows, hd] (normal, sd 42, clipped to +-127) and fp16 scales [n_rows, hd/32]
    uniform in [0.01, 0.03) (values of roughly N(0,1) size)."""
    codes = torch.randn((n_rows, hd), device=device, generator=gen).mul_(42.0).round_().clamp_(-127, 127)
    scales = torch.rand((n_rows, hd // 32), device=device, generator=gen).mul_(0.02).add_(0.01)
    return codes.to(torch.int8), scales.to(torch.float16)


# ---------------------------------------------------------------- model shapes

class StackShape:
    """Layer shapes of the synthetic decoder stack (hidden, intermediate, heads)."""

    def __init__(self, n_layers=64, hidden=5120, inter=17408, n_qh=48, n_kvh=8, head_dim=128):
        self.n_layers, self.hidden, self.inter = n_layers, hidden, inter
        self.n_qh, self.n_kvh, self.head_dim = n_qh, n_kvh, head_dim

    @property
    def qkv_rows(self):
        return (self.n_qh + 2 * self.n_kvh) * self.head_dim

    def weight_bytes_per_layer(self):
        h, i = self.hidden, self.inter
        q4 = (self.qkv_rows * h + h * self.n_qh * self.head_dim + 2 * i * h) // QK * Q4K_BLOCK_BYTES
        q6 = h * i // QK * Q6K_BLOCK_BYTES
        return q4 + q6


# Matrix tags used to seed each tensor independently.
TAG_Q, TAG_K, TAG_V, TAG_O, TAG_GATE, TAG_UP, TAG_DOWN = range(7)


def layer_weight_tag(layer: int, mat: int) -> int:
    return 1000 + 16 * layer + mat
