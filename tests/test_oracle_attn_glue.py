"""Pins for the oracle's attention, layer glue and row packer (CPU only).

Attention (OpenJet page, section 只搬一次权重: each agent reads its own KV
cache; drafts are verified in the same pass) is checked against torch's
``scaled_dot_product_attention`` in float64 with an explicit causal/GQA mask,
and against closed forms: one visible key, identical keys, one dominant key,
head permutation within a group, and the equivalence of the draft rows with
one-at-a-time decoding.

RMSNorm and SiLU*mul are checked against torch's float64 functions; the row
packer against a hand-derived example; one decoder layer against an
independent numpy/torch composition built from library routines
(gguf dequantisation, torch attention and normalisation).
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import synth
from conftest import SEED, golden


def _f64(b):
    import oracle
    return oracle.bf16_array_to_f64(b)


def _attn_case(lens, n_rows, n_qh=6, n_kvh=2, hd=128, seed=1, qscale=1.0):
    A = len(lens)
    cap = max(l + n for l, n in zip(lens, n_rows)) + 3
    ars = np.concatenate([[0], np.cumsum(n_rows)]).astype(np.int32)
    M = int(ars[-1])
    Q = synth.bf16_normal_np(SEED, 100 + seed, (M, n_qh, hd), scale=qscale)
    Kc = synth.bf16_normal_np(SEED, 200 + seed, (A, n_kvh, cap, hd))
    Vc = synth.bf16_normal_np(SEED, 300 + seed, (A, n_kvh, cap, hd))
    return Q, Kc, Vc, np.array(lens, np.int32), ars, cap


def _torch_ref(Q, Kc, Vc, lens, ars, n_qh, n_kvh, hd):
    q = torch.from_numpy(_f64(Q))
    k = torch.from_numpy(_f64(Kc))
    v = torch.from_numpy(_f64(Vc))
    out = torch.zeros(q.shape, dtype=torch.float64)
    G = n_qh // n_kvh
    for a in range(len(lens)):
        r0, r1 = int(ars[a]), int(ars[a + 1])
        if r1 == r0:
            continue
        nk = int(lens[a]) + (r1 - r0)
        qa = q[r0:r1].permute(1, 0, 2)                     # [n_qh, rows, hd]
        ka = k[a, :, :nk].repeat_interleave(G, 0)          # [n_qh, nk, hd]
        va = v[a, :, :nk].repeat_interleave(G, 0)
        pos = torch.arange(r1 - r0) + int(lens[a])
        mask = torch.arange(nk)[None, :] <= pos[:, None]  # row j sees keys 0..lens+j
        o = F.scaled_dot_product_attention(qa, ka, va, attn_mask=mask)
        out[r0:r1] = o.permute(1, 0, 2)
    return out.numpy()


@pytest.mark.parametrize("lens,n_rows", [([40, 0, 7, 129], [3, 3, 3, 3]), ([5, 300], [1, 4]),
                                         ([0, 1, 2], [3, 0, 2])])
def test_attn_against_torch_sdpa(orc, lens, n_rows):
    Q, Kc, Vc, lens, ars, cap = _attn_case(lens, n_rows)
    O, B = orc.decode_attn(Q, Kc, Vc, lens, ars, 6, 2, 128, cap)
    ref = _torch_ref(Q, Kc, Vc, lens, ars, 6, 2, 128)
    assert np.allclose(O, ref, rtol=1e-10, atol=1e-12)
    assert (B >= np.abs(O) - 1e-12).all()


def test_attn_single_key_returns_value(orc):
    Q, Kc, Vc, lens, ars, cap = _attn_case([0], [1])
    O, _ = orc.decode_attn(Q, Kc, Vc, lens, ars, 6, 2, 128, cap)
    for h in range(6):
        assert np.array_equal(O[0, h], _f64(Vc[0, h // 3, 0]))


def test_attn_identical_keys_average_values(orc):
    Q, Kc, Vc, lens, ars, cap = _attn_case([9], [1])
    Kc[0, :, :] = Kc[0, :, :1]
    O, _ = orc.decode_attn(Q, Kc, Vc, lens, ars, 6, 2, 128, cap)
    for h in range(6):
        assert np.allclose(O[0, h], _f64(Vc[0, h // 3, :10]).mean(0), rtol=1e-12, atol=1e-14)


def test_attn_dominant_key(orc):
    Q, Kc, Vc, lens, ars, cap = _attn_case([20], [1])
    q = _f64(Q[0, 0])
    # key 7 of kv-head 0 = 64 * q direction -> score ~ 64*|q|^2/sqrt(128) >> others
    Kc[0, 0, 7] = synth.bf16_bits_np((q * 64).astype(np.float32))
    O, _ = orc.decode_attn(Q, Kc, Vc, lens, ars, 6, 2, 128, cap)
    assert np.allclose(O[0, 0], _f64(Vc[0, 0, 7]), atol=1e-6)


def test_attn_head_permutation_within_group(orc):
    Q, Kc, Vc, lens, ars, cap = _attn_case([33, 4], [3, 2])
    O, _ = orc.decode_attn(Q, Kc, Vc, lens, ars, 6, 2, 128, cap)
    perm = [2, 0, 1, 5, 3, 4]  # permute within each group of 3 q-heads
    O2, _ = orc.decode_attn(np.ascontiguousarray(Q[:, perm]), Kc, Vc, lens, ars, 6, 2, 128, cap)
    assert np.array_equal(O2, O[:, perm])


def test_attn_draft_rows_equal_sequential_decoding(orc):
    Q, Kc, Vc, lens, ars, cap = _attn_case([50], [3])
    O, _ = orc.decode_attn(Q, Kc, Vc, lens, ars, 6, 2, 128, cap)
    for j in range(3):
        Oj, _ = orc.decode_attn(np.ascontiguousarray(Q[j:j + 1]), Kc, Vc, np.array([50 + j], np.int32),
                                np.array([0, 1], np.int32), 6, 2, 128, cap)
        assert np.array_equal(Oj[0], O[j])


def test_rmsnorm_against_torch(orc):
    g = np.random.default_rng(1)
    h = g.standard_normal((5, 384)) * np.array([[1e-3], [1.0], [7.0], [300.0], [1e-9]])
    out = orc.rmsnorm_bf16(h, 1e-6)
    ref = F.rms_norm(torch.from_numpy(h), (384,), eps=1e-6).numpy()
    assert np.array_equal(out, orc.f64_array_to_bf16(ref))


def test_rmsnorm_constant_row_closed_form(orc):
    for c in (0.5, -3.0, 1e-4):
        out = orc.rmsnorm_bf16(np.full((1, 64), c), 1e-6)
        assert (out == orc.double_to_bf16(c / np.sqrt(c * c + 1e-6))).all()


def test_silu_mul_against_torch(orc):
    g = np.random.default_rng(2)
    a = g.standard_normal(4000) * 6
    b = g.standard_normal(4000) * 3
    out = orc.silu_mul_bf16(a, b)
    ref = (F.silu(torch.from_numpy(a)) * torch.from_numpy(b)).numpy()
    got = orc.bf16_array_to_f64(out)
    # torch's silu may differ from the exact value by an ulp of fp64, which can
    # move a value across a bf16 rounding boundary only when it lies on one
    exact_bf16 = orc.bf16_array_to_f64(orc.f64_array_to_bf16(ref))
    assert (got == exact_bf16).mean() > 0.9999
    assert np.allclose(got, ref, rtol=2.0 ** -8, atol=0)
    assert orc.silu_mul_bf16(np.zeros(3), np.ones(3)).tolist() == [0, 0, 0]


def test_pack_rows_hand_example(orc):
    gd = golden("pack_rows.json")
    H = 16
    rows = [synth.bf16_normal_np(SEED, 40 + a, (n, H)) for a, n in enumerate(gd["n_rows"])]
    X, ra, rp, ars = orc.pack_rows(rows, gd["lens"], H)
    assert ra.tolist() == gd["row_agent"] and rp.tolist() == gd["row_pos"]
    assert ars.tolist() == gd["agent_row_start"]
    assert np.array_equal(X, np.concatenate([r for r in rows if len(r)]))


def test_decode_layer_against_library_composition(orc):
    """One layer of the stack versus the same definition composed from library
    routines: gguf dequantisation + numpy matmul, torch rms_norm, torch SDPA,
    torch silu; bf16 rounding points via torch float64 -> float32 -> bf16 is
    avoided by rounding with the separately pinned converter."""
    gguf = pytest.importorskip("gguf")
    from gguf import quants
    H, I, n_qh, n_kvh, hd = 256, 512, 4, 2, 128
    nq, nkv = n_qh * hd, n_kvh * hd
    lens = np.array([6, 0, 11], np.int32)
    ars = np.array([0, 3, 5, 6], np.int32)
    M, A = 6, 3
    cap = 20
    Wqkv = synth.q4k_matrix_np(SEED, 50, nq + 2 * nkv, H)
    Wo = synth.q4k_matrix_np(SEED, 51, H, nq)
    Wgu = synth.q4k_matrix_np(SEED, 52, 2 * I, H)
    Wd = synth.q6k_matrix_np(SEED, 53, H, I)
    Kc = synth.bf16_normal_np(SEED, 54, (A, n_kvh, cap, hd))
    Vc = synth.bf16_normal_np(SEED, 55, (A, n_kvh, cap, hd))
    h0 = orc.bf16_array_to_f64(synth.bf16_normal_np(SEED, 56, (M, H)))
    h = h0.copy()
    Kc1, Vc1 = Kc.copy(), Vc.copy()
    inter = orc.decode_layer(Wqkv, Wo, Wgu, Wd, H, I, n_qh, n_kvh, hd, h, ars, lens, Kc1, Vc1, cap, want=True)

    def dq(W, N, K, t, bs):
        return quants.dequantize(W.reshape(-1, bs), t).astype(np.float64).reshape(N, K)
    T4, T6 = gguf.GGMLQuantizationType.Q4_K, gguf.GGMLQuantizationType.Q6_K
    wqkv, wo = dq(Wqkv, nq + 2 * nkv, H, T4, 144), dq(Wo, H, nq, T4, 144)
    wgu, wd = dq(Wgu, 2 * I, H, T4, 144), dq(Wd, H, I, T6, 210)
    rnd = lambda a: orc.bf16_array_to_f64(orc.f64_array_to_bf16(a))  # noqa: E731

    # each stage starts from the oracle's own previous intermediate (teacher forcing),
    # so a rounding flip can't propagate; each stage is then an independent restatement
    x1 = rnd(F.rms_norm(torch.from_numpy(h0), (H,), eps=1e-6).numpy())
    assert np.array_equal(x1, orc.bf16_array_to_f64(inter["x1"]))
    qkv = x1 @ wqkv.T
    lib_tol = lambda x, w: 8 * 2.0 ** -23 * (np.abs(x) @ np.abs(w).T) + 1e-12  # noqa: E731
    assert (np.abs(inter["qkv"] - qkv) <= lib_tol(x1, wqkv)).all()
    for r in range(M):
        a = int(np.searchsorted(ars, r, side="right") - 1)
        pos = lens[a] + r - ars[a]
        kv = orc.f64_array_to_bf16(inter["qkv"][r, nq:])
        assert np.array_equal(Kc1[a, :, pos].reshape(-1), kv[:nkv])
        assert np.array_equal(Vc1[a, :, pos].reshape(-1), kv[nkv:])
    Qb = orc.f64_array_to_bf16(inter["qkv"][:, :nq]).reshape(M, n_qh, hd)
    o = _torch_ref(Qb, Kc1, Vc1, lens, ars, n_qh, n_kvh, hd).reshape(M, nq)
    assert np.abs(orc.bf16_array_to_f64(inter["attn"]) - o).max() <= 2.0 ** -8 * np.abs(o).max()
    hmid = h0 + orc.bf16_array_to_f64(inter["attn"]) @ wo.T
    assert (np.abs(inter["hmid"] - hmid) <= lib_tol(orc.bf16_array_to_f64(inter["attn"]), wo) + 1e-9).all()
    x2 = rnd(F.rms_norm(torch.from_numpy(inter["hmid"]), (H,), eps=1e-6).numpy())
    assert np.array_equal(x2, orc.bf16_array_to_f64(inter["x2"]))
    gu = x2 @ wgu.T
    assert (np.abs(inter["gu"] - gu) <= lib_tol(x2, wgu)).all()
    act = (F.silu(torch.from_numpy(inter["gu"][:, :I])) * torch.from_numpy(inter["gu"][:, I:])).numpy()
    assert np.abs(orc.bf16_array_to_f64(inter["act"]) - act).max() <= 2.0 ** -8 * np.abs(act).max()
    hout = inter["hmid"] + orc.bf16_array_to_f64(inter["act"]) @ wd.T
    assert (np.abs(h - hout) <= lib_tol(orc.bf16_array_to_f64(inter["act"]), wd) + 1e-9).all()
