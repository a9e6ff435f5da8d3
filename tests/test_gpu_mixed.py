"""GPU parity of the mixed step (decode rows + one agent's prompt chunk through
the dense tensor-core GEMMs) against the fp64 oracle, teacher-forced per layer.

The oracle's layer is the same definition with the chunk agent holding C rows
at positions chunk_len .. chunk_len + C - 1 (causal, like draft rows).
Tolerances: every GEMM output 1e-3 * sum |w x| (each weight enters the dense
tensor-core product within 2^-11 of its value, see the dense GEMM tests);
attention, decode and chunk rows alike, 2e-3 * sum p|v| plus half a bf16 ulp
(2^-8 relative) of the output; bf16 rounding points equal except for rare
one-ulp flips at rounding ties.
"""
import numpy as np
import pytest
import torch

import synth
from conftest import SEED
from test_gpu_step import Stack, _bits, bf16_close, dbg_views

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import quantized_agent_decode_b200 as q
    from quantized_agent_decode_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return q


def _dense_check(orc, fmt, W, N, K, Xb, Y_gpu, base=None):
    Yr, A = orc.gemm(fmt, W, N, K, Xb)
    ref = Yr if base is None else base + Yr
    slack = 0 if base is None else 8 * 2.0 ** -24 * (np.abs(base) + np.abs(Yr))
    ratio = np.abs(Y_gpu.astype(np.float64) - ref) / (1e-3 * A + slack + 1e-30)
    assert ratio.max() <= 1.0, ratio.max()


@pytest.mark.parametrize("n_rows,lens,C", [([3, 2, 0], [40, 7, 17], 70), ([3, 3, 0], [5, 300, 0], 130),
                                           ([0], [9], 64)])
def test_mixed_step_teacher_forced(q, orc, n_rows, lens, C):
    """The chunk agent is the last one (no decode rows), so the GPU's row order
    (decode rows, then the chunk) is the oracle's agent-major order."""
    st = Stack(q, 2, 512, 1024, 8, 2, n_rows, lens, seed=40 + C, extra_cap=C + 4)
    M = st.M
    ca, clen = st.A - 1, int(lens[-1])
    R = M + C
    Xc = synth.bf16_normal_np(SEED, 9000 + C, (C, st.H))
    Xall = np.concatenate([st.X, Xc]) if M else Xc
    Xd = torch.from_numpy(Xall.view(np.int16)).view(torch.bfloat16).cuda()
    Hd = torch.empty(R, st.H, dtype=torch.float32, device="cuda")
    ws = q.alloc_ws(st.model.mixed_ws_bytes(M, C))
    dbg = st.model.set_debug_mixed(M, C)
    st.model.mixed_step(Xd, M, st.arsd if M else None, st.A, max(st.max_rows, 1), st.lensd if M else None, ca, clen,
                        C, Hd, ws)
    torch.cuda.synchronize()
    ars_o = np.concatenate([st.ars[:-1], [R]]).astype(np.int32)  # the chunk agent's rows are the last C
    h = orc.bf16_array_to_f64(Xall).astype(np.float32)
    for l in range(st.L):
        v = dbg_views(dbg, l, R, st.H, st.I, st.nq, st.nqkv)
        W = st.W[l]
        kc = _bits(st.d["kc"][l]).reshape(W["kc"].shape)
        vc = _bits(st.d["vc"][l]).reshape(W["vc"].shape)
        assert bf16_close(v["x1"], orc.rmsnorm_bf16(h.astype(np.float64)), orc)
        _dense_check(orc, 4, W["qkv"], st.nqkv, st.H, v["x1"], v["qkv"])
        kvb = orc.f64_array_to_bf16(v["qkv"][:, st.nq:].astype(np.float64))
        for r in range(R):
            a = int(np.searchsorted(ars_o, r, side="right") - 1)
            pos = st.lens[a] + r - ars_o[a]
            assert np.array_equal(kc[a, :, pos].reshape(-1), kvb[r, :st.nkv])
            assert np.array_equal(vc[a, :, pos].reshape(-1), kvb[r, st.nkv:])
        Qb = orc.f64_array_to_bf16(v["qkv"][:, :st.nq].astype(np.float64)).reshape(R, st.n_qh, 128)
        O_ref, B = orc.decode_attn(Qb, kc, vc, st.lens, ars_o, st.n_qh, st.n_kvh, 128, st.cap)
        o = orc.bf16_array_to_f64(v["attn"]).reshape(O_ref.shape)
        assert (np.abs(o - O_ref) <= 2e-3 * B + np.abs(O_ref) * 2.0 ** -8 + 1e-30).all()
        _dense_check(orc, 4, W["o"], st.H, st.nq, v["attn"], v["hmid"], base=h.astype(np.float64))
        assert bf16_close(v["x2"], orc.rmsnorm_bf16(v["hmid"].astype(np.float64)), orc)
        _dense_check(orc, 4, W["gu"], 2 * st.I, st.H, v["x2"], v["gu"])
        gu = v["gu"].astype(np.float64)
        assert bf16_close(v["act"], orc.silu_mul_bf16(gu[:, :st.I], gu[:, st.I:]), orc, frac=5e-3)
        _dense_check(orc, 6, W["down"], st.H, st.I, v["act"], v["hout"], base=v["hmid"].astype(np.float64))
        h = v["hout"]
    assert np.array_equal(h, Hd.cpu().numpy())
    assert q.dense_status() == 0 and q.device_status() == 0


def test_mixed_step_rejects_bad_arguments(q):
    st = Stack(q, 1, 256, 512, 4, 2, [2, 0], [3, 5], seed=3, extra_cap=8)
    X = torch.zeros(2 + 8, 256, dtype=torch.bfloat16, device="cuda")
    H = torch.empty(10, 256, dtype=torch.float32, device="cuda")
    ws = q.alloc_ws(st.model.mixed_ws_bytes(2, 8))
    with pytest.raises(q.QadError):  # chunk runs past the cache
        st.model.mixed_step(X, 2, st.arsd, st.A, 2, st.lensd, 1, st.cap - 4, 8, H, ws)
    with pytest.raises(q.QadError):  # no such agent
        st.model.mixed_step(X, 2, st.arsd, st.A, 2, st.lensd, st.A, 0, 8, H, ws)
    with pytest.raises(q.QadError):  # workspace too small
        st.model.mixed_step(X, 2, st.arsd, st.A, 2, st.lensd, 1, 5, 8, H, ws[:1024])


def test_mixed_step_full_stack_2048_chunk_sampled(q, orc):
    """The mixed step at full size: the 64-layer bench stack, agents 0-2 decoding
    3 rows each at 23000 cached tokens and agent 3's 2048-row prompt chunk at
    positions 23000 .. 25047. Layer 0 and the deepest layer whose input is still
    finite (at least layer 32) teacher-forced from the step's own
    intermediates: every x1, x2 and act row, 96 sampled output columns of each
    GEMM, the k/v append of every row, the attention of every decode row and of
    24 sampled chunk rows (one oracle call per row, at its own position)."""
    import bench
    from test_gpu_step import bf16_close, dbg_views
    CTX, C, rpa = 23000, 2048, 3
    w = bench.Workload("stack12_ctx23k", ctx=CTX + C + 4)
    sh = w.shape
    H, I = sh.hidden, sh.inter
    nq, nkv = sh.n_qh * 128, sh.n_kvh * 128
    nqkv = nq + 2 * nkv
    A, M = 4, 3 * rpa
    R = M + C
    rng = np.random.default_rng(7)
    X = synth.bf16_normal_np(SEED, 9300, (R, H))
    Xd = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).cuda()
    ars = np.array([0, 3, 6, 9, 9], np.int32)
    lens = np.array([CTX] * A, np.int32)
    ars_d, lens_d = torch.from_numpy(ars).cuda(), torch.from_numpy(lens).cuda()
    Hd = torch.empty(R, H, dtype=torch.float32, device="cuda")
    ws = q.alloc_ws(w.model.mixed_ws_bytes(M, C))
    dbg = w.model.set_debug_mixed(M, C)
    w.model.mixed_step(Xd, M, ars_d, A, rpa, lens_d, 3, CTX, C, Hd, ws)
    torch.cuda.synchronize()
    assert q.device_status() == 0 and q.dense_status() == 0
    ars_o = np.array([0, 3, 6, 9, R], np.int32)  # agent 3 holds the chunk rows
    cols = lambda N: np.sort(rng.choice(N, size=96, replace=False))  # noqa: E731

    def dense(fmt, Wm, N, K, Xb, Y, base=None):
        sel = cols(N)
        Yr, Aabs = orc.gemm_rows(fmt, Wm, K, sel, Xb)
        ref = Yr if base is None else base[:, sel] + Yr
        slack = 0 if base is None else 8 * 2.0 ** -24 * (np.abs(base[:, sel]) + np.abs(Yr))
        ratio = np.abs(Y[:, sel].astype(np.float64) - ref) / (1e-3 * Aabs + slack + 1e-30)
        assert ratio.max() <= 1.0, ratio.max()

    # The synthetic stack's residual grows layer by layer (random weights); the chunk rows overflow fp32
    # near the last layers. The deep layer checked is the deepest whose input is still finite.
    deep = next(l for l in range(sh.n_layers - 1, 0, -1)
                if np.isfinite(dbg_views(dbg, l - 1, R, H, I, nq, nqkv)["hout"]).all())
    assert deep >= sh.n_layers // 2, deep
    for l in (0, deep):
        v = dbg_views(dbg, l, R, H, I, nq, nqkv)
        if l == 0:
            h_in = orc.bf16_array_to_f64(X).astype(np.float32)
        else:
            h_in = dbg_views(dbg, l - 1, R, H, I, nq, nqkv)["hout"]
        assert bf16_close(v["x1"], orc.rmsnorm_bf16(h_in.astype(np.float64)), orc)
        dense(4, w.w_qkv[l].cpu().numpy(), nqkv, H, v["x1"], v["qkv"])
        kc = _bits(w.kc[l]).reshape(w.kc[l].shape)
        vc = _bits(w.vc[l]).reshape(w.vc[l].shape)
        kvb = orc.f64_array_to_bf16(v["qkv"][:, nq:].astype(np.float64))
        pos = np.concatenate([lens[a] + np.arange(ars_o[a + 1] - ars_o[a]) for a in range(A)])
        agent = np.repeat(np.arange(A), np.diff(ars_o))
        assert np.array_equal(kc[agent, :, pos].reshape(R, -1), kvb[:, :nkv])
        assert np.array_equal(vc[agent, :, pos].reshape(R, -1), kvb[:, nkv:])
        Qb = orc.f64_array_to_bf16(v["qkv"][:, :nq].astype(np.float64)).reshape(R, sh.n_qh, 128)
        o = orc.bf16_array_to_f64(v["attn"]).reshape(R, sh.n_qh, 128)
        O_ref, B = orc.decode_attn(Qb[:M], kc[:3], vc[:3], lens[:3], ars[:4], sh.n_qh, sh.n_kvh, 128, w.kv_cap)
        assert (np.abs(o[:M] - O_ref) <= 2e-3 * B + np.abs(O_ref) * 2.0 ** -8 + 1e-30).all()
        for j in np.sort(rng.choice(C, size=24, replace=False)):
            r = M + int(j)
            O1, B1 = orc.decode_attn(Qb[r:r + 1], kc[3:4], vc[3:4], [CTX + int(j)], [0, 1], sh.n_qh, sh.n_kvh, 128,
                                     w.kv_cap)
            assert (np.abs(o[r:r + 1] - O1) <= 2e-3 * B1 + np.abs(O1) * 2.0 ** -8 + 1e-30).all(), j
        dense(4, w.w_o[l].cpu().numpy(), H, nq, v["attn"], v["hmid"], base=h_in.astype(np.float64))
        assert bf16_close(v["x2"], orc.rmsnorm_bf16(v["hmid"].astype(np.float64)), orc)
        dense(4, w.w_gu[l].cpu().numpy(), 2 * I, H, v["x2"], v["gu"])
        gu = v["gu"].astype(np.float64)
        assert bf16_close(v["act"], orc.silu_mul_bf16(gu[:, :I], gu[:, I:]), orc, frac=5e-3)
        dense(6, w.down_gguf(l).cpu().numpy(), H, I, v["act"], v["hout"], base=v["hmid"].astype(np.float64))
    last = dbg_views(dbg, sh.n_layers - 1, R, H, I, nq, nqkv)["hout"]
    assert np.array_equal(last, Hd.cpu().numpy(), equal_nan=True)
