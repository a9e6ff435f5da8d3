"""GPU parity of the whole decode-and-verify step through the C ABI.

Teacher-forced per layer: every fused stage of the GPU step (RMSNorm -> qkv
GEMM -> k/v append -> attention -> o GEMM + residual -> RMSNorm -> gate|up
GEMM -> silu*up -> down GEMM + residual) is checked against the fp64 oracle
fed with the GPU's own input to that stage (read from the debug buffer), so a
legitimate rounding difference upstream cannot propagate. Tolerances: GEMMs
1e-3 * sum|w x| per output (plus fp32 rounding of the residual add),
attention 2e-3 * sum p|v| plus half a bf16 ulp, bf16 rounding points exact
except for values within the fp32/fp64 disagreement of a rounding tie (at most
one bf16 ulp, in a small fraction of elements).
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


def a256(x):
    return (x + 255) // 256 * 256


def dbg_views(buf, layer, M, H, I, nq, nqkv):
    """Slices of one layer's debug record (layout documented in include/qad.h)."""
    sizes = [("x1", M * H * 2), ("qkv", M * nqkv * 4), ("attn", M * nq * 2), ("hmid", M * H * 4),
             ("x2", M * H * 2), ("gu", M * 2 * I * 4), ("act", M * I * 2), ("hout", M * H * 4)]
    per = sum(a256(s) for _, s in sizes)
    raw = buf[layer * per:(layer + 1) * per].cpu().numpy()
    out, off = {}, 0
    shapes = {"x1": (M, H), "qkv": (M, nqkv), "attn": (M, nq), "hmid": (M, H), "x2": (M, H), "gu": (M, 2 * I),
              "act": (M, I), "hout": (M, H)}
    for name, s in sizes:
        seg = raw[off:off + s]
        dt = np.uint16 if name in ("x1", "attn", "x2", "act") else np.float32
        out[name] = seg.view(dt).reshape(shapes[name])
        off += a256(s)
    return out


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_close(gpu_bits, ref_bits, orc, frac=1e-3):
    """Equal except for at most `frac` of elements that differ by one bf16 ulp."""
    g = orc.bf16_array_to_f64(gpu_bits)
    r = orc.bf16_array_to_f64(ref_bits)
    diff = g != r
    if diff.mean() > frac:
        return False
    ulp = np.abs(r) * 2.0 ** -7 + 1e-38
    return bool((np.abs(g - r)[diff] <= ulp[diff] * 1.01).all())


class Stack:
    """A small synthetic stack with ragged agents, built on the GPU from host arrays."""

    def __init__(self, q, n_layers, H, I, n_qh, n_kvh, n_rows, lens, seed, extra_cap=4, kv="bf16", orc=None):
        self.q = q
        self.kv = kv
        self.L, self.H, self.I, self.n_qh, self.n_kvh = n_layers, H, I, n_qh, n_kvh
        hd = 128
        self.nq, self.nkv = n_qh * hd, n_kvh * hd
        self.nqkv = self.nq + 2 * self.nkv
        self.A = len(lens)
        self.cap = max(l + n for l, n in zip(lens, n_rows)) + extra_cap
        self.ars = np.concatenate([[0], np.cumsum(n_rows)]).astype(np.int32)
        self.M = int(self.ars[-1])
        self.lens = np.array(lens, np.int32)
        self.max_rows = int(max(n_rows))
        self.W = []
        for l in range(n_layers):
            t = 100 * l + seed
            self.W.append(dict(
                qkv=np.concatenate([synth.q4k_matrix_np(SEED, t + 1, self.nq, H),
                                    synth.q4k_matrix_np(SEED, t + 2, self.nkv, H),
                                    synth.q4k_matrix_np(SEED, t + 3, self.nkv, H)]),
                o=synth.q4k_matrix_np(SEED, t + 4, H, self.nq),
                gu=np.concatenate([synth.q4k_matrix_np(SEED, t + 5, I, H), synth.q4k_matrix_np(SEED, t + 6, I, H)]),
                down=synth.q6k_matrix_np(SEED, t + 7, H, I),
                kc=synth.bf16_normal_np(SEED, t + 8, (self.A, n_kvh, self.cap, hd)),
                vc=synth.bf16_normal_np(SEED, t + 9, (self.A, n_kvh, self.cap, hd))))
            if kv == "q8_0":  # the cached rows: q8_0 of N(0,1) values (the oracle's quantiser)
                w = self.W[-1]
                for name in ("kc", "vc"):
                    w[name + "8"] = orc.q8_0_quantize(orc.bf16_array_to_f64(w[name]).astype(np.float32))
        self.X = synth.bf16_normal_np(SEED, seed + 7777, (self.M, H))
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
        bdev = lambda a: dev(a.view(np.int16)).view(torch.bfloat16)  # noqa: E731
        self.d = dict(qkv=[dev(w["qkv"]) for w in self.W], o=[dev(w["o"]) for w in self.W],
                      gu=[dev(w["gu"]) for w in self.W],
                      down=[q.q6k_pack(dev(w["down"]), H, I) for w in self.W])
        if kv == "q8_0":
            nbytes = q.kv_cache_bytes(q.KV_Q8_0, self.A, n_kvh, self.cap)
            self.d["kc"] = [torch.zeros(nbytes, dtype=torch.uint8, device="cuda") for _ in self.W]
            self.d["vc"] = [torch.zeros(nbytes, dtype=torch.uint8, device="cuda") for _ in self.W]
            self.reset_caches()
        else:
            self.d["kc"] = [bdev(w["kc"]) for w in self.W]
            self.d["vc"] = [bdev(w["vc"]) for w in self.W]
        self.model = q.Model(hidden=H, inter=I, n_qh=n_qh, n_kvh=n_kvh, head_dim=hd, max_agents=self.A,
                             kv_cap=self.cap, w_qkv=self.d["qkv"], w_o=self.d["o"], w_gu=self.d["gu"],
                             w_down=self.d["down"], k_cache=self.d["kc"], v_cache=self.d["vc"],
                             kv_format=q.KV_Q8_0 if kv == "q8_0" else q.KV_BF16)
        self.Xd = bdev(self.X)
        self.arsd = dev(self.ars)
        self.lensd = dev(self.lens)
        self.Hd = torch.empty(self.M, H, dtype=torch.float32, device="cuda")
        self.ws = q.alloc_ws(self.model.ws_bytes(self.M))

    def planes(self, l):
        """Host copies (Kq, Kd, Vq, Vd) of layer l's q8_0 caches."""
        out = []
        for buf in (self.d["kc"][l], self.d["vc"][l]):
            codes, scales = self.q.q8_cache_planes(buf, self.A, self.n_kvh, self.cap)
            out += [codes.cpu().numpy(), scales.cpu().numpy().view(np.uint16)]
        return out

    def reset_caches(self):
        for l in range(self.L):
            if self.kv == "q8_0":
                for name in ("kc", "vc"):
                    codes, scales = self.q.q8_cache_planes(self.d[name][l], self.A, self.n_kvh, self.cap)
                    qn, dn = self.W[l][name + "8"]
                    codes.copy_(torch.from_numpy(qn))
                    scales.copy_(torch.from_numpy(dn.view(np.int16)))
                continue
            self.d["kc"][l].copy_(torch.from_numpy(self.W[l]["kc"].view(np.int16)).view(torch.bfloat16))
            self.d["vc"][l].copy_(torch.from_numpy(self.W[l]["vc"].view(np.int16)).view(torch.bfloat16))

    def run(self, debug=True):
        dbg = self.model.set_debug(self.M) if debug else None
        self.model.decode_step(self.Xd, self.M, self.arsd, self.A, self.max_rows, self.lensd, self.Hd, self.ws)
        torch.cuda.synchronize()
        return dbg


def check_layer(st, orc, dbg, l, h_in, kc_after, vc_after, rows=None, q8=None):
    """Teacher-forced checks of layer l. h_in: the layer's fp32 input (GPU values).
    rows: optional subset of output rows for the GEMM checks (full size).
    q8: (Kq, Kd, Vq, Vd) host copies of a q8_0 cache after the step (kc/vc unused)."""
    v = dbg_views(dbg, l, st.M, st.H, st.I, st.nq, st.nqkv)
    W = st.W[l] if isinstance(st.W[l], dict) else st.W[l]()
    # x1 = bf16(rmsnorm(h))
    assert bf16_close(v["x1"], orc.rmsnorm_bf16(h_in.astype(np.float64)), orc)

    def gemm_check(fmt, Wm, N, K, Xb, Y_gpu, base=None):
        sel = np.arange(N) if rows is None else np.asarray(rows(N), np.int32)
        Yr, A = orc.gemm_rows(fmt, Wm, K, sel, Xb)
        ref = Yr if base is None else base[:, sel] + Yr
        slack = 0 if base is None else 8 * 2.0 ** -24 * (np.abs(base[:, sel]) + np.abs(Yr))
        err = np.abs(Y_gpu[:, sel].astype(np.float64) - ref)
        ratio = err / (1e-3 * A + slack + 1e-30)
        assert ratio.max() <= 1.0, ratio.max()

    gemm_check(4, W["qkv"], st.nqkv, st.H, v["x1"], v["qkv"])
    if q8 is not None:
        # k, v appended as q8_0 of the fp32 projection, bit-exact (same fp32 decisions)
        Kq, Kd, Vq, Vd = q8
        for r in range(st.M):
            a = int(np.searchsorted(st.ars, r, side="right") - 1)
            pos = st.lens[a] + r - st.ars[a]
            kq, kd = orc.q8_0_quantize(v["qkv"][r, st.nq:st.nq + st.nkv].reshape(st.n_kvh, 128))
            vq, vd = orc.q8_0_quantize(v["qkv"][r, st.nq + st.nkv:].reshape(st.n_kvh, 128))
            assert np.array_equal(Kq[a, :, pos], kq) and np.array_equal(Kd[a, :, pos], kd)
            assert np.array_equal(Vq[a, :, pos], vq) and np.array_equal(Vd[a, :, pos], vd)
        Qb = orc.f64_array_to_bf16(v["qkv"][:, :st.nq].astype(np.float64)).reshape(st.M, st.n_qh, 128)
        O_ref, B = orc.decode_attn_q8(Qb, Kq, Kd, Vq, Vd, st.lens, st.ars, st.n_qh, st.n_kvh, 128, st.cap)
        o = orc.bf16_array_to_f64(v["attn"]).reshape(O_ref.shape)
        # fp16 V and P leave the fp32 result within 2e-3 * B; bf16 output: half an ulp (2^-8 relative) more
        assert (np.abs(o - O_ref) <= 2e-3 * B + np.abs(O_ref) * 2.0 ** -8 + 1e-30).all()
        return _check_after_attn(st, orc, v, W, h_in, gemm_check)
    # k, v appended as bf16 of the fp32 projection, exactly
    kvb = orc.f64_array_to_bf16(v["qkv"][:, st.nq:].astype(np.float64)) if rows is None else None
    for r in range(st.M):
        a = int(np.searchsorted(st.ars, r, side="right") - 1)
        pos = st.lens[a] + r - st.ars[a]
        krow = kc_after[a, :, pos].reshape(-1)
        vrow = vc_after[a, :, pos].reshape(-1)
        if kvb is not None:
            assert np.array_equal(krow, kvb[r, :st.nkv]) and np.array_equal(vrow, kvb[r, st.nkv:])
        else:
            ref = orc.f64_array_to_bf16(v["qkv"][r, st.nq:st.nq + 256].astype(np.float64))
            assert np.array_equal(krow[:256], ref)
    # attention on the GPU's Q and caches
    Qb = orc.f64_array_to_bf16(v["qkv"][:, :st.nq].astype(np.float64)).reshape(st.M, st.n_qh, 128)
    O_ref, B = orc.decode_attn(Qb, kc_after, vc_after, st.lens, st.ars, st.n_qh, st.n_kvh, 128, st.cap)
    o = orc.bf16_array_to_f64(v["attn"]).reshape(O_ref.shape)
    assert (np.abs(o - O_ref) <= 2e-3 * B + np.abs(O_ref) * 2.0 ** -9 + 1e-30).all()
    return _check_after_attn(st, orc, v, W, h_in, gemm_check)


def _check_after_attn(st, orc, v, W, h_in, gemm_check):
    # h += O Wo^T
    gemm_check(4, W["o"], st.H, st.nq, v["attn"], v["hmid"], base=h_in.astype(np.float64))
    # x2, gate|up
    assert bf16_close(v["x2"], orc.rmsnorm_bf16(v["hmid"].astype(np.float64)), orc)
    gemm_check(4, W["gu"], 2 * st.I, st.H, v["x2"], v["gu"])
    # act = bf16(silu(gate) * up)
    gu = v["gu"].astype(np.float64)
    assert bf16_close(v["act"], orc.silu_mul_bf16(gu[:, :st.I], gu[:, st.I:]), orc, frac=5e-3)
    # h += act Wdown^T
    gemm_check(6, W["down"], st.H, st.I, v["act"], v["hout"], base=v["hmid"].astype(np.float64))
    return v["hout"]


@pytest.mark.parametrize("n_rows,lens", [([3, 1, 2], [40, 0, 7]), ([3, 3, 3, 3], [5, 17, 33, 2]),
                                         ([16], [3]), ([0, 2, 3], [9, 0, 130])])
def test_step_teacher_forced_small_stack(q, orc, n_rows, lens):
    st = Stack(q, 2, 512, 1024, 8, 2, n_rows, lens, seed=len(n_rows))
    dbg = st.run()
    kc = [_bits(t).reshape(st.W[l]["kc"].shape) for l, t in enumerate(st.d["kc"])]
    vc = [_bits(t).reshape(st.W[l]["vc"].shape) for l, t in enumerate(st.d["vc"])]
    h = orc.bf16_array_to_f64(st.X).astype(np.float32)
    for l in range(st.L):
        h = check_layer(st, orc, dbg, l, h, kc[l], vc[l])
    assert np.array_equal(h, st.Hd.cpu().numpy())
    assert q.device_status() == 0


@pytest.mark.parametrize("n_rows,lens", [([3, 1, 2], [40, 0, 7]), ([3, 3, 3, 3], [5, 17, 33, 2]),
                                         ([0, 2, 3], [9, 0, 130])])
def test_step_q8_0_cache_teacher_forced(q, orc, n_rows, lens):
    """The same step over q8_0 caches: appended codes bit-exact, attention within
    the attention tolerance of the oracle over the GPU's caches."""
    st = Stack(q, 2, 512, 1024, 8, 2, n_rows, lens, seed=20 + len(n_rows), kv="q8_0", orc=orc)
    dbg = st.run()
    h = orc.bf16_array_to_f64(st.X).astype(np.float32)
    for l in range(st.L):
        h = check_layer(st, orc, dbg, l, h, None, None, q8=st.planes(l))
    assert np.array_equal(h, st.Hd.cpu().numpy())
    assert q.device_status() == 0


def test_step_graph_and_host_paths_match_eager(q, orc):
    st = Stack(q, 2, 512, 1024, 8, 2, [3, 3, 3, 3], [11, 0, 5, 64], seed=9)
    st.run(debug=False)
    ref = st.Hd.cpu().numpy().copy()
    st.model.set_debug(None)
    stream = torch.cuda.Stream()
    st.reset_caches()
    g = st.model.graph(st.Xd, st.M, st.arsd, st.A, st.max_rows, st.lensd, st.Hd, st.ws, stream)
    st.Hd.zero_()
    for _ in range(3):  # replays rewrite the same cache slots (rollback by overwrite)
        g.launch(stream)
    stream.synchronize()
    got = st.Hd.cpu().numpy()
    scale = np.abs(ref).max()
    assert np.allclose(got, ref, rtol=1e-4, atol=1e-5 * scale)
    g.close()
    Xh = torch.from_numpy(st.X.view(np.int16)).view(torch.bfloat16).pin_memory()
    Hh = torch.empty(st.M, st.H, dtype=torch.float32).pin_memory()
    st.model.decode_step_host(Xh, st.M, torch.from_numpy(st.ars).pin_memory(), st.A, st.max_rows,
                              torch.from_numpy(st.lens).pin_memory(), Hh, st.ws, stream)
    assert np.allclose(Hh.numpy(), ref, rtol=1e-4, atol=1e-5 * scale)
    assert q.device_status() == 0


def test_step_rejects_bad_arguments(q):
    st = Stack(q, 1, 256, 512, 4, 2, [2], [3], seed=3)
    with pytest.raises(q.QadError):
        st.model.decode_step(st.Xd, 17, st.arsd, st.A, 2, st.lensd, st.Hd, st.ws)
    with pytest.raises(q.QadError):  # workspace too small
        st.model.decode_step(st.Xd, st.M, st.arsd, st.A, 2, st.lensd, st.Hd, st.ws[:256])
    with pytest.raises(q.QadError):  # more agents than the model holds
        st.model.decode_step(st.Xd, st.M, st.arsd, st.A + 1, 2, st.lensd, st.Hd, st.ws)


def _full_stack_check(q, orc, workload, layers_to_check, n_rows_checked=96):
    import bench
    w = bench.Workload(workload)
    rng = np.random.default_rng(0)

    class View:  # adapter: the oracle side of check_layer reads host copies on demand
        pass
    st = View()
    sh = w.shape
    st.M, st.H, st.I, st.n_qh, st.n_kvh = w.M, sh.hidden, sh.inter, sh.n_qh, sh.n_kvh
    st.nq, st.nkv = sh.n_qh * 128, sh.n_kvh * 128
    st.nqkv = st.nq + 2 * st.nkv
    st.ars = w.ars.cpu().numpy()
    st.lens = w.lens.cpu().numpy()
    st.cap = w.kv_cap
    st.W = [(lambda l=l: dict(qkv=w.w_qkv[l].cpu().numpy(), o=w.w_o[l].cpu().numpy(),
                              gu=w.w_gu[l].cpu().numpy(), down=w.down_gguf(l).cpu().numpy()))
            for l in range(sh.n_layers)]
    dbg = w.model.set_debug(w.M)
    w.step()
    torch.cuda.synchronize()
    rows = lambda N: np.sort(rng.choice(N, size=min(N, n_rows_checked), replace=False))  # noqa: E731
    for l in layers_to_check:
        if l == 0:
            h_in = orc.bf16_array_to_f64(_bits(w.X)).astype(np.float32)
        else:
            h_in = dbg_views(dbg, l - 1, st.M, st.H, st.I, st.nq, st.nqkv)["hout"]
        kc = _bits(w.kc[l]).reshape(w.kc[l].shape)
        vc = _bits(w.vc[l]).reshape(w.vc[l].shape)
        check_layer(st, orc, dbg, l, h_in, kc, vc, rows=rows)
    last = dbg_views(dbg, sh.n_layers - 1, st.M, st.H, st.I, st.nq, st.nqkv)["hout"]
    assert np.array_equal(last, w.H_out.cpu().numpy())
    assert np.isfinite(last).all()
    assert q.device_status() == 0


def test_full_stack_bench_configuration_sampled(q, orc):
    """The benchmarked configuration (64 layers, 12 rows = 4 agents x 3, 1024-token
    contexts), layers 0, 31 and 63 teacher-forced on sampled GEMM outputs and
    every attention output."""
    _full_stack_check(q, orc, "stack12_ctx1k", [0, 31, 63])


def test_full_stack_23k_context_sampled(q, orc):
    """64 layers with 23000 cached tokens per agent; layers 0 and 63."""
    _full_stack_check(q, orc, "stack12_ctx23k", [0, 63])
