"""Guard regions around every buffer an entry point writes.

Stand-in for a memory checker (none runs on this GPU pool): each output,
workspace and cache buffer is carved out of a larger allocation whose guard
bands before and after hold a byte pattern; after the call (and a device
synchronisation) the bands must be unchanged, so a write past either end of any
buffer fails the test. Shapes are ragged on purpose (N, K, row counts and
cached lengths that end inside tiles, chunks and splits).
"""
import numpy as np
import pytest
import torch

import synth
from conftest import SEED

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side (a multiple of 256: interiors keep the workspace alignment)
PATTERN = 0xA5


@pytest.fixture(scope="module")
def q():
    import quantized_agent_decode_b200 as q
    from quantized_agent_decode_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return q


class Guarded:
    """A tensor of the given shape and dtype inside guard bands of PATTERN bytes."""

    def __init__(self, shape, dtype, fill=None):
        esize = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(shape)) * esize
        self.n = (n + 255) // 256 * 256
        self.raw = torch.full((GUARD + self.n + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(*shape)
        if fill is not None:
            self.t.copy_(fill)

    def intact(self):
        torch.cuda.synchronize()
        host = self.raw.cpu().numpy()
        return bool((host[:GUARD] == PATTERN).all() and (host[GUARD + self.n:] == PATTERN).all())


def _bf16(t):
    return t.to(torch.bfloat16)


@pytest.mark.parametrize("fmt,N,K,M", [(4, 300, 1280, 5), (4, 1000, 5120, 16), (6, 260, 2304, 7), (6, 129, 256, 1)])
def test_skinny_gemm_writes_stay_inside(q, fmt, N, K, M):
    g = synth.torch_gen(SEED, "cuda", 500 + N)
    W = (synth.q4k_matrix_torch if fmt == 4 else synth.q6k_matrix_torch)(g, N, K, "cuda")
    if fmt == 6:
        W = q.q6k_pack(W, N, K)
    X = synth.bf16_normal_torch(g, (M, K), "cuda")
    Y = Guarded((M, N), torch.float32)
    ws = Guarded((q.gemm_ws_bytes(K, M),), torch.uint8)
    (q.q4k_gemm if fmt == 4 else q.q6k_gemm)(W, N, K, X, M, Y.t, ws=ws.t)
    assert Y.intact() and ws.intact()
    assert q.device_status() == 0


@pytest.mark.parametrize("fmt,N,K,M", [(4, 300, 1280, 77), (6, 260, 2304, 130),
                                       (6, 2000, 6656, 290)])  # last round split (zeroing + atomic adds)
def test_dense_gemm_writes_stay_inside(q, fmt, N, K, M):
    g = synth.torch_gen(SEED, "cuda", 600 + N)
    W = (synth.q4k_matrix_torch if fmt == 4 else synth.q6k_matrix_torch)(g, N, K, "cuda")
    if fmt == 6:
        W = q.q6k_pack(W, N, K)
    X = synth.bf16_normal_torch(g, (M, K), "cuda")
    Y = Guarded((M, N), torch.float32)
    ws = Guarded((q.dense_gemm_ws_bytes(K, M),), torch.uint8)
    (q.q4k_gemm_dense if fmt == 4 else q.q6k_gemm_dense)(W, N, K, X, M, Y.t, ws=ws.t)
    assert Y.intact() and ws.intact()
    assert q.dense_status() == 0


def test_decode_attention_writes_stay_inside(q):
    A, n_qh, n_kvh, hd = 3, 16, 2, 128
    rows, lens = [3, 1, 2], [130, 0, 777]
    cap = max(l + r for l, r in zip(lens, rows)) + 5
    M = sum(rows)
    g = synth.torch_gen(SEED, "cuda", 700)
    ars = torch.tensor(np.concatenate([[0], np.cumsum(rows)]), dtype=torch.int32, device="cuda")
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    Kc = Guarded((A, n_kvh, cap, hd), torch.bfloat16, synth.bf16_normal_torch(g, (A, n_kvh, cap, hd), "cuda"))
    Vc = Guarded((A, n_kvh, cap, hd), torch.bfloat16, synth.bf16_normal_torch(g, (A, n_kvh, cap, hd), "cuda"))
    Q = synth.bf16_normal_torch(g, (M, n_qh, hd), "cuda")
    O = Guarded((M, n_qh, hd), torch.bfloat16)
    ws = Guarded((q.decode_attn_ws_bytes(A, n_qh, n_kvh, cap, max(rows)),), torch.uint8)
    q.decode_attn(Q, Kc.t, Vc.t, ln, ars, A, max(rows), cap, n_qh, n_kvh, hd, O.t, ws=ws.t)
    assert O.intact() and ws.intact() and Kc.intact() and Vc.intact()


def test_prefill_attention_writes_stay_inside(q):
    n_qh, n_kvh, hd, len_, C = 16, 2, 128, 333, 130
    cap = len_ + C + 3
    g = synth.torch_gen(SEED, "cuda", 800)
    Kc = Guarded((n_kvh, cap, hd), torch.bfloat16, synth.bf16_normal_torch(g, (n_kvh, cap, hd), "cuda"))
    Vc = Guarded((n_kvh, cap, hd), torch.bfloat16, synth.bf16_normal_torch(g, (n_kvh, cap, hd), "cuda"))
    Q = synth.bf16_normal_torch(g, (C, n_qh, hd), "cuda")
    O = Guarded((C, n_qh, hd), torch.bfloat16)
    q.prefill_attn(Q, Kc.t, Vc.t, len_, C, cap, n_qh, n_kvh, hd, O.t)
    assert O.intact() and Kc.intact() and Vc.intact()
    assert q.prefill_status() == 0


def _guarded_model(q, L, H, I, n_qh, n_kvh, A, cap, seed):
    g = synth.torch_gen(SEED, "cuda", seed)
    nq, nkv = n_qh * 128, n_kvh * 128
    ws, caches = [], []
    for _ in range(L):
        ws.append(dict(
            qkv=torch.cat([synth.q4k_matrix_torch(g, nq, H, "cuda"), synth.q4k_matrix_torch(g, nkv, H, "cuda"),
                           synth.q4k_matrix_torch(g, nkv, H, "cuda")]),
            o=synth.q4k_matrix_torch(g, H, nq, "cuda"),
            gu=torch.cat([synth.q4k_matrix_torch(g, I, H, "cuda"), synth.q4k_matrix_torch(g, I, H, "cuda")]),
            down=q.q6k_pack(synth.q6k_matrix_torch(g, H, I, "cuda"), H, I)))
        caches.append((Guarded((A, n_kvh, cap, 128), torch.bfloat16, synth.bf16_normal_torch(g, (A, n_kvh, cap, 128), "cuda")),
                       Guarded((A, n_kvh, cap, 128), torch.bfloat16, synth.bf16_normal_torch(g, (A, n_kvh, cap, 128), "cuda"))))
    model = q.Model(hidden=H, inter=I, n_qh=n_qh, n_kvh=n_kvh, head_dim=128, max_agents=A, kv_cap=cap,
                    w_qkv=[w["qkv"] for w in ws], w_o=[w["o"] for w in ws], w_gu=[w["gu"] for w in ws],
                    w_down=[w["down"] for w in ws], k_cache=[c[0].t for c in caches],
                    v_cache=[c[1].t for c in caches])
    return model, caches, g


def test_decode_step_writes_stay_inside(q):
    H, I, n_qh, n_kvh, A = 512, 1024, 8, 2, 3
    rows, lens = [3, 2, 1], [40, 0, 260]
    cap = max(l + r for l, r in zip(lens, rows)) + 3
    model, caches, g = _guarded_model(q, 2, H, I, n_qh, n_kvh, A, cap, 900)
    M = sum(rows)
    X = synth.bf16_normal_torch(g, (M, H), "cuda")
    ars = torch.tensor(np.concatenate([[0], np.cumsum(rows)]), dtype=torch.int32, device="cuda")
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    Hout = Guarded((M, H), torch.float32)
    ws = Guarded((model.ws_bytes(M),), torch.uint8)
    model.decode_step(X, M, ars, A, max(rows), ln, Hout.t, ws.t)
    assert Hout.intact() and ws.intact()
    assert all(k.intact() and v.intact() for k, v in caches)
    assert q.device_status() == 0


def test_mixed_step_writes_stay_inside(q):
    H, I, n_qh, n_kvh, A = 512, 1024, 8, 2, 3
    rows, lens, C = [3, 2, 0], [40, 9, 17], 150
    cap = max(lens[2] + C, max(l + r for l, r in zip(lens, rows))) + 3
    model, caches, g = _guarded_model(q, 2, H, I, n_qh, n_kvh, A, cap, 950)
    M = sum(rows)
    X = synth.bf16_normal_torch(g, (M + C, H), "cuda")
    ars = torch.tensor(np.concatenate([[0], np.cumsum(rows)]), dtype=torch.int32, device="cuda")
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    Hout = Guarded((M + C, H), torch.float32)
    ws = Guarded((model.mixed_ws_bytes(M, C),), torch.uint8)
    model.mixed_step(X, M, ars, A, max(rows), ln, 2, lens[2], C, Hout.t, ws.t)
    assert Hout.intact() and ws.intact()
    assert all(k.intact() and v.intact() for k, v in caches)
    assert q.device_status() == 0 and q.dense_status() == 0


def test_verify_step_writes_stay_inside(q):
    H, vocab, A = 512, 3001, 2
    rows = [3, 2]
    M = sum(rows)
    g = synth.torch_gen(SEED, "cuda", 990)
    Wh = synth.q4k_matrix_torch(g, vocab, H, "cuda")
    Hd = synth.bf16_normal_torch(g, (M, H), "cuda").float()
    ars = torch.tensor(np.concatenate([[0], np.cumsum(rows)]), dtype=torch.int32, device="cuda")
    toks = torch.randint(0, vocab, (M,), generator=g, dtype=torch.int32, device="cuda")
    lens = Guarded((A,), torch.int32, torch.tensor([10, 20], dtype=torch.int32))
    out = Guarded((M,), torch.int32)
    acc = Guarded((A,), torch.int32)
    amax = Guarded((M,), torch.int32)
    logits = Guarded((M, vocab), torch.float32)
    ws = Guarded((q.verify_ws_bytes(H, vocab, M),), torch.uint8)
    q.verify_step(Hd, M, H, Wh, vocab, ars, A, toks, lens.t, out.t, acc.t, row_argmax=amax.t, logits=logits.t,
                  ws=ws.t)
    assert all(b.intact() for b in (lens, out, acc, amax, logits, ws))
