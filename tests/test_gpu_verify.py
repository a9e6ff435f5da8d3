"""GPU parity of the verify tail: logits through the Q4_K output head, the
per-row argmax, greedy draft acceptance and the KV-length commit.

- logits vs the oracle GEMM on bf16(rmsnorm(H)): |y - y_ref| <= 1e-3 * A;
- the argmax is decided on the kernel's fp32 logits, so it must equal the
  first index of the maximum of those logits exactly, and be a valid argmax
  of the oracle's logits up to the two entries' tolerances;
- acceptance, emitted tokens and the new lengths must equal the oracle's
  greedy rule applied to the GPU's argmaxes, exactly.
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


def _run(q, orc, H, W, hidden, vocab, n_rows, lens, row_tokens, rows=None):
    M = int(sum(n_rows))
    ars = np.concatenate([[0], np.cumsum(n_rows)]).astype(np.int32)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    Hd = dev(H.astype(np.float32))
    Wd = W if isinstance(W, torch.Tensor) else dev(W)
    lens_d = dev(np.array(lens, np.int32))
    out = torch.full((M,), -7, dtype=torch.int32, device="cuda")
    acc = torch.full((len(lens),), -7, dtype=torch.int32, device="cuda")
    amax = torch.full((M,), -7, dtype=torch.int32, device="cuda")
    logits = torch.full((M, vocab), float("nan"), device="cuda")
    q.verify_step(Hd, M, hidden, Wd, vocab, dev(ars), len(lens), dev(np.array(row_tokens, np.int32)), lens_d, out,
                  acc, row_argmax=amax, logits=logits)
    torch.cuda.synchronize()
    Lg = logits.cpu().numpy()
    am = amax.cpu().numpy()
    # argmax decided on the kernel's fp32 logits: first index of the maximum
    assert np.array_equal(am, np.argmax(Lg, axis=1))
    # logits vs the oracle (all vocab rows, or the sampled ones plus every argmax)
    x = orc.rmsnorm_bf16(H.astype(np.float64))
    Wn = W.cpu().numpy() if isinstance(W, torch.Tensor) else W
    if rows is None:
        Yr, A = orc.gemm(4, Wn, vocab, hidden, x)
        sel = np.arange(vocab)
    else:
        sel = np.unique(np.concatenate([rows, am])).astype(np.int32)
        Yr, A = orc.gemm_rows(4, Wn, hidden, sel, x)
    tol = 1e-3 * A
    assert (np.abs(Lg[:, sel] - Yr) <= tol).all(), (np.abs(Lg[:, sel] - Yr) / tol).max()
    if rows is None:
        for r in range(M):
            ref = orc.argmax(Yr[r])
            assert Yr[r, am[r]] >= Yr[r, ref] - tol[r, am[r]] - tol[r, ref]
    # acceptance and commit: the oracle's greedy rule on the GPU's argmaxes
    lens2, out_ref, acc_ref = orc.accept_greedy(am, row_tokens, ars, lens)
    assert out.cpu().numpy().tolist() == out_ref.tolist()
    assert acc.cpu().numpy().tolist() == acc_ref.tolist()
    assert lens_d.cpu().numpy().tolist() == lens2.tolist()
    return am, acc.cpu().numpy()


def test_verify_small_head_all_paths(q, orc):
    hidden, vocab = 512, 1000
    n_rows, lens = [3, 3, 1, 0, 2], [40, 7, 0, 5, 13]
    M = sum(n_rows)
    W = synth.q4k_matrix_np(SEED, 950, vocab, hidden)
    H = orc.bf16_array_to_f64(synth.bf16_normal_np(SEED, 951, (M, hidden))) * 3.0
    # first pass with random drafts gives the argmaxes; then drafts that agree with them
    # for agent 0 (accept both), agent 1 (accept the first only) and agent 4 (accept)
    rng = np.random.default_rng(5)
    tokens = rng.integers(0, vocab, M).astype(np.int32)
    am, _ = _run(q, orc, H, W, hidden, vocab, n_rows, lens, tokens)
    t2 = tokens.copy()
    t2[1], t2[2] = am[0], am[1]            # agent 0: rows 0..2
    t2[4] = am[3]                          # agent 1: rows 3..5, draft 1 matches
    t2[5] = (am[4] + 1) % vocab            #          draft 2 does not
    t2[8] = am[7]                          # agent 4: rows 7..8
    _, acc = _run(q, orc, H, W, hidden, vocab, n_rows, lens, t2)
    assert acc.tolist() == [2, 1, 0, 0, 1]


def test_verify_full_vocab_head(q, orc):
    """4 agents x 3 rows through a 151936 x 5120 Q4_K head (the vocabulary size is a
    parameter; the pages do not give it), sampled logits checked."""
    hidden, vocab = 5120, 151936
    n_rows, lens = [3, 3, 3, 3], [1024, 500, 23000, 1]
    M = 12
    g = synth.torch_gen(SEED, "cuda", 960)
    Wd = synth.q4k_matrix_torch(g, vocab, hidden, "cuda")
    H = orc.bf16_array_to_f64(synth.bf16_normal_np(SEED, 961, (M, hidden)))
    rng = np.random.default_rng(9)
    tokens = rng.integers(0, vocab, M).astype(np.int32)
    rows = np.concatenate([[0, 1, 127, 128, vocab - 1], rng.integers(0, vocab, 40)])
    am, _ = _run(q, orc, H, Wd, hidden, vocab, n_rows, lens, tokens, rows=rows)
    t2 = tokens.copy()
    t2[1], t2[2] = am[0], am[1]
    _run(q, orc, H, Wd, hidden, vocab, n_rows, lens, t2, rows=rows)
