"""KV reuse across an agent's requests.

OpenJet page, section 真正重要的是少互相堵车: when an agent sends its next
request, the context it already has in its KV cache is kept and only the new
part of the prompt is prefilled, which is what makes the time to the first
token small. With the library: qad_common_prefix gives the reusable length P of
the old and new token sequences, the agent's cache length is set to P, and the
new suffix goes through qad_mixed_step as a chunk at positions P ...

Property checked: a prompt fed as its prefix, then the suffix on top of the
cached prefix, gives every row the hidden state it gets when the whole prompt is
fed at once from position 0. The cached keys and values of the prefix are the
bf16 of their projections whichever step wrote them; what may differ is only
the summation order inside the chunk attention (a different split of the keys
between the cache and the chunk), so the rows agree to fp32 rounding, far
inside the layer tolerances of the teacher-forced tests.
"""
import numpy as np
import pytest
import torch

import synth
from conftest import SEED
from test_gpu_step import Stack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import quantized_agent_decode_b200 as q
    from quantized_agent_decode_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return q


def _prefill(q, st, X, start, C, ws):
    """C prompt rows of agent 0 at positions start .. start + C - 1 (no decode rows)."""
    Xd = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).view(torch.bfloat16).cuda()
    Hd = torch.empty(C, st.H, dtype=torch.float32, device="cuda")
    st.model.mixed_step(Xd, 0, None, st.A, 1, None, 0, start, C, Hd, ws)
    torch.cuda.synchronize()
    return Hd.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("P,S", [(96, 40), (257, 64), (64, 129)])
def test_suffix_prefill_on_cached_prefix_matches_full_prefill(q, P, S):
    st = Stack(q, 2, 512, 1024, 8, 2, [0], [0], seed=60 + S, extra_cap=P + S + 4)
    X = synth.bf16_normal_np(SEED, 9100 + P, (P + S, st.H))
    old_tokens = list(range(1000, 1000 + P))
    new_tokens = old_tokens + list(range(5000, 5000 + S))
    reuse = q.common_prefix(old_tokens, new_tokens)
    assert reuse == P
    ws = q.alloc_ws(st.model.mixed_ws_bytes(0, P + S))
    # the whole prompt from an empty context
    full = _prefill(q, st, X, 0, P + S, ws)
    # the previous request's context, then the new suffix on top of the cached prefix
    st.reset_caches()
    first = _prefill(q, st, X[:P], 0, P, ws)
    second = _prefill(q, st, X[P:], reuse, S, ws)
    assert q.device_status() == 0 and q.dense_status() == 0
    scale = np.abs(full).max()
    for got, ref in ((first, full[:P]), (second, full[P:])):
        err = np.abs(got - ref)
        assert np.isfinite(got).all()
        assert err.max() <= 1e-3 * scale, (err.max(), scale)
        assert err.mean() <= 1e-4 * scale, (err.mean(), scale)


def test_common_prefix_lengths(q):
    assert q.common_prefix([1, 2, 3], [1, 2, 3, 4]) == 3
    assert q.common_prefix([1, 2, 3], [1, 9, 3]) == 1
    assert q.common_prefix([], [7]) == 0
    assert q.common_prefix([5, 6], [5, 6]) == 2
