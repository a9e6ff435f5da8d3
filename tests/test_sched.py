"""Host-side scheduler, prompt-lookup drafting and prefix reuse (no GPU needed:
these are plain host functions of the library)."""
import numpy as np
import pytest


@pytest.fixture(scope="module")
def q():
    import quantized_agent_decode_b200 as q
    from quantized_agent_decode_b200 import build
    build.build()
    return q


def test_prompt_lookup_hand_cases(q, orc):
    assert q.prompt_lookup([1, 2, 3, 4, 1, 2], n_draft=2) == [3, 4]        # 2-gram [1, 2] recurs at 0
    assert q.prompt_lookup([1, 2, 3, 9, 2, 3, 7, 1, 2, 3], n_draft=2) == [9, 2]  # 3-gram wins over the later 2-gram
    assert q.prompt_lookup([5, 5, 5], n_draft=2) == [5]                     # overlapping match, one token follows
    assert q.prompt_lookup([1, 2, 3], n_draft=2) == []                      # nothing recurs
    assert q.prompt_lookup([], n_draft=2) == []
    assert q.prompt_lookup([4, 8, 4, 6, 4], n_draft=3) == [6, 4]           # latest earlier 1-gram (pos 2)
    for toks, want in (([1, 2, 3, 4, 1, 2], [3, 4]), ([5, 5, 5], [5]), ([4, 8, 4, 6, 4], [6, 4])):
        assert orc.prompt_lookup(toks, 1, 3, 3)[:2] == want[:2]


def test_prompt_lookup_matches_oracle_on_random_streams(q, orc):
    rng = np.random.default_rng(5)
    for _ in range(400):
        n = int(rng.integers(0, 60))
        toks = rng.integers(0, int(rng.integers(2, 12)), n).tolist()
        mn, mx = sorted(rng.integers(1, 5, 2).tolist())
        nd = int(rng.integers(0, 5))
        assert q.prompt_lookup(toks, n_draft=nd, min_ngram=mn, max_ngram=mx) == orc.prompt_lookup(toks, mn, mx, nd)


def test_common_prefix(q):
    assert q.common_prefix([1, 2, 3], [1, 2, 4, 5]) == 2
    assert q.common_prefix([], [1]) == 0
    assert q.common_prefix([7, 8], [7, 8]) == 2


def _states(s, lens, prompts, active=None, drafts=None):
    for a in range(s.n):
        s.agents[a].len = lens[a]
        s.agents[a].prompt_left = prompts[a]
        s.agents[a].active = 1 if active is None else active[a]
        s.agents[a].drafts = 0 if drafts is None else drafts[a]


def test_plan_rows_chunk_and_budget(q):
    s = q.Scheduler(4, chunk_tokens=2048, max_decode_rows=12, n_draft=2)
    _states(s, [100, 200, 0, 50], [0, 0, 20480, 0], drafts=[2, 1, 0, 5])
    rows, ca, cr = s.plan()
    assert rows == [3, 2, 0, 3] and (ca, cr) == (2, 2048)
    # a tight budget: every decoding agent first gets one row, then drafts from the rotating start
    s = q.Scheduler(4, max_decode_rows=4, n_draft=2)
    _states(s, [1, 1, 1, 1], [0, 0, 0, 0], drafts=[2, 2, 2, 2])
    s.step = 1
    rows, ca, cr = s.plan()
    assert sum(rows) == 4 and min(rows) == 1 and ca == -1
    # paused agents get nothing
    s = q.Scheduler(3)
    _states(s, [5, 5, 5], [0, 0, 0], active=[1, 0, 1], drafts=[2, 2, 2])
    assert s.plan()[0] == [3, 0, 3]


def test_plan_round_robin_when_agents_exceed_budget(q):
    s = q.Scheduler(6, max_decode_rows=4, n_draft=0)
    _states(s, [1] * 6, [0] * 6)
    served = np.zeros(6, int)
    for step in range(12):
        s.step = step
        rows = s.plan()[0]
        assert sum(rows) == 4
        served += np.array(rows)
    assert served.min() == served.max() == 8  # every agent served equally over a full rotation


def test_prefill_first_holds_decoders(q):
    s = q.Scheduler(4, chunk_tokens=2048, mode=q.SCHED_PREFILL_FIRST)
    _states(s, [1024, 1024, 0, 1024], [0, 0, 5000, 0])
    rows, ca, cr = s.plan()
    assert rows == [0, 0, 0, 0] and (ca, cr) == (2, 2048)


@pytest.mark.parametrize("mode,every", [(0, 0), (0, 2), (1, 0)])
def test_simulated_twenty_k_prompt(q, mode, every):
    """Three decoding agents and one 20480-token prompt: interleaved chunks keep
    the decoders moving (one token per step each when no draft is accepted);
    prefill-first stalls them until the prompt is in."""
    s = q.Scheduler(4, chunk_tokens=2048, decode_steps_per_chunk=every, max_decode_rows=12, n_draft=2, mode=mode)
    _states(s, [1024, 1024, 0, 1024], [0, 0, 20480, 0])
    steps_to_prompt = None
    while True:
        rows, ca, cr = s.plan()
        s.commit(rows, ca, cr, n_accept=[0] * 4)
        if steps_to_prompt is None and s.agents[2].prompt_left == 0:
            steps_to_prompt = s.step
            dec_tokens = s.agents[0].len - 1024
            break
    assert s.agents[2].len == 20480
    if mode == q.SCHED_PREFILL_FIRST:
        assert steps_to_prompt == 10 and dec_tokens == 0
    else:
        assert steps_to_prompt == 1 + 9 * (every + 1) and dec_tokens == steps_to_prompt


def test_commit_accepts_drafts_and_rejects_bad_plans(q):
    s = q.Scheduler(2, n_draft=2)
    _states(s, [10, 0], [0, 300], drafts=[2, 0])
    rows, ca, cr = s.plan()
    assert rows == [3, 0] and (ca, cr) == (1, 300)
    s.commit(rows, ca, cr, n_accept=[5, 0])  # clamped to rows - 1 = 2
    assert s.agents[0].len == 13 and s.agents[0].drafts == 0
    assert s.agents[1].len == 300 and s.agents[1].prompt_left == 0
    with pytest.raises(q.QadError):
        s.commit([0, 1], 0, 1)   # agent 0 has no prompt left to chunk


def test_prompt_lookup_drafts_pay_off_on_repetitive_streams(q, orc):
    """A toy agent whose true continuation repeats its context (as code edits
    often do): prompt-lookup drafts are accepted by the greedy rule (oracle),
    so each scheduled step commits more than one token."""
    rng = np.random.default_rng(7)
    base = rng.integers(0, 1000, 40).tolist()
    truth = base * 6                       # the stream the agent will produce
    ctx = truth[:50]                       # already cached (prompt + earlier output)
    s = q.Scheduler(1, n_draft=2, max_decode_rows=3)
    s.agents[0].len, s.agents[0].prompt_left, s.agents[0].active = len(ctx), 0, 1
    steps = 0
    while len(ctx) < 200:
        drafts = q.prompt_lookup(ctx, n_draft=2)
        s.agents[0].drafts = len(drafts)
        rows, ca, cr = s.plan()
        n = rows[0]
        row_tokens = [ctx[-1]] + drafts[:n - 1]           # inputs of the agent's rows
        pos = len(ctx)
        row_argmax = [truth[pos + k] for k in range(n)]   # what the model predicts after each row
        ars = np.array([0, n], np.int32)
        lens2, out, acc = orc.accept_greedy(row_argmax, row_tokens, ars, [s.agents[0].len])
        s.commit(rows, ca, cr, n_accept=[int(acc[0])])
        ctx += [int(t) for t in out if t >= 0]
        assert s.agents[0].len == len(ctx) == int(lens2[0])
        steps += 1
    assert ctx[:200] == truth[:len(ctx)][:200]
    assert (len(ctx) - 50) / steps > 2.5  # close to 3 tokens per step once the pattern repeats
