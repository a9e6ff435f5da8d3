// sched.cu -- host-side step scheduler for several agents sharing one model:
// which agents decode (and with how many draft rows), which prompt is fed as
// a chunk, prompt-lookup drafting and the reuse of a cached prefix.
//
// [OpenJet page] = rebasdaily.com 2026-10-29, "OpenJet ... multi-agent
// serving": the agents' next tokens and drafts share one weight stream
// (section 只搬一次权重), a long prompt must not stall the others (section
// 真正重要的是少互相堵车, which feeds prompts in pieces) and an agent's earlier
// context stays cached so a follow-up request only prefills what is new
// (time to first token). Drafts come from prompt lookup: the tokens that
// followed the latest earlier occurrence of the context's last n-gram (the
// page names speculative drafts; the lookup rule is the plainest reading).
//
// Plain host C++; no CUDA calls.
#include <cstring>

#include "common.cuh"

namespace {

bool valid_policy(const qad_sched_policy *p)
{
    return p && p->chunk_tokens >= 1 && p->decode_steps_per_chunk >= 0 && p->max_decode_rows >= 1 &&
           p->max_decode_rows <= QAD_MAX_ROWS && p->n_draft >= 0 && p->n_draft < QAD_MAX_ROWS &&
           (p->mode == QAD_SCHED_INTERLEAVE || p->mode == QAD_SCHED_PREFILL_FIRST);
}

}  // namespace

extern "C" int qad_sched_plan(const qad_sched_policy *p, const qad_sched_agent *agents, int n_agents, long long step,
                              int *decode_rows, int *chunk_agent, int *chunk_rows)
{
    if (!valid_policy(p) || !agents || n_agents <= 0 || step < 0 || !decode_rows || !chunk_agent || !chunk_rows)
        return qad::fail(QAD_ERR_INVALID, "qad_sched_plan: invalid policy or arguments");
    for (int a = 0; a < n_agents; ++a)
        if (agents[a].len < 0 || agents[a].prompt_left < 0 || agents[a].drafts < 0)
            return qad::fail(QAD_ERR_INVALID, "qad_sched_plan: agent %d has a negative count", a);
    std::memset(decode_rows, 0, sizeof(int) * (size_t)n_agents);
    *chunk_agent = -1;
    *chunk_rows = 0;

    // the prompt to feed: the lowest-index active agent with prompt tokens left
    int pa = -1;
    for (int a = 0; a < n_agents && pa < 0; ++a)
        if (agents[a].active && agents[a].prompt_left > 0)
            pa = a;
    int n_dec = 0;
    for (int a = 0; a < n_agents; ++a)
        if (agents[a].active && agents[a].prompt_left == 0)
            ++n_dec;
    bool chunk_now = false;
    if (pa >= 0) {
        if (p->mode == QAD_SCHED_PREFILL_FIRST || n_dec == 0)
            chunk_now = true;
        else
            chunk_now = step % (p->decode_steps_per_chunk + 1) == 0;
    }
    if (chunk_now) {
        *chunk_agent = pa;
        *chunk_rows = agents[pa].prompt_left < p->chunk_tokens ? agents[pa].prompt_left : p->chunk_tokens;
    }
    if (pa >= 0 && p->mode == QAD_SCHED_PREFILL_FIRST)
        return 0;  // a pending prompt holds every decoding agent back

    // decode rows: one per decoding agent (round-robin start so a budget smaller
    // than the agent count rotates), then drafts in the same order
    int budget = p->max_decode_rows, M = 0;
    const int start = (int)(step % n_agents);
    for (int i = 0; i < n_agents && budget > 0; ++i) {
        const int a = (start + i) % n_agents;
        if (agents[a].active && agents[a].prompt_left == 0) {
            decode_rows[a] = 1;
            --budget;
            ++M;
        }
    }
    for (int i = 0; i < n_agents && budget > 0; ++i) {
        const int a = (start + i) % n_agents;
        if (!decode_rows[a])
            continue;
        int want = agents[a].drafts < p->n_draft ? agents[a].drafts : p->n_draft;
        if (want > budget)
            want = budget;
        decode_rows[a] += want;
        budget -= want;
        M += want;
    }
    return M;
}

extern "C" int qad_sched_commit(qad_sched_agent *agents, int n_agents, const int *decode_rows, int chunk_agent,
                                int chunk_rows, const int *n_accept)
{
    if (!agents || n_agents <= 0 || !decode_rows || chunk_agent >= n_agents || chunk_rows < 0 ||
        (chunk_agent >= 0 && (chunk_rows == 0 || chunk_rows > agents[chunk_agent].prompt_left)) ||
        (chunk_agent < 0 && chunk_rows != 0))
        return qad::fail(QAD_ERR_INVALID, "qad_sched_commit: inconsistent plan");
    for (int a = 0; a < n_agents; ++a) {
        const int r = decode_rows[a];
        if (r < 0 || (r > 0 && (a == chunk_agent || agents[a].prompt_left > 0)))
            return qad::fail(QAD_ERR_INVALID, "qad_sched_commit: agent %d cannot decode this step", a);
    }
    for (int a = 0; a < n_agents; ++a) {
        const int r = decode_rows[a];
        if (!r)
            continue;
        int k = n_accept ? n_accept[a] : 0;
        k = k < 0 ? 0 : (k > r - 1 ? r - 1 : k);
        agents[a].len += k + 1;  // the accepted drafts plus the token after them
        agents[a].drafts = 0;    // spent: the caller drafts again from the new context
    }
    if (chunk_agent >= 0) {
        agents[chunk_agent].len += chunk_rows;
        agents[chunk_agent].prompt_left -= chunk_rows;
    }
    return QAD_OK;
}

extern "C" int qad_prompt_lookup(const int *tokens, int n_tokens, int min_ngram, int max_ngram, int n_draft,
                                 int *drafts)
{
    if ((!tokens && n_tokens > 0) || n_tokens < 0 || min_ngram < 1 || max_ngram < min_ngram || n_draft < 0 ||
        (!drafts && n_draft > 0))
        return qad::fail(QAD_ERR_INVALID, "qad_prompt_lookup: invalid arguments");
    for (int n = max_ngram; n >= min_ngram; --n) {
        if (n >= n_tokens)
            continue;  // the suffix needs an earlier occurrence that ends before it
        const int *suf = tokens + n_tokens - n;
        for (int j = n_tokens - n - 1; j >= 0; --j) {  // latest earlier occurrence first
            if (std::memcmp(tokens + j, suf, sizeof(int) * (size_t)n) != 0)
                continue;
            int k = 0;
            while (k < n_draft && j + n + k < n_tokens) {
                drafts[k] = tokens[j + n + k];
                ++k;
            }
            return k;
        }
    }
    return 0;
}

extern "C" int qad_common_prefix(const int *a, int na, const int *b, int nb)
{
    if ((!a && na > 0) || (!b && nb > 0) || na < 0 || nb < 0)
        return qad::fail(QAD_ERR_INVALID, "qad_common_prefix: invalid arguments");
    int k = 0;
    while (k < na && k < nb && a[k] == b[k])
        ++k;
    return k;
}
