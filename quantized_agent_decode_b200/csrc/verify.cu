// verify.cu -- the verify tail of a decode-and-verify step: logits of every
// row through a quantized output head, per-row argmax, greedy acceptance of
// each agent's drafts and the commit of its KV length.
//
// [OpenJet page] = rebasdaily.com 2026-10-29, "OpenJet ... multi-agent
// serving", section 只搬一次权重: the two drafts of every agent are checked
// in the same forward pass as its next token. The acceptance rule is not on
// the page; the rule implemented is greedy: draft j+1 is kept iff every
// earlier draft was and the argmax of row j equals it. The agent then emits
// the argmax of rows 0..k (k accepted drafts plus the token after them) and
// its cache length grows by k+1; the rejected rows' cache slots are simply
// overwritten by the next step.
//
// Design: the head is one more skinny Q4_K GEMM (the same prep + TMA/warp-MMA
// kernel as the stack, RMSNorm fused into the prep). The argmax runs as a
// grid of (row, vocabulary chunk) CTAs producing order-preserving 64-bit keys
// (float bits mapped to an unsigned order, then the complement of the index
// so ties resolve to the lowest index); one small CTA reduces the chunks and
// applies the acceptance rule.
#include "gemm.cuh"

namespace qad {

constexpr int VCHUNKS = 16;  // vocabulary chunks per row

__device__ __forceinline__ unsigned long long argmax_key(float f, int idx)
{
    uint32_t u = __float_as_uint(f);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    if (f != f)
        u = 0;  // NaN never wins
    return ((unsigned long long)u << 32) | (0xFFFFFFFFu - (uint32_t)idx);
}

__global__ void __launch_bounds__(256) k_argmax_partial(const float *__restrict__ logits, int vocab,
                                                        unsigned long long *__restrict__ keys)
{
    __shared__ unsigned long long red[8];
    const int r = blockIdx.y, ch = blockIdx.x, tid = threadIdx.x;
    pdl_trigger();
    pdl_wait();
    const int per = (vocab + VCHUNKS - 1) / VCHUNKS;
    const int lo = ch * per, hi = min(vocab, lo + per);
    const float *row = logits + (size_t)r * vocab;
    unsigned long long best = 0;
    for (int i = lo + tid; i < hi; i += 256) {
        const unsigned long long k = argmax_key(row[i], i);
        best = k > best ? k : best;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        const unsigned long long k = __shfl_xor_sync(0xffffffffu, best, o);
        best = k > best ? k : best;
    }
    if ((tid & 31) == 0)
        red[tid >> 5] = best;
    __syncthreads();
    if (tid == 0) {
        for (int w = 1; w < 8; ++w)
            best = red[w] > best ? red[w] : best;
        keys[(size_t)r * VCHUNKS + ch] = best;
    }
}

// One CTA: row tokens from the chunk keys, then one thread per agent applies
// the greedy rule and commits the length.
__global__ void __launch_bounds__(256) k_accept(const unsigned long long *__restrict__ keys, int M,
                                                const int *__restrict__ ars, int n_agents,
                                                const int *__restrict__ row_tokens, int *__restrict__ lens,
                                                int *__restrict__ out_tokens, int *__restrict__ n_accept,
                                                int *__restrict__ row_argmax_out)
{
    __shared__ int amax[QAD_MAX_ROWS];
    pdl_trigger();
    pdl_wait();
    for (int r = threadIdx.x; r < M; r += blockDim.x) {
        unsigned long long best = 0;
        for (int c = 0; c < VCHUNKS; ++c) {
            const unsigned long long k = keys[(size_t)r * VCHUNKS + c];
            best = k > best ? k : best;
        }
        amax[r] = (int)(0xFFFFFFFFu - (uint32_t)(best & 0xFFFFFFFFu));
        if (row_argmax_out)
            row_argmax_out[r] = amax[r];
    }
    __syncthreads();
    for (int a = threadIdx.x; a < n_agents; a += blockDim.x) {
        const int r0 = ars[a], n = ars[a + 1] - r0;
        int k = 0;
        while (k + 1 < n && amax[r0 + k] == row_tokens[r0 + k + 1])
            ++k;
        for (int j = 0; j < n; ++j)
            out_tokens[r0 + j] = j <= k ? amax[r0 + j] : -1;
        n_accept[a] = n > 0 ? k : 0;
        if (n > 0)
            lens[a] += k + 1;
    }
}

static size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t verify_ws_bytes(int hidden, int vocab, int M)
{
    return a256(frag_bytes(hidden, 2)) + a256((size_t)M * vocab * 4) + a256((size_t)M * VCHUNKS * 8);
}

}  // namespace qad

extern "C" size_t qad_verify_ws_bytes(int hidden, int vocab, int M)
{
    if (hidden <= 0 || hidden % 256 || vocab <= 0 || M <= 0 || M > QAD_MAX_ROWS)
        return 0;
    return qad::verify_ws_bytes(hidden, vocab, M);
}

extern "C" int qad_verify_step(const float *H, int M, int hidden, float rms_eps, const void *W_head, int vocab,
                               const int *agent_row_start, int n_agents, const int *row_tokens, int *lens,
                               int *out_tokens, int *n_accept, int *row_argmax, float *logits_out, void *ws,
                               size_t ws_bytes, void *stream)
{
    if (!H || !W_head || !agent_row_start || !row_tokens || !lens || !out_tokens || !n_accept || !ws || M <= 0 ||
        hidden <= 0 || vocab <= 0 || n_agents <= 0)
        return qad::fail(QAD_ERR_INVALID, "qad_verify_step: null pointer or non-positive size");
    if (M > QAD_MAX_ROWS || hidden % 256 || hidden > 65536)
        return qad::fail(QAD_ERR_UNSUPPORTED, "qad_verify_step: need M <= 16 and hidden %% 256 == 0, <= 65536");
    if (((uintptr_t)H | (uintptr_t)W_head | (uintptr_t)logits_out) & 15 || (uintptr_t)ws & 255)
        return qad::fail(QAD_ERR_INVALID, "qad_verify_step: H, W_head, logits must be 16-byte aligned, ws 256-byte");
    if (ws_bytes < qad::verify_ws_bytes(hidden, vocab, M))
        return qad::fail(QAD_ERR_WORKSPACE, "qad_verify_step: workspace %zu < %zu bytes", ws_bytes,
                         qad::verify_ws_bytes(hidden, vocab, M));
    cudaStream_t s = (cudaStream_t)stream;
    char *w = (char *)ws;
    qad::FragBuf fb = qad::frag_carve(w, hidden, 2);
    w += qad::a256(qad::frag_bytes(hidden, 2));
    float *logits = logits_out ? logits_out : (float *)w;
    w += qad::a256((size_t)M * vocab * 4);
    unsigned long long *keys = (unsigned long long *)w;

    qad::WeightMapsBlob maps;
    int rc = qad::make_weight_maps(4, W_head, vocab, hidden, &maps);
    if (rc)
        return rc;
    qad::PrepSrc src = {};
    src.kind = qad::PREP_RMSNORM;
    src.xf = H;
    src.ldx = hidden;
    src.eps = rms_eps;
    src.zero = logits;
    src.zero_n = (long long)M * vocab;
    if ((rc = qad::launch_prep(4, hidden, M, src, fb, s, false)))
        return rc;
    if ((rc = qad::launch_gemm(4, maps, vocab, hidden, M, fb, logits, vocab, s, true)))
        return rc;
    cudaError_t e = qad::launch_pdl(qad::k_argmax_partial, dim3(qad::VCHUNKS, M), dim3(256), 0, s, (const float *)logits,
                                    vocab, keys);
    if ((rc = qad::cuda_check(e, "argmax launch")))
        return rc;
    e = qad::launch_pdl(qad::k_accept, dim3(1), dim3(256), 0, s, (const unsigned long long *)keys, M, agent_row_start,
                        n_agents, row_tokens, lens, out_tokens, n_accept, row_argmax);
    return qad::cuda_check(e, "accept launch");
}
