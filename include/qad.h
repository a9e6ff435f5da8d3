/*
 * qad.h -- C ABI of the B200 (sm_100a) multi-agent quantized decode step.
 *
 * One batched decode-and-verify step for several coding agents that share one
 * Q4_K-quantized model: every active agent contributes its next token plus its
 * draft tokens, all rows are stacked into one batch, the quantized weights are
 * streamed from HBM once per step and each weight is used for every row, and
 * each agent's rows attend over that agent's own KV cache.
 *
 * Citations name the page and its section:
 *   [OpenJet page] rebasdaily.com, 2026-10-29, "OpenJet ... Qwen3.8-27B
 *   multi-agent serving": intro (four coding agents, one GPU, Q4_K_M weights);
 *   section 只搬一次权重 ("move the weights once": 4 agents x (next token +
 *   2 drafts) = 12 rows, one pass over the weights for all rows, drafts
 *   verified in the same pass, each agent reads its own KV cache).
 *   [P3 page] rebasdaily.com, 2026-09-10, dual-4090 llama.cpp agent
 *   concurrency, section 真正昂贵的是“同时记住” (KV cache per agent).
 *
 * Conventions for every entry point:
 *   - Pointers named d_* or documented "device" are device pointers owned by
 *     the caller; the library never frees or retains them past the call
 *     (except the model handle, which keeps the pointers it was given).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = legacy default stream) unless stated otherwise. Nothing here
 *     allocates device memory on the hot path: scratch space is a caller
 *     workspace whose size a *_ws_bytes() query returns.
 *   - bf16 values are passed as uint16_t bit patterns.
 *   - Row-major layouts. Quantized matrices are [N rows][K/256 blocks]:
 *     row n's blocks are contiguous, rows follow each other.
 *   - Return 0 on success, or a negative QAD_ERR_* code; the thread-local
 *     text of the last error is available from qad_last_error(). Arguments
 *     are checked on the host before any launch; a failed check launches
 *     nothing.
 */
#ifndef QAD_H
#define QAD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QAD_OK 0
#define QAD_ERR_INVALID (-1)     /* null pointer, negative size, inconsistent sizes */
#define QAD_ERR_UNSUPPORTED (-2) /* shape outside the supported range (e.g. M > 16, K % 256) */
#define QAD_ERR_WORKSPACE (-3)   /* workspace smaller than the *_ws_bytes() query */
#define QAD_ERR_CUDA (-4)        /* a CUDA runtime call or launch failed */

#define QAD_MAX_ROWS 16          /* rows of one step (skinny path) */
#define QAD_QK 256               /* weights per quantized block */
#define QAD_Q4K_BLOCK_BYTES 144
#define QAD_Q6K_BLOCK_BYTES 210

/* Text of the last error on this thread ("" if none). */
const char *qad_last_error(void);

/* ABI version (major*100 + minor). */
int qad_version(void);

/* ---------------------------------------------------------------- codecs
 * Q4_K super-block (the "Q4_K_M" weights of [OpenJet page], intro; block
 * layout per the GGUF Q4_K convention): 144 bytes = d fp16, dmin fp16,
 * 12 bytes of packed 6-bit sub-block scales/mins, 128 bytes of 4-bit quants;
 * weight i = d*sc_{i/32}*q_i - dmin*m_{i/32}.
 *
 * qad_q4k_unpack: decodes n_blocks device blocks at W into
 *   q [n_blocks][256] (0..15), sc [n_blocks][8], m [n_blocks][8] (0..63),
 *   d [n_blocks], dmin [n_blocks] (fp16 bit patterns). All device pointers.
 *   Bit-exact. Used by tests and diagnostics.
 * qad_q6k_unpack: Q6_K-like block (210 bytes: ql[128], qh[64], int8
 *   scales[16], d fp16); weight i = d*scales_{i/16}*(q_i - 32).
 *   q [n_blocks][256] (0..63), sc [n_blocks][16] (int8), d [n_blocks]. */
int qad_q4k_unpack(const void *W, long long n_blocks, uint8_t *q, uint8_t *sc, uint8_t *m,
                   uint16_t *d, uint16_t *dmin, void *stream);
int qad_q6k_unpack(const void *W, long long n_blocks, uint8_t *q, int8_t *sc, uint16_t *d,
                   void *stream);

/* ---------------------------------------------------------------- skinny GEMM
 * Y[r][n] = sum_k w[n][k] * X[r][k] for r < M, n < N: the shared weight pass
 * of [OpenJet page], section 只搬一次权重 -- each quantized block is read from
 * HBM once and used for all M rows.
 *   W  device, 16-byte aligned: Q4_K [N][K/256 blocks] (q4k), or Q6_K-like in
 *      the packed layout of qad_q6k_pack (q6k)
 *   X  device bf16 [M][K]
 *   Y  device fp32 [M][N]; overwritten, or accumulated into (Y += X W^T) when
 *      `accumulate` is non-zero
 *   ws device workspace of at least qad_gemm_ws_bytes(K, M) bytes, 256-byte
 *      aligned; its contents are scratch
 * 1 <= M <= 16, K % 256 == 0, K <= 65536, N >= 1. Results are fp32-accumulated
 * products of exact operands (the tensor-core operand of X is fp16 with a
 * per-row power-of-two scale, see the design notes); the result is not
 * bit-reproducible across launches because partial sums are combined with
 * atomic adds. */
size_t qad_gemm_ws_bytes(int K, int M);

/* Q6_K-like weights are streamed from a packed device layout that keeps every
 * field 16-byte aligned (a 210-byte block cannot be addressed by the tensor
 * memory accelerator): plane A [N][K/256][208] holds the first 208 bytes of
 * each block (ql, qh, int8 scales, unchanged), followed by plane D
 * [N][ceil8(K/256)] holding each block's fp16 d (rows padded with zeros to a
 * multiple of 8 blocks). Same bytes per block as the GGUF layout, plus the
 * padding. qad_q6k_pack converts N x K GGUF-layout blocks W (device) into
 * W_packed (device, 16-byte aligned, qad_q6k_packed_bytes(N, K) bytes); it is
 * a one-time load step, not part of the decode step. */
size_t qad_q6k_packed_bytes(long long N, int K);
int qad_q6k_pack(const void *W, int N, int K, void *W_packed, void *stream);

/* qad_q4k_gemm for callers that cannot allocate device memory at call time
 * (the pages have no counterpart: this is a library-integration entry point).
 * Such callers include servers that reserve all of HBM for weights and
 * KV-cache pools at start-up and forbid later allocations, code that must not
 * trigger the device-wide synchronisation cudaFree can cause while other
 * streams are decoding, and plain C integrations that only hold pointers to
 * buffers owned elsewhere. Arguments and result are those of qad_q4k_gemm
 * without the workspace: the scratch is a fixed array of
 * qad_q4k_gemm_noalloc_scratch_bytes() bytes (1 MiB; enough for K <= 30464,
 * for every row count M from 1 to 16) in device memory that every GPU loading
 * this library holds until the process exits. Calls that need more scratch
 * fail with QAD_ERR_UNSUPPORTED before any launch. Outside stream capture each
 * call looks up the array's device address (cudaGetSymbolAddress), so a device
 * reset in between is harmless; a call whose stream is being captured reuses
 * the address an earlier call found on that device, so make one call before
 * any stream capture (a first call during capture fails with QAD_ERR_INVALID). All calls on a device share the one array, and
 * each call rewrites the parts it reads, so calls that overlap on the GPU
 * (different streams, or different host threads without ordering) race and
 * must be serialised by the caller. Nothing here calls cudaMalloc, cudaFree
 * or any allocating routine. */
size_t qad_q4k_gemm_noalloc_scratch_bytes(void);
int qad_q4k_gemm_noalloc(const void *W, int N, int K, const uint16_t *X, int M, float *Y, int accumulate,
                         void *stream);

/* Device status word of the GEMM pipelines on the current device: 0 if every
 * shared-memory pipeline wait completed; non-zero if a wait gave up (after
 * about 2 s; the kernel then returned early and its outputs are incomplete). Synchronous (reads device memory); reset != 0 clears it.
 * Returns the status (>= 0) or a negative QAD_ERR_* code. */
int qad_device_status(int reset);

/* Test hook for the bounded waits (no counterpart on the pages): makes the
 * producer of CTA 0 of the next launches of one pipeline on the current
 * device stop issuing copies,
 * so that CTA's waits on them run out and the kernel takes its early exit
 * (records a status, waits for the copies and tensor-core work it already
 * issued, frees its tensor memory, returns) instead of completing.
 *   kernel = 0: the skinny GEMM (qad_q4k_gemm, qad_q6k_gemm and the decode
 *               step); no operand-record copy from CTA 0's unit `at` on
 *               (its status: qad_device_status);
 *   kernel = 1: the dense GEMM (qad_q4k_gemm_dense, qad_q6k_gemm_dense);
 *               no copy from CTA 0's activation k-step `at` on (qad_dense_status);
 *   kernel = 2: the prefill attention (qad_prefill_attn and the mixed step);
 *               no K/V tile from CTA (0, 0)'s tile `at` on (qad_prefill_status).
 * at < 0 switches the hook off. The outputs of an affected launch are
 * incomplete. Each timed-out wait takes about 2 s. Synchronous (writes device
 * memory). Returns QAD_OK, or QAD_ERR_INVALID for an unknown kernel. */
int qad_debug_stall(int kernel, int at);
int qad_q4k_gemm(const void *W, int N, int K, const uint16_t *X, int M, float *Y, int accumulate,
                 void *ws, size_t ws_bytes, void *stream);
int qad_q6k_gemm(const void *W, int N, int K, const uint16_t *X, int M, float *Y, int accumulate,
                 void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------- prefill-chunk GEMM
 * OpenJet page, section 真正重要的是少互相堵车: a long prompt is processed in
 * chunks (2048 prompt rows of one agent, plus the 12 decode rows) through the
 * same quantized weights; at that M the product is compute-bound.
 *
 * Y[m][n] = sum_k w[n][k] * x[m][k] for M >= 1 rows on the 5th-generation
 * tensor cores (tcgen05, fp16 operands, fp32 accumulate in TMEM). Each weight
 * is formed in fp32 (d*sc*q - dmin*m for Q4_K, d*sc*(q - 32) for Q6_K-like)
 * and rounded to fp16 once in shared memory, so it is within (2^-11 + 2^-24)
 * of its exact value relative to |w|; x enters as fp16 of x * 2^e_m with a
 * per-row power of two (exact for bf16 rows whose dynamic range is below
 * 2^38). When the last round of 128 x 256 output tiles would leave many SMs
 * idle, its tiles are split between CTAs along K and their parts are added
 * into Y with fp32 atomics; such launches are not bit-reproducible run to run
 * (the rest of Y is).
 *   W   device: Q4_K [N][K/256][144] (qad_q4k_gemm_dense) or the packed
 *       Q6_K-like layout of qad_q6k_pack (qad_q6k_gemm_dense); 16-byte aligned
 *   X   device bf16 [M][K], 16-byte aligned;  Y  device fp32 [M][N], overwritten
 *   ws  device workspace of qad_dense_gemm_ws_bytes(K, M) bytes, 256-byte aligned
 * K % 256 == 0, K <= 65536. Returns 0 or a negative QAD_ERR_* code. Launches
 * two kernels on `stream`. */
size_t qad_dense_gemm_ws_bytes(int K, int M);
int qad_q4k_gemm_dense(const void *W, int N, int K, const uint16_t *X, int M, float *Y, void *ws,
                       size_t ws_bytes, void *stream);
int qad_q6k_gemm_dense(const void *W, int N, int K, const uint16_t *X, int M, float *Y, void *ws,
                       size_t ws_bytes, void *stream);
/* 0 if every pipeline wait of the dense GEMM completed since the last reset
 * (else 1 raw blocks, 2 activation tiles, 3 weight tiles, 4 accumulator,
 * 5 teardown); reset != 0 clears it. Negative QAD_ERR_* on a CUDA error. */
int qad_dense_status(int reset);

/* ---------------------------------------------------------------- attention
 * Grouped-query decode attention of each agent's rows over that agent's own
 * bf16 KV cache ([OpenJet page], section 只搬一次权重; [P3 page]).
 * Agent a owns rows r = agent_row_start[a] .. agent_row_start[a+1]-1; row
 * j = r - agent_row_start[a] sits at position lens[a] + j and attends over
 * keys t = 0 .. lens[a] + j (cached context plus the agent's new rows up to
 * itself: the draft rows see exactly what one-at-a-time decoding would).
 * q-head h reads kv-head h * n_kvh / n_qh.
 *   Q      device bf16 [M][n_qh][hd]
 *   Kc, Vc device bf16 [n_agents][n_kvh][kv_cap][hd]; positions
 *          lens[a] .. lens[a]+n_rows-1 must already hold the new rows' keys
 *          and values (qad_decode_step writes them itself)
 *   lens, agent_row_start  device int32 [n_agents], [n_agents+1]
 *   O      device bf16 [M][n_qh][hd]
 *   ws     device workspace of qad_decode_attn_ws_bytes(...) bytes
 * hd == 128, n_qh % n_kvh == 0, rows per agent * (n_qh/n_kvh) <= 96,
 * lens[a] + rows <= kv_cap (entries beyond kv_cap are skipped on the device).
 * scale is the softmax temperature (1/sqrt(hd) for standard attention). */
size_t qad_decode_attn_ws_bytes(int n_agents, int n_qh, int n_kvh, int kv_cap, int max_rows_per_agent);
int qad_decode_attn(const uint16_t *Q, const uint16_t *Kc, const uint16_t *Vc, const int *lens,
                    const int *agent_row_start, int n_agents, int max_rows_per_agent, int kv_cap,
                    int n_qh, int n_kvh, int hd, float scale, uint16_t *O, void *ws, size_t ws_bytes,
                    void *stream);

/* ---------------------------------------------------------------- q8_0 KV cache
 * dual-4090 page (rebasdaily.com 2026-09-10, llama.cpp agent concurrency on two
 * RTX 4090s): its tests keep the KV cache in q8_0. Block format (llama.cpp's
 * q8_0): 32 consecutive values share one fp16 scale and hold int8 codes,
 *   d = amax / 127 (fp32 division), id = d != 0 ? 1 / d : 0 (fp32),
 *   q_i = roundf(x_i * id) (fp32 product, ties away from zero), scale = fp16_RNE(d),
 * value = fp16(d) * q. A q8_0 cache tensor is ONE allocation of
 * qad_kv_cache_bytes(QAD_KV_Q8_0, ...) bytes: the codes [agents][n_kvh][kv_cap][hd]
 * int8 first, then, at the next 256-byte boundary, the scales
 * [agents][n_kvh][kv_cap][hd/32] fp16. Values must be finite and within the
 * fp16 range. */
#define QAD_KV_BF16 0
#define QAD_KV_Q8_0 8
/* Bytes of one K (or V) cache tensor of the given format; 0 for invalid
 * arguments (hd must be 128). */
size_t qad_kv_cache_bytes(int kv_format, int n_agents, int n_kvh, int kv_cap, int hd);
/* q8_0 of n values (n % 32 == 0): x device fp32 (x_is_bf16 == 0) or bf16
 * [n], 16-byte aligned; q device int8 [n], 16-byte aligned; d device fp16
 * [n/32]. One launch on `stream`. Bit-exact with the definition above. */
int qad_q8_0_quantize(const void *x, int x_is_bf16, long long n, int8_t *q, uint16_t *d, void *stream);
/* Decode attention (the definition of qad_decode_attn) over a q8_0 cache:
 *   Kq, Vq  device int8 codes [n_agents][n_kvh][kv_cap][hd], 16-byte aligned
 *   Kd, Vd  device fp16 scales [n_agents][n_kvh][kv_cap][hd/32], 8-byte aligned
 * Other arguments, limits and the workspace are those of qad_decode_attn
 * (qad_decode_attn_ws_bytes). Keys enter the product exactly (int8 codes,
 * per-block scales applied in fp32); V is dequantised to fp16 (one rounding)
 * and the probabilities are fp16. Q 8-byte aligned. */
int qad_decode_attn_q8(const uint16_t *Q, const int8_t *Kq, const uint16_t *Kd, const int8_t *Vq,
                       const uint16_t *Vd, const int *lens, const int *agent_row_start, int n_agents,
                       int max_rows_per_agent, int kv_cap, int n_qh, int n_kvh, int hd, float scale,
                       uint16_t *O, void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------- verify tail
 * OpenJet page, section 只搬一次权重: every agent's drafts are checked in the
 * same pass as its next token. The acceptance rule is not on the page; the
 * rule implemented is greedy. For the step's final hidden states H:
 *   logits = bf16(rmsnorm(H)) . W_head^T          (Q4_K head, fp32 [M][vocab])
 *   row_argmax[r] = first index of the row's maximum logit (fp32 decision)
 *   per agent a (rows r0 .. r0+n-1, inputs row_tokens[]): draft j+1 (the input
 *   of row j+1) is accepted iff all earlier drafts were and
 *   row_argmax[r0+j] == row_tokens[r0+j+1]; with k accepted,
 *   out_tokens[r0+j] = row_argmax[r0+j] for j <= k and -1 after,
 *   n_accept[a] = k, lens[a] += k + 1 (agents with no rows: unchanged).
 *   H          device fp32 [M][hidden], 16-byte aligned
 *   W_head     device Q4_K [vocab][hidden/256][144], 16-byte aligned
 *   agent_row_start device int32 [n_agents+1]; row_tokens device int32 [M]
 *   lens       device int32 [n_agents], updated in place (the KV-length commit)
 *   out_tokens device int32 [M]; n_accept device int32 [n_agents]
 *   row_argmax optional device int32 [M]; logits_out optional device fp32
 *              [M][vocab] (else the logits live in ws)
 *   ws         device workspace of qad_verify_ws_bytes(hidden, vocab, M) bytes
 * 1 <= M <= 16, hidden % 256 == 0. Four launches on `stream`. Returns 0 or a
 * negative QAD_ERR_* code. */
size_t qad_verify_ws_bytes(int hidden, int vocab, int M);
int qad_verify_step(const float *H, int M, int hidden, float rms_eps, const void *W_head, int vocab,
                    const int *agent_row_start, int n_agents, const int *row_tokens, int *lens, int *out_tokens,
                    int *n_accept, int *row_argmax, float *logits_out, void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------- prefill-chunk attention
 * OpenJet page, section 真正重要的是少互相堵车: a prompt chunk of one agent
 * (C rows at positions len .. len+C-1) attends causally over the agent's own
 * cache: row j, q-head h (kv-head h / (n_qh/n_kvh)) sees keys 0 .. len+j,
 *   o = softmax(q . K[0..len+j]^T * scale) V[0..len+j]
 * (the decode attention's definition with C rows). The chunk's k, v must
 * already be in the cache at positions len .. len+C-1.
 *   Q       device bf16 [C][n_qh][128]
 *   Kc, Vc  device bf16 [n_kvh][kv_cap][128] (this agent's cache); len + C <= kv_cap
 *   O       device bf16 [C][n_qh][128], written
 * Tensor-core products (tcgen05, S and O in TMEM) with fp32 softmax; the
 * probabilities enter the PV product rounded to bf16 (relative error <= 2^-9).
 * hd must be 128. Q, caches and O 16-byte aligned. Returns 0 or a negative
 * QAD_ERR_* code. */
int qad_prefill_attn(const uint16_t *Q, const uint16_t *Kc, const uint16_t *Vc, int len, int C, int kv_cap,
                     int n_qh, int n_kvh, int hd, float scale, uint16_t *O, void *stream);
/* Status of the prefill attention's bounded pipeline waits since the last
 * reset: 0 = none timed out, > 0 = the stage that timed out (the launch then
 * skips its remaining work). reset != 0 clears it. Negative QAD_ERR_* on a
 * CUDA error. */
int qad_prefill_status(int reset);

/* ---------------------------------------------------------------- row packer
 * Host-only. Stacks every agent's rows (next token + drafts) agent-major into
 * one batch ([OpenJet page], section 只搬一次权重). An agent paused for a tool
 * call passes n_rows = 0.
 *   agents[a].rows   host bf16 [n_rows][hidden]
 *   agents[a].len    cached tokens before the step
 * Writes X [M][hidden], row_agent[M], row_pos[M] (= len + j) and
 * agent_row_start[n_agents+1] (host arrays of capacity max_rows rows).
 * Returns M >= 0, or a negative QAD_ERR_* code (M > max_rows, n_rows < 0 ...). */
typedef struct {
    const uint16_t *rows;
    int n_rows;
    int len;
} qad_agent_rows;

int qad_pack_rows(const qad_agent_rows *agents, int n_agents, int hidden, int max_rows, uint16_t *X,
                  int *row_agent, int *row_pos, int *agent_row_start);

/* ---------------------------------------------------------------- decode step
 * [OpenJet page], section 只搬一次权重 (move the weights once): one model
 * serves several coding agents; its quantized weights are read from memory once
 * per step for the stacked rows of all active agents, and each agent keeps its
 * own KV cache. The page ships it as one persistent kernel over a Q4_K_M model
 * (intro: Qwen3.8-27B Q4_K_M); here the model is the stack of decoder layers
 * below, Q4_K matrices with a Q6_K-like down projection.
 * A model is a stack of decoder layers whose weights and KV caches the caller
 * owns. Per layer (device pointers):
 *   w_qkv  Q4_K [(n_qh + 2 n_kvh) hd][hidden]   rows: q heads, k heads, v heads
 *   w_o    Q4_K [hidden][n_qh hd]
 *   w_gu   Q4_K [2 inter][hidden]               rows: gate, then up
 *   w_down Q6_K-like [hidden][inter], packed by qad_q6k_pack
 *   k_cache, v_cache bf16 [max_agents][n_kvh][kv_cap][hd] (kv_format
 *          QAD_KV_BF16), or q8_0 cache allocations of qad_kv_cache_bytes(
 *          QAD_KV_Q8_0, max_agents, n_kvh, kv_cap, hd) bytes (kv_format
 *          QAD_KV_Q8_0; the new rows' k, v are quantised from the fp32
 *          projection)
 * The descriptor's pointer arrays are host arrays of n_layers entries and are
 * copied by qad_model_create. A zero-initialised kv_format is bf16. */
typedef struct {
    int n_layers, hidden, inter, n_qh, n_kvh, head_dim;
    int max_agents, kv_cap;
    float rms_eps;
    const void *const *w_qkv;
    const void *const *w_o;
    const void *const *w_gu;
    const void *const *w_down;
    uint16_t *const *k_cache;
    uint16_t *const *v_cache;
    int kv_format;
} qad_model_desc;

typedef struct qad_model qad_model;

int qad_model_create(const qad_model_desc *desc, qad_model **out);
void qad_model_destroy(qad_model *model);

/* One decode-and-verify forward step for the packed batch ([OpenJet page],
 * section 只搬一次权重: every agent's next token and its drafts form the rows
 * of one batch, each weight read once is used for every row, the drafts are
 * checked in the same pass, and each agent's rows attend over that agent's own
 * cache), per layer:
 *   x1 = bf16(rmsnorm(h)); qkv = x1 Wqkv^T; Q = bf16(q); append bf16 k, v of
 *   every row at its position; o = attention; h += bf16(o) Wo^T;
 *   x2 = bf16(rmsnorm(h)); gu = x2 Wgu^T; h += bf16(silu(gate)*up) Wdown^T.
 *   X        device bf16 [M][hidden] (the rows' input hidden states)
 *   agent_row_start, lens  device int32 [n_agents+1], [n_agents]; lens are
 *            the cached lengths before the step (the caller commits accepted
 *            tokens afterwards; rejected slots are overwritten next step)
 *   H_out    device fp32 [M][hidden], 16-byte aligned: the residual stream
 *            after the last layer
 *   ws       device workspace of qad_decode_step_ws_bytes(model, M) bytes,
 *            256-byte aligned
 * 1 <= M <= 16, n_agents <= max_agents. */
size_t qad_decode_step_ws_bytes(const qad_model *model, int M);
int qad_decode_step(qad_model *model, const uint16_t *X, int M, const int *agent_row_start,
                    int n_agents, int max_rows_per_agent, const int *lens, float *H_out, void *ws,
                    size_t ws_bytes, void *stream);

/* The same step with HOST inputs and output: copies X, agent_row_start and
 * lens into the workspace, runs the step (replaying a CUDA graph captured on
 * the first call for this (model, M, n_agents, workspace)), copies H_out back
 * and synchronises the stream. Host buffers should be pinned for speed. */
int qad_decode_step_host(qad_model *model, const uint16_t *X_host, int M,
                         const int *agent_row_start_host, int n_agents, int max_rows_per_agent,
                         const int *lens_host, float *H_out_host, void *ws, size_t ws_bytes,
                         void *stream);

/* CUDA-graph form of qad_decode_step: capture once, replay each step. The
 * graph records the given device pointers; refresh their contents between
 * replays. */
typedef struct qad_step_graph qad_step_graph;
int qad_step_graph_create(qad_model *model, const uint16_t *X, int M, const int *agent_row_start,
                          int n_agents, int max_rows_per_agent, const int *lens, float *H_out,
                          void *ws, size_t ws_bytes, void *stream, qad_step_graph **out);
int qad_step_graph_launch(qad_step_graph *g, void *stream);
void qad_step_graph_destroy(qad_step_graph *g);

/* ---------------------------------------------------------------- mixed step (chunked prefill)
 * OpenJet page, section 真正重要的是少互相堵车: a long prompt is fed in chunks
 * so the other agents keep decoding. One mixed step runs the decode batch (M
 * rows, exactly as qad_decode_step) together with C prompt rows of one more
 * agent (chunk_agent, positions chunk_len .. chunk_len + C - 1 of its cache),
 * all R = M + C rows through the dense tensor-core GEMMs of the layer
 * definition above. The decode rows attend as in qad_decode_step; chunk row j
 * attends causally to keys 0 .. chunk_len + j of its agent (its own k, v are
 * appended first), i.e. the same definition with C rows.
 *   X       device bf16 [R][hidden]: the M decode rows (agent-major) then the C
 *           chunk rows, 16-byte aligned
 *   agent_row_start, lens  as qad_decode_step (ignored when M == 0); the chunk
 *           agent must have no decode rows in this step
 *   H_out   device fp32 [R][hidden], 16-byte aligned
 *   ws      qad_mixed_step_ws_bytes(model, M, C) bytes, 256-byte aligned
 * 0 <= M <= 16, C >= 0, M + C >= 1; bf16 KV caches only (the prompt-chunk
 * attention reads bf16). Precision: the dense GEMM's (fp16 weight tiles) and
 * the prefill attention's (bf16 probabilities) for every row. Synchronous
 * with respect to nothing: all launches go to `stream`. With
 * qad_model_set_debug, a buffer of qad_mixed_step_debug_bytes(model, M, C)
 * receives the per-layer intermediates in the qad_decode_step layout for R rows. */
size_t qad_mixed_step_ws_bytes(const qad_model *model, int M, int C);
size_t qad_mixed_step_debug_bytes(const qad_model *model, int M, int C);
int qad_mixed_step(qad_model *model, const uint16_t *X, int M, const int *agent_row_start, int n_agents,
                   int max_rows_per_agent, const int *lens, int chunk_agent, int chunk_len, int C, float *H_out,
                   void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------- step scheduler (host only)
 * OpenJet page: the agents' tokens and drafts share one weight stream
 * (section 只搬一次权重), a long prompt is fed in pieces so it does not stall
 * the others (section 真正重要的是少互相堵车), and an agent's cached context is
 * reused by its next request (time to first token). Plain host code, no CUDA.
 *
 * Policy: chunk_tokens prompt rows per chunk; in QAD_SCHED_INTERLEAVE mode a
 * chunk rides along with the decode rows on every (decode_steps_per_chunk+1)-th
 * step (every step when nobody decodes); QAD_SCHED_PREFILL_FIRST runs a
 * pending prompt's chunks alone, holding the decoding agents back (the
 * behaviour without chunked prefill, kept as the comparison). Decode rows:
 * one per decoding agent, then up to n_draft drafts each, within
 * max_decode_rows (<= 16); a round-robin start (step mod n_agents) rotates who
 * goes first when the budget is short. */
#define QAD_SCHED_INTERLEAVE 0
#define QAD_SCHED_PREFILL_FIRST 1
typedef struct {
    int chunk_tokens;
    int decode_steps_per_chunk;
    int max_decode_rows;
    int n_draft;
    int mode;
} qad_sched_policy;

/* One agent's host-side state (caller-owned). */
typedef struct {
    int len;          /* tokens in its KV cache */
    int prompt_left;  /* prompt tokens still to prefill (0: decoding) */
    int active;       /* 0: paused (e.g. waiting on a tool call) */
    int drafts;       /* draft tokens ready for its next decode step */
} qad_sched_agent;

/* Plan step number `step`: decode_rows[a] (host int [n_agents]) rows per
 * agent, the chunk's agent (-1: none) and row count. Returns M (the decode
 * rows) or a negative QAD_ERR_* code. */
int qad_sched_plan(const qad_sched_policy *policy, const qad_sched_agent *agents, int n_agents, long long step,
                   int *decode_rows, int *chunk_agent, int *chunk_rows);
/* Apply a planned step: a decoding agent with k accepted drafts (n_accept,
 * host int [n_agents] or NULL for none; clamped to its rows - 1) grows by
 * k + 1 and its drafts are spent; the chunk's agent grows by the chunk and its
 * prompt_left shrinks by it. Returns 0 or QAD_ERR_INVALID for a plan that does
 * not fit the states. */
int qad_sched_commit(qad_sched_agent *agents, int n_agents, const int *decode_rows, int chunk_agent,
                     int chunk_rows, const int *n_accept);
/* Prompt-lookup drafting: for n = max_ngram down to min_ngram, find the latest
 * earlier occurrence of the last n tokens of tokens[0..n_tokens) (one that is
 * followed by at least one token) and copy up to n_draft of the tokens that
 * followed it into drafts. Returns the number written (0 if no n-gram recurs). */
int qad_prompt_lookup(const int *tokens, int n_tokens, int min_ngram, int max_ngram, int n_draft, int *drafts);
/* Length of the common prefix of two token sequences: how much of an agent's
 * cached context a new request can keep (set len to it; the rest is prompt). */
int qad_common_prefix(const int *a, int na, const int *b, int nb);

/* Number of kernel launches one qad_decode_step issues (for accounting). */
int qad_decode_step_launches(const qad_model *model);

/* Teacher-forced checking aid. When a debug buffer of
 * qad_decode_step_debug_bytes(model, M) bytes is attached, every following
 * qad_decode_step also copies, per layer l, the intermediates x1 (bf16
 * [M][hidden]), qkv (fp32 [M][(n_qh+2 n_kvh) hd]), attention output (bf16
 * [M][n_qh hd]), h after the o projection (fp32 [M][hidden]), x2 (bf16),
 * gate|up (fp32 [M][2 inter]), silu(gate)*up (bf16 [M][inter]) and h after
 * the layer (fp32), each at a 256-byte aligned offset in that order, into
 * layer l's slice. The buffer must be 256-byte aligned. Pass dbg = NULL to
 * detach. Graph capture refuses a model
 * with a debug buffer attached. */
size_t qad_decode_step_debug_bytes(const qad_model *model, int M);
int qad_model_set_debug(qad_model *model, void *dbg, size_t bytes);

/* Per-launch event profiler. While enabled, every eager qad_decode_step records
 * a CUDA event before and after each of its launches (which serialises the
 * launch chain) and qad_model_profile_read() accumulates the elapsed times per
 * kernel class into ms[k], count[k] (k: 0 init, 1 prep (including the
 * attention split merge), 2 qkv GEMM, 3 attention (including the k/v append),
 * 4 o GEMM, 5 gate|up GEMM, 6 down GEMM; n_kinds >= 7) and returns the number
 * of classes. Read after every profiled
 * step (a step not read before the next one is dropped). Enabling resets the
 * totals. Graph capture refuses a model with the profiler on. */
/* Per-launch device trace (works in eager steps and in graphs captured while
 * it is attached). With a device buffer of 3 * n_records u64 attached, launch
 * k of each following step (k < n_records; launch order: init, then per layer
 * prep, qkv GEMM, attention, prep, o GEMM, prep, gate|up GEMM, prep, down
 * GEMM) records %globaltimer nanoseconds into words 3k..3k+2 with atomicMin:
 * the first CTA's start, the first CTA past its wait on the previous kernel,
 * and the bitwise NOT of the last warp's exit. Fill the buffer with 0xFF bytes
 * before a step. Pass buf = NULL to detach. Returns 0 or QAD_ERR_INVALID. */
int qad_model_set_trace(qad_model *model, unsigned long long *buf, int n_records);
int qad_model_set_profile(qad_model *model, int enable);
int qad_model_profile_read(qad_model *model, double *ms, long long *count, int n_kinds);

#ifdef __cplusplus
}
#endif
#endif /* QAD_H */
