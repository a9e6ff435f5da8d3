/*
 * qad_oracle.c -- plain, slow, fp64 CPU reference of the multi-agent
 * decode-and-verify step. TEST INFRASTRUCTURE ONLY: the tests, the package's
 * smoke check and the bench's CPU-baseline leg may load it; the product path
 * never does. It shares no code, header or table with the CUDA library.
 *
 * Sources (cited by page title and section heading):
 *   [OpenJet page]  rebasdaily.com, 2026-10-29, "OpenJet ... Qwen3.8-27B
 *                   multi-agent serving". Sections: intro (Q4_K_M weights, four
 *                   coding agents on one GPU); "妙处是只搬一次权重" (move the
 *                   weights once: 12 rows = 4 agents x (next token + 2 drafts),
 *                   one pass over the quantized weights shared by all rows,
 *                   drafts checked in the same pass, each agent reads its own
 *                   KV cache).
 *   [Q4_K/Q6_K]     The pages only name "Q4_K_M". The block layouts below are
 *                   the public GGUF Q4_K / Q6_K super-block conventions (256
 *                   weights per block; Q4_K: 8 sub-blocks of 32 with 6-bit
 *                   scales/mins and fp16 d/dmin; Q6_K: 16 sub-blocks of 16 with
 *                   int8 scales and fp16 d), restated here from their
 *                   definition.
 *   Readings where the pages are silent (RMSNorm with unit gain and eps 1e-6,
 *   no RoPE, rounding points of the layer glue, causal order of the draft
 *   rows) are the plainest ones and are listed in the design notes.
 *
 * Every function computes in double. Dequantised weights are exact in double
 * (at most 11+6+4 significant bits per product), so the GEMM reference is the
 * exact sum up to fp64 rounding of the accumulation.
 *
 * Parity pins: every function here is pinned by a -m "not gpu" test
 * (closed forms, brute force, the gguf library's dequantiser, torch's
 * attention routine on fp64). The 64-layer composition (orc_decode_layer
 * chained) is "parity unpinned" beyond its per-operation pins.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define QK 256
#define Q4K_BYTES 144
#define Q6K_BYTES 210

/* ------------------------------------------------------------------ formats */

/* IEEE 754 binary16 -> double (exact). */
double orc_half_to_double(uint16_t h)
{
    int s = h >> 15, e = (h >> 10) & 31, f = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);                /* subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f | 1024), e - 25);    /* (1024+f) * 2^(e-15-10) */
    return s ? -v : v;
}

/* bfloat16 (upper half of an IEEE binary32) -> double (exact). */
double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* double -> bfloat16, round to nearest, ties to even, directly from the double
 * (no intermediate float rounding). Overflow gives +-inf. */
uint16_t orc_double_to_bf16(double x)
{
    if (isnan(x))
        return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return sign | 0x7F80;
    int e;
    frexp(a, &e);                 /* a = f * 2^e, f in [0.5, 1) */
    int q = e - 8;                /* 8 significant bits: a = M * 2^q, M in [128, 256) */
    if (q < -133)
        q = -133;                 /* subnormal spacing of bf16 is 2^-133 */
    double M = ldexp(a, -q);      /* exact */
    double R = nearbyint(M);      /* default rounding mode: nearest, ties to even */
    double r = ldexp(R, q);
    if (r >= ldexp(1.0, 128))
        return sign | 0x7F80;
    float f = (float)r;           /* exact: r has <= 8 significant bits and is in range */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ Q4_K */

/* Decode one 144-byte Q4_K super-block.
 * Bytes [0:2] d (fp16 LE), [2:4] dmin (fp16 LE), [4:16] scales[12],
 * [16:144] qs[128]. Sub-block j covers weights 32j..32j+31:
 *   j < 4 : sc_j = scales[j] & 63,  m_j = scales[j+4] & 63
 *   j >= 4: sc_j = (scales[j+4] & 15) | (scales[j-4] >> 6) << 4
 *           m_j  = (scales[j+4] >> 4) | (scales[j]   >> 6) << 4
 * Quant byte qs[32p+l] holds weight 64p+l in its low nibble and weight
 * 64p+32+l in its high nibble (p = 0..3, l = 0..31). */
void orc_q4k_decode(const uint8_t *blk, uint8_t *q, uint8_t *sc, uint8_t *m,
                    uint16_t *d, uint16_t *dmin)
{
    const uint8_t *s = blk + 4, *qs = blk + 16;
    *d = (uint16_t)(blk[0] | blk[1] << 8);
    *dmin = (uint16_t)(blk[2] | blk[3] << 8);
    for (int j = 0; j < 8; ++j) {
        if (j < 4) {
            sc[j] = s[j] & 63;
            m[j] = s[j + 4] & 63;
        } else {
            sc[j] = (uint8_t)((s[j + 4] & 15) | ((s[j - 4] >> 6) << 4));
            m[j] = (uint8_t)((s[j + 4] >> 4) | ((s[j] >> 6) << 4));
        }
    }
    for (int p = 0; p < 4; ++p)
        for (int l = 0; l < 32; ++l) {
            q[64 * p + l] = qs[32 * p + l] & 15;
            q[64 * p + 32 + l] = qs[32 * p + l] >> 4;
        }
}

/* Inverse of orc_q4k_decode (q in 0..15, sc and m in 0..63). */
void orc_q4k_encode(const uint8_t *q, const uint8_t *sc, const uint8_t *m,
                    uint16_t d, uint16_t dmin, uint8_t *blk)
{
    uint8_t *s = blk + 4, *qs = blk + 16;
    blk[0] = d & 255;
    blk[1] = d >> 8;
    blk[2] = dmin & 255;
    blk[3] = dmin >> 8;
    memset(s, 0, 12);
    for (int j = 0; j < 8; ++j) {
        if (j < 4) {
            s[j] |= sc[j] & 63;
            s[j + 4] |= m[j] & 63;
        } else {
            s[j + 4] = (uint8_t)((sc[j] & 15) | ((m[j] & 15) << 4));
            s[j - 4] |= (uint8_t)((sc[j] >> 4) << 6);
            s[j] |= (uint8_t)((m[j] >> 4) << 6);
        }
    }
    for (int p = 0; p < 4; ++p)
        for (int l = 0; l < 32; ++l)
            qs[32 * p + l] = (uint8_t)((q[64 * p + l] & 15) | ((q[64 * p + 32 + l] & 15) << 4));
}

/* w_i = d * sc_{i/32} * q_i - dmin * m_{i/32}, exact in double. */
void orc_q4k_dequant_block(const uint8_t *blk, double *w)
{
    uint8_t q[QK], sc[8], m[8];
    uint16_t d, dmin;
    orc_q4k_decode(blk, q, sc, m, &d, &dmin);
    double dd = orc_half_to_double(d), dm = orc_half_to_double(dmin);
    for (int i = 0; i < QK; ++i)
        w[i] = dd * sc[i / 32] * q[i] - dm * m[i / 32];
}

/* ------------------------------------------------------------------ Q6_K */

/* Decode one 210-byte Q6_K-like block: [0:128] ql, [128:192] qh,
 * [192:208] int8 scales[16], [208:210] d (fp16 LE). For half h (weights
 * 128h..128h+127) and l = 0..31, with L = ql + 64h and H = qh + 32h:
 *   q[128h+l]    = (L[l]    & 15) | ((H[l]      & 3) << 4)
 *   q[128h+l+32] = (L[l+32] & 15) | ((H[l] >> 2 & 3) << 4)
 *   q[128h+l+64] = (L[l]    >> 4) | ((H[l] >> 4 & 3) << 4)
 *   q[128h+l+96] = (L[l+32] >> 4) | ((H[l] >> 6 & 3) << 4) */
void orc_q6k_decode(const uint8_t *blk, uint8_t *q, int8_t *sc, uint16_t *d)
{
    for (int h = 0; h < 2; ++h) {
        const uint8_t *L = blk + 64 * h, *H = blk + 128 + 32 * h;
        for (int l = 0; l < 32; ++l) {
            q[128 * h + l] = (uint8_t)((L[l] & 15) | ((H[l] & 3) << 4));
            q[128 * h + l + 32] = (uint8_t)((L[l + 32] & 15) | (((H[l] >> 2) & 3) << 4));
            q[128 * h + l + 64] = (uint8_t)((L[l] >> 4) | (((H[l] >> 4) & 3) << 4));
            q[128 * h + l + 96] = (uint8_t)((L[l + 32] >> 4) | (((H[l] >> 6) & 3) << 4));
        }
    }
    for (int i = 0; i < 16; ++i)
        sc[i] = (int8_t)blk[192 + i];
    *d = (uint16_t)(blk[208] | blk[209] << 8);
}

/* Inverse of orc_q6k_decode (q in 0..63). */
void orc_q6k_encode(const uint8_t *q, const int8_t *sc, uint16_t d, uint8_t *blk)
{
    memset(blk, 0, Q6K_BYTES);
    for (int h = 0; h < 2; ++h) {
        uint8_t *L = blk + 64 * h, *H = blk + 128 + 32 * h;
        for (int l = 0; l < 32; ++l) {
            uint8_t a = q[128 * h + l], b = q[128 * h + l + 32];
            uint8_t c = q[128 * h + l + 64], e = q[128 * h + l + 96];
            L[l] = (uint8_t)((a & 15) | ((c & 15) << 4));
            L[l + 32] = (uint8_t)((b & 15) | ((e & 15) << 4));
            H[l] = (uint8_t)((a >> 4) | ((b >> 4) << 2) | ((c >> 4) << 4) | ((e >> 4) << 6));
        }
    }
    for (int i = 0; i < 16; ++i)
        blk[192 + i] = (uint8_t)sc[i];
    blk[208] = d & 255;
    blk[209] = d >> 8;
}

/* w_i = d * sc_{i/16} * (q_i - 32), exact in double. */
void orc_q6k_dequant_block(const uint8_t *blk, double *w)
{
    uint8_t q[QK];
    int8_t sc[16];
    uint16_t d;
    orc_q6k_decode(blk, q, sc, &d);
    double dd = orc_half_to_double(d);
    for (int i = 0; i < QK; ++i)
        w[i] = dd * sc[i / 16] * ((int)q[i] - 32);
}

/* fmt 4: Q4_K, fmt 6: Q6_K. Dequantise row-major matrix [N x K] to double. */
static void dequant_row(int fmt, const uint8_t *W, int K, int n, double *w)
{
    int nb = K / QK;
    if (fmt == 4) {
        const uint8_t *row = W + (size_t)n * nb * Q4K_BYTES;
        for (int b = 0; b < nb; ++b)
            orc_q4k_dequant_block(row + (size_t)b * Q4K_BYTES, w + (size_t)b * QK);
    } else {
        const uint8_t *row = W + (size_t)n * nb * Q6K_BYTES;
        for (int b = 0; b < nb; ++b)
            orc_q6k_dequant_block(row + (size_t)b * Q6K_BYTES, w + (size_t)b * QK);
    }
}

void orc_dequant_matrix(int fmt, const uint8_t *W, int N, int K, double *w)
{
    for (int n = 0; n < N; ++n)
        dequant_row(fmt, W, K, n, w + (size_t)n * K);
}

/* ------------------------------------------------------------------ GEMM */

/* Y[r][n] = sum_k w[n][k] * x[r][k]   (x: bf16 [M][K], natural k order)
 * A[r][n] = sum_k |w[n][k] * x[r][k]| (scale of the per-output tolerance).
 * This is the product the shared weight pass computes for all rows at once
 * ([OpenJet page], section 只搬一次权重). Rows n are independent. */
void orc_gemm(int fmt, const uint8_t *W, int N, int K, const uint16_t *X, int M,
              double *Y, double *A, int nthreads)
{
    double *xd = malloc(sizeof(double) * (size_t)M * K);
    for (size_t i = 0; i < (size_t)M * K; ++i)
        xd[i] = orc_bf16_to_double(X[i]);
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *w = malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(static)
        for (int n = 0; n < N; ++n) {
            dequant_row(fmt, W, K, n, w);
            for (int r = 0; r < M; ++r) {
                const double *x = xd + (size_t)r * K;
                double s = 0.0, a = 0.0;
                for (int k = 0; k < K; ++k) {
                    double p = w[k] * x[k];
                    s += p;
                    a += fabs(p);
                }
                Y[(size_t)r * N + n] = s;
                if (A)
                    A[(size_t)r * N + n] = a;
            }
        }
        free(w);
    }
    free(xd);
}

/* Same product for a subset of output rows (full-size sampled checks):
 * Y[r][i] = sum_k w[rows[i]][k] x[r][k], Y is [M][nrows]. */
void orc_gemm_rows(int fmt, const uint8_t *W, int K, const int *rows, int nrows,
                   const uint16_t *X, int M, double *Y, double *A)
{
    double *w = malloc(sizeof(double) * (size_t)K);
    for (int i = 0; i < nrows; ++i) {
        dequant_row(fmt, W, K, rows[i], w);
        for (int r = 0; r < M; ++r) {
            double s = 0.0, a = 0.0;
            for (int k = 0; k < K; ++k) {
                double p = w[k] * orc_bf16_to_double(X[(size_t)r * K + k]);
                s += p;
                a += fabs(p);
            }
            Y[(size_t)r * nrows + i] = s;
            if (A)
                A[(size_t)r * nrows + i] = a;
        }
    }
    free(w);
}

/* ------------------------------------------------------------------ attention */

/* Grouped-query decode attention over each agent's own KV cache
 * ([OpenJet page], section 只搬一次权重: every agent reads its own KV cache;
 * the draft rows are verified in the same pass).
 * Rows of agent a are r = ars[a] .. ars[a+1]-1; row j = r - ars[a] sits at
 * position lens[a] + j and sees keys t = 0 .. lens[a] + j (its cached context
 * plus the agent's new rows up to itself), so the rows reproduce one-at-a-time
 * decoding. q-head h reads kv-head g = h * n_kvh / n_qh.
 *   Q  bf16 [M][n_qh][hd];  Kc, Vc bf16 [n_agents][n_kvh][cap][hd]
 *   O  [M][n_qh][hd] = sum_t p_t v_t with p = softmax(scale * q.k_t)
 *   B  [M][n_qh][hd] = sum_t p_t |v_t|   (scale of the per-element tolerance) */
void orc_decode_attn(const uint16_t *Q, const uint16_t *Kc, const uint16_t *Vc,
                     const int *lens, const int *ars, int n_agents, int cap,
                     int n_qh, int n_kvh, int hd, double scale, double *O, double *B,
                     int nthreads)
{
    int M = ars[n_agents];
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *s = NULL;
        int s_cap = 0;
#pragma omp for schedule(dynamic) collapse(2)
        for (int r = 0; r < M; ++r)
            for (int h = 0; h < n_qh; ++h) {
                int a = 0;
                while (!(ars[a] <= r && r < ars[a + 1]))
                    ++a;
                int j = r - ars[a];
                int nk = lens[a] + j + 1;
                int g = h * n_kvh / n_qh;
                if (nk > s_cap) {
                    free(s);
                    s_cap = nk;
                    s = malloc(sizeof(double) * (size_t)s_cap);
                }
                const uint16_t *q = Q + ((size_t)r * n_qh + h) * hd;
                const uint16_t *kb = Kc + ((size_t)a * n_kvh + g) * (size_t)cap * hd;
                const uint16_t *vb = Vc + ((size_t)a * n_kvh + g) * (size_t)cap * hd;
                double mx = -INFINITY;
                for (int t = 0; t < nk; ++t) {
                    double dot = 0.0;
                    for (int d = 0; d < hd; ++d)
                        dot += orc_bf16_to_double(q[d]) * orc_bf16_to_double(kb[(size_t)t * hd + d]);
                    s[t] = scale * dot;
                    if (s[t] > mx)
                        mx = s[t];
                }
                double z = 0.0;
                for (int t = 0; t < nk; ++t) {
                    s[t] = exp(s[t] - mx);
                    z += s[t];
                }
                double *o = O + ((size_t)r * n_qh + h) * hd;
                double *bb = B ? B + ((size_t)r * n_qh + h) * hd : NULL;
                for (int d = 0; d < hd; ++d) {
                    double acc = 0.0, aabs = 0.0;
                    for (int t = 0; t < nk; ++t) {
                        double v = orc_bf16_to_double(vb[(size_t)t * hd + d]);
                        acc += s[t] * v;
                        aabs += s[t] * fabs(v);
                    }
                    o[d] = acc / z;
                    if (bb)
                        bb[d] = aabs / z;
                }
            }
        free(s);
    }
}

/* fp16 bits of x, rounded to nearest with ties to even (subnormals kept). */
uint16_t orc_double_to_half(double x)
{
    if (isnan(x))
        return 0x7E00;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e);                 /* a = f * 2^e, f in [0.5, 1) */
    int q = e - 11;               /* 11 significant bits: a = M * 2^q, M in [1024, 2048) */
    if (q < -24)
        q = -24;                  /* subnormal spacing of fp16 is 2^-24 */
    double R = nearbyint(ldexp(a, -q));
    double r = ldexp(R, q);
    if (r >= 65520.0)             /* rounds past the largest finite value 65504 */
        return sign | 0x7C00;
    /* encode r exactly */
    if (r < ldexp(1.0, -14))
        return sign | (uint16_t)(r * ldexp(1.0, 24));             /* subnormal: r / 2^-24 */
    int ex;
    double f = frexp(r, &ex);     /* r = f * 2^ex, f in [0.5, 1) */
    uint16_t mant = (uint16_t)(ldexp(f, 11) - 1024.0);             /* 10 fraction bits */
    return sign | (uint16_t)((ex - 1 + 15) << 10) | mant;
}

/* q8_0 quantisation of n values (n % 32 == 0), the GGUF q8_0 rule: per block of
 * 32 values d = amax / 127, q = round(x / d) (half away from zero) with the
 * reciprocal taken once, d stored as fp16. The code is decided in fp32 (the
 * kernel's precision): x, amax, d, 1/d and x * (1/d) are all fp32 operations.
 * Used for the q8_0 KV-cache variant (dual-4090 page, section 真正昂贵的是
 * "同时记住": llama.cpp's q8_0 KV cache per agent). */
void orc_q8_0_quantize(const float *x, long n, int8_t *q, uint16_t *d)
{
    for (long b = 0; b < n / 32; ++b) {
        float amax = 0.0f;
        for (int i = 0; i < 32; ++i) {
            float v = fabsf(x[32 * b + i]);
            if (v > amax)
                amax = v;
        }
        float dF = amax / 127.0f;
        float id = dF != 0.0f ? 1.0f / dF : 0.0f;
        for (int i = 0; i < 32; ++i)
            q[32 * b + i] = (int8_t)roundf(x[32 * b + i] * id);
        d[b] = orc_double_to_half((double)dF);
    }
}

/* Grouped-query attention of orc_decode_attn over a q8_0 cache: key/value
 * element (agent a, kv-head g, position t, dim k) = half(Kd[.., t, k / 32]) *
 * Kq[.., t, k] (exact in double). Kq, Vq int8 [A][n_kvh][cap][hd]; Kd, Vd fp16
 * [A][n_kvh][cap][hd / 32]. */
void orc_decode_attn_q8(const uint16_t *Q, const int8_t *Kq, const uint16_t *Kd, const int8_t *Vq,
                        const uint16_t *Vd, const int *lens, const int *ars, int n_agents, int cap, int n_qh,
                        int n_kvh, int hd, double scale, double *O, double *B, int nthreads)
{
    int M = ars[n_agents];
    const int nb = hd / 32;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *s = NULL;
        int s_cap = 0;
#pragma omp for schedule(dynamic) collapse(2)
        for (int r = 0; r < M; ++r)
            for (int h = 0; h < n_qh; ++h) {
                int a = 0;
                while (!(ars[a] <= r && r < ars[a + 1]))
                    ++a;
                int j = r - ars[a];
                int nk = lens[a] + j + 1;
                int g = h * n_kvh / n_qh;
                if (nk > s_cap) {
                    free(s);
                    s_cap = nk;
                    s = malloc(sizeof(double) * (size_t)s_cap);
                }
                const uint16_t *q = Q + ((size_t)r * n_qh + h) * hd;
                const size_t hb = ((size_t)a * n_kvh + g) * (size_t)cap;
                double mx = -INFINITY;
                for (int t = 0; t < nk; ++t) {
                    double dot = 0.0;
                    for (int k = 0; k < hd; ++k)
                        dot += orc_bf16_to_double(q[k]) * orc_half_to_double(Kd[(hb + t) * nb + k / 32]) *
                               (double)Kq[(hb + t) * hd + k];
                    s[t] = scale * dot;
                    if (s[t] > mx)
                        mx = s[t];
                }
                double z = 0.0;
                for (int t = 0; t < nk; ++t) {
                    s[t] = exp(s[t] - mx);
                    z += s[t];
                }
                double *o = O + ((size_t)r * n_qh + h) * hd;
                double *bb = B ? B + ((size_t)r * n_qh + h) * hd : NULL;
                for (int k = 0; k < hd; ++k) {
                    double acc = 0.0, aabs = 0.0;
                    for (int t = 0; t < nk; ++t) {
                        double v = orc_half_to_double(Vd[(hb + t) * nb + k / 32]) * (double)Vq[(hb + t) * hd + k];
                        acc += s[t] * v;
                        aabs += s[t] * fabs(v);
                    }
                    o[k] = acc / z;
                    if (bb)
                        bb[k] = aabs / z;
                }
            }
        free(s);
    }
}

/* ------------------------------------------------------------------ glue */

/* RMSNorm with unit gain, then bf16: out = bf16(h / sqrt(mean(h^2) + eps)). */
void orc_rmsnorm_bf16(const double *h, int M, int H, double eps, uint16_t *out)
{
    for (int r = 0; r < M; ++r) {
        const double *x = h + (size_t)r * H;
        double ss = 0.0;
        for (int i = 0; i < H; ++i)
            ss += x[i] * x[i];
        double inv = 1.0 / sqrt(ss / H + eps);
        for (int i = 0; i < H; ++i)
            out[(size_t)r * H + i] = orc_double_to_bf16(x[i] * inv);
    }
}

/* out = bf16(silu(g) * u), silu(g) = g / (1 + exp(-g)). */
void orc_silu_mul_bf16(const double *g, const double *u, long n, uint16_t *out)
{
    for (long i = 0; i < n; ++i)
        out[i] = orc_double_to_bf16(g[i] / (1.0 + exp(-g[i])) * u[i]);
}

/* Row packer: stack every agent's rows (next token + drafts) agent-major into
 * one batch ([OpenJet page], section 只搬一次权重: all active agents' work is
 * stacked into one batch of 12 rows). Agents with zero rows (paused for a
 * tool call) contribute nothing.
 *   rows[a]: bf16 [n_rows[a]][H];  lens[a]: cached tokens before the step
 * Outputs: X [M][H], row_agent[M], row_pos[M] = lens[a] + j,
 * agent_row_start[n_agents+1]. Returns M. */
int orc_pack_rows(const uint16_t *const *rows, const int *n_rows, const int *lens,
                  int n_agents, int H, uint16_t *X, int *row_agent, int *row_pos,
                  int *agent_row_start)
{
    int r = 0;
    for (int a = 0; a < n_agents; ++a) {
        agent_row_start[a] = r;
        for (int j = 0; j < n_rows[a]; ++j, ++r) {
            memcpy(X + (size_t)r * H, rows[a] + (size_t)j * H, sizeof(uint16_t) * H);
            row_agent[r] = a;
            row_pos[r] = lens[a] + j;
        }
    }
    agent_row_start[n_agents] = r;
    return r;
}

/* First index of the largest value (ties resolve to the lowest index). */
long orc_argmax(const double *v, long n)
{
    long best = 0;
    for (long i = 1; i < n; ++i)
        if (v[i] > v[best])
            best = i;
    return best;
}

/* Greedy verification of the drafts and commit of the KV lengths
 * ([OpenJet page], section 只搬一次权重: the two draft tokens of every agent
 * are checked in the same forward pass as its next token). The pages do not
 * state the acceptance rule; the reading taken is greedy: row j of an agent
 * (position lens[a] + j, input token row_tokens[r0 + j]) predicts
 * row_argmax[r0 + j]; draft j + 1 (the input of row j + 1) is accepted iff
 * every earlier draft was and row_argmax[r0 + j] == row_tokens[r0 + j + 1].
 * With k drafts accepted the agent emits row_argmax[r0 .. r0 + k] (k + 1
 * tokens: the accepted drafts and the next token after them), its cache holds
 * valid keys up to position lens[a] + k, so lens[a] += k + 1; the rows after
 * r0 + k are rejected (their cache slots are overwritten by the next step).
 *   out_tokens[r]: the emitted token of row r, or -1 for rejected rows
 *   n_accept[a]:   k (agents with no rows: 0, lens unchanged) */
void orc_accept_greedy(const int *row_argmax, const int *row_tokens, const int *ars, int n_agents, int *lens,
                       int *out_tokens, int *n_accept)
{
    for (int a = 0; a < n_agents; ++a) {
        const int r0 = ars[a], n = ars[a + 1] - ars[a];
        int k = 0;
        while (k + 1 < n && row_argmax[r0 + k] == row_tokens[r0 + k + 1])
            ++k;
        for (int j = 0; j < n; ++j)
            out_tokens[r0 + j] = j <= k ? row_argmax[r0 + j] : -1;
        n_accept[a] = n > 0 ? k : 0;
        if (n > 0)
            lens[a] += k + 1;
    }
}

/* One decoder layer of the synthetic stack for the packed batch, with the
 * rounding points of the design notes:
 *   x1  = bf16(rmsnorm(h))
 *   qkv = x1 . Wqkv^T            (rows: q [n_qh*hd], k [n_kvh*hd], v [n_kvh*hd])
 *   Q   = bf16(q); K/V of every row appended as bf16 at its position
 *   o   = attention(Q, caches);  ob = bf16(o)
 *   h   = h + ob . Wo^T
 *   x2  = bf16(rmsnorm(h))
 *   gu  = x2 . Wgu^T             (rows: gate [I], up [I])
 *   act = bf16(silu(gate) * up)
 *   h   = h + act . Wdown^T      (Q6_K)
 * h is the fp64 residual stream [M][H], updated in place. The caches are
 * updated in place. Intermediates are returned when the pointers are non-null
 * (used by teacher-forced checks). */
/* KV cache of one layer: bf16 planes, or q8_0 codes plus fp16 scales. */
typedef struct {
    int q8;
    uint16_t *Kc, *Vc;             /* bf16 [A][n_kvh][cap][hd] */
    int8_t *Kq, *Vq;               /* q8_0 codes [A][n_kvh][cap][hd] */
    uint16_t *Kd, *Vd;             /* q8_0 scales [A][n_kvh][cap][hd/32] */
} orc_kv;

static void decode_layer_impl(const uint8_t *Wqkv, const uint8_t *Wo, const uint8_t *Wgu,
                              const uint8_t *Wdown, int H, int I, int n_qh, int n_kvh, int hd,
                              double eps, double *h, int M, const int *ars, int n_agents,
                              const int *lens, orc_kv kv, int cap, int nthreads,
                              uint16_t *x1_out, double *qkv_out, uint16_t *attn_out,
                              double *hmid_out, uint16_t *x2_out, double *gu_out, uint16_t *act_out)
{
    int nq = n_qh * hd, nkv = n_kvh * hd, nqkv = nq + 2 * nkv;
    uint16_t *x1 = malloc(sizeof(uint16_t) * (size_t)M * H);
    double *qkv = malloc(sizeof(double) * (size_t)M * nqkv);
    uint16_t *Qb = malloc(sizeof(uint16_t) * (size_t)M * nq);
    double *o = malloc(sizeof(double) * (size_t)M * nq);
    uint16_t *ob = malloc(sizeof(uint16_t) * (size_t)M * nq);
    double *y = malloc(sizeof(double) * (size_t)M * (2 * (size_t)I > (size_t)H ? 2 * (size_t)I : (size_t)H));
    uint16_t *x2 = malloc(sizeof(uint16_t) * (size_t)M * H);
    uint16_t *act = malloc(sizeof(uint16_t) * (size_t)M * I);

    orc_rmsnorm_bf16(h, M, H, eps, x1);
    orc_gemm(4, Wqkv, nqkv, H, x1, M, qkv, NULL, nthreads);
    for (int r = 0; r < M; ++r) {
        int a = 0;
        while (!(ars[a] <= r && r < ars[a + 1]))
            ++a;
        int pos = lens[a] + (r - ars[a]);
        for (int i = 0; i < nq; ++i)
            Qb[(size_t)r * nq + i] = orc_double_to_bf16(qkv[(size_t)r * nqkv + i]);
        for (int g = 0; g < n_kvh; ++g) {
            size_t row = ((size_t)a * n_kvh + g) * cap + pos;
            if (!kv.q8) {
                for (int d = 0; d < hd; ++d) {
                    kv.Kc[row * hd + d] = orc_double_to_bf16(qkv[(size_t)r * nqkv + nq + g * hd + d]);
                    kv.Vc[row * hd + d] = orc_double_to_bf16(qkv[(size_t)r * nqkv + nq + nkv + g * hd + d]);
                }
            } else {
                /* q8_0 append: the fp32 projection row, 32-value blocks */
                float *kf = malloc(sizeof(float) * 2 * (size_t)hd), *vf = kf + hd;
                for (int d = 0; d < hd; ++d) {
                    kf[d] = (float)qkv[(size_t)r * nqkv + nq + g * hd + d];
                    vf[d] = (float)qkv[(size_t)r * nqkv + nq + nkv + g * hd + d];
                }
                orc_q8_0_quantize(kf, hd, kv.Kq + row * hd, kv.Kd + row * (hd / 32));
                orc_q8_0_quantize(vf, hd, kv.Vq + row * hd, kv.Vd + row * (hd / 32));
                free(kf);
            }
        }
    }
    if (!kv.q8)
        orc_decode_attn(Qb, kv.Kc, kv.Vc, lens, ars, n_agents, cap, n_qh, n_kvh, hd,
                        1.0 / sqrt((double)hd), o, NULL, nthreads);
    else
        orc_decode_attn_q8(Qb, kv.Kq, kv.Kd, kv.Vq, kv.Vd, lens, ars, n_agents, cap, n_qh, n_kvh, hd,
                           1.0 / sqrt((double)hd), o, NULL, nthreads);
    for (size_t i = 0; i < (size_t)M * nq; ++i)
        ob[i] = orc_double_to_bf16(o[i]);
    orc_gemm(4, Wo, H, nq, ob, M, y, NULL, nthreads);
    for (size_t i = 0; i < (size_t)M * H; ++i)
        h[i] += y[i];
    if (hmid_out)
        memcpy(hmid_out, h, sizeof(double) * (size_t)M * H);
    orc_rmsnorm_bf16(h, M, H, eps, x2);
    orc_gemm(4, Wgu, 2 * I, H, x2, M, y, NULL, nthreads);
    if (gu_out)
        memcpy(gu_out, y, sizeof(double) * (size_t)M * 2 * I);
    for (int r = 0; r < M; ++r)
        orc_silu_mul_bf16(y + (size_t)r * 2 * I, y + (size_t)r * 2 * I + I, I, act + (size_t)r * I);
    orc_gemm(6, Wdown, H, I, act, M, y, NULL, nthreads);
    for (size_t i = 0; i < (size_t)M * H; ++i)
        h[i] += y[i];

    if (x1_out)
        memcpy(x1_out, x1, sizeof(uint16_t) * (size_t)M * H);
    if (qkv_out)
        memcpy(qkv_out, qkv, sizeof(double) * (size_t)M * nqkv);
    if (attn_out)
        memcpy(attn_out, ob, sizeof(uint16_t) * (size_t)M * nq);
    if (x2_out)
        memcpy(x2_out, x2, sizeof(uint16_t) * (size_t)M * H);
    if (act_out)
        memcpy(act_out, act, sizeof(uint16_t) * (size_t)M * I);
    free(x1);
    free(qkv);
    free(Qb);
    free(o);
    free(ob);
    free(y);
    free(x2);
    free(act);
}

/* One decoder layer over bf16 caches (the rounding points listed at the top). */
void orc_decode_layer(const uint8_t *Wqkv, const uint8_t *Wo, const uint8_t *Wgu,
                      const uint8_t *Wdown, int H, int I, int n_qh, int n_kvh, int hd,
                      double eps, double *h, int M, const int *ars, int n_agents,
                      const int *lens, uint16_t *Kc, uint16_t *Vc, int cap, int nthreads,
                      uint16_t *x1_out, double *qkv_out, uint16_t *attn_out,
                      double *hmid_out, uint16_t *x2_out, double *gu_out, uint16_t *act_out)
{
    orc_kv kv = {0, Kc, Vc, NULL, NULL, NULL, NULL};
    decode_layer_impl(Wqkv, Wo, Wgu, Wdown, H, I, n_qh, n_kvh, hd, eps, h, M, ars, n_agents, lens, kv,
                      cap, nthreads, x1_out, qkv_out, attn_out, hmid_out, x2_out, gu_out, act_out);
}

/* The same layer over a q8_0 cache: the new rows' k, v are the fp32 values of
 * the projection, quantised by orc_q8_0_quantize; attention dequantises. */
void orc_decode_layer_q8(const uint8_t *Wqkv, const uint8_t *Wo, const uint8_t *Wgu,
                         const uint8_t *Wdown, int H, int I, int n_qh, int n_kvh, int hd,
                         double eps, double *h, int M, const int *ars, int n_agents,
                         const int *lens, int8_t *Kq, uint16_t *Kd, int8_t *Vq, uint16_t *Vd, int cap,
                         int nthreads, uint16_t *x1_out, double *qkv_out, uint16_t *attn_out,
                         double *hmid_out, uint16_t *x2_out, double *gu_out, uint16_t *act_out)
{
    orc_kv kv = {1, NULL, NULL, Kq, Vq, Kd, Vd};
    decode_layer_impl(Wqkv, Wo, Wgu, Wdown, H, I, n_qh, n_kvh, hd, eps, h, M, ars, n_agents, lens, kv,
                      cap, nthreads, x1_out, qkv_out, attn_out, hmid_out, x2_out, gu_out, act_out);
}

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
