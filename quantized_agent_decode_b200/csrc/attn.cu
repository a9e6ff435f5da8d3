// attn.cu -- grouped-query decode attention of each agent's rows over that
// agent's own bf16 KV cache, split along the keys (flash-decoding style), then
// a log-sum-exp combine of the splits.
//
// [OpenJet page] = rebasdaily.com 2026-10-29, "OpenJet ... multi-agent
// serving", section 只搬一次权重: every agent reads its own KV cache, and the
// two draft rows are checked in the same pass as the next-token row. Row j of
// an agent sits at position len + j and sees keys 0..len+j, which is exactly
// what decoding the rows one at a time would see.
//
// Design (sm_100a): one CTA = (split of the agent's keys, group of up to 24
// query vectors, agent, kv-head). The query vectors of one kv-head are all of
// the agent's rows times the q-heads that share it (3 rows x 6 heads = 18).
// The products run on the tensor cores with keys in the MMA's M dimension:
//   S^T[key][q] = K Q^T      (A = K tile via ldmatrix, B = Q^T in registers)
//   O^T[d][q]  += V^T P^T    (A = V^T tile via ldmatrix.trans, B = P^T via movmatrix)
// so 18 query vectors pad to 24 (three n=8 tiles) instead of 32. Keys and
// values stream HBM -> shared memory with cp.async (3 stages per warp, XOR
// swizzled 16-byte chunks so ldmatrix is bank-conflict free). The softmax is
// online in fp32 (exp2 with the scale folded in); P enters the bf16 MMA as a
// hi + lo pair of bf16 values, so its rounding error is ~2^-17 relative.
#include "attn.cuh"

// Fewest keys one split of the decode attention covers (build-time tunable, multiple of 64).
#ifndef QAD_ATTN_MIN_SPLIT_KEYS
#define QAD_ATTN_MIN_SPLIT_KEYS 256
#endif

// CTAs per SM the short-cache plan aims for (build-time tunable).
#ifndef QAD_ATTN_SHORT_CTAS_PER_SM
#define QAD_ATTN_SHORT_CTAS_PER_SM 1
#endif

namespace qad {

constexpr int QG = ATT_QG;      // query vectors per CTA
constexpr int KT = 16;          // keys per tile (one MMA M tile)
constexpr int ATT_WARPS = 4;
constexpr int ATT_STAGES_LONG = 3;   // per-warp ring for long caches (two CTAs per SM)
constexpr int ATT_STAGES_SHORT = 6;  // short caches: a split's cached tiles all in flight at once
constexpr int TILE_BYTES = KT * 128 * 2;  // 4 KB (K) ; V follows
constexpr float M_SLACK = 8.f;            // scores may pass the reference maximum by 2^8
constexpr int PART_FLOATS = ATT_PART_FLOATS;

struct AttnArgs {
    const uint16_t *Q, *Kc, *Vc;   // standalone: bf16 Q [M][n_qh][128]
    const float *qkv;              // fused: fp32 q | k | v rows [M][ldqkv]
    uint16_t *Kw, *Vw;             // fused: the caches, written at the new positions
    int ldqkv;
    const int *lens, *ars;
    int n_kvh, kv_cap, n_qh, G, CH, n_rg, max_splits;
    float scale_log2;
    float *part;
    unsigned long long *trace;
};

__device__ __forceinline__ int swz(int key, int chunk) { return key * 256 + ((chunk ^ (key & 7)) << 4); }

// FUSED: Q and the new rows' k, v come from the fp32 projection (rounded to
// bf16 here, as the unfused path rounds them before the cache write); key
// positions len .. len+na-1 are taken from there instead of the cache, and the
// row-group-0 CTA of the split holding a new position writes it to the cache.
template <bool FUSED, int STAGES>
__global__ void __launch_bounds__(128, 2) k_decode_attn(AttnArgs p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int sp = blockIdx.x, rg = blockIdx.y, ag = blockIdx.z;
    const int a = ag / p.n_kvh, g = ag - a * p.n_kvh;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, gq = lane >> 2, c = lane & 3;
    trace_start(p.trace);
    pdl_trigger();
    // Agent offsets, lengths and the cached keys below len are constant for the
    // whole step, so they are read before waiting on the previous kernel; Q and
    // the new rows' k, v (fused form) only after it.
    const int r0 = p.ars[a], na = p.ars[a + 1] - r0;
    const int len = p.lens[a];
    const int R = na * p.G;
    const int q0 = rg * QG;
    if (q0 >= R) {
        trace_end(p.trace);
        return;
    }
    const int L = min(len + na, p.kv_cap);
    const int kbeg = sp * p.CH;
    if (kbeg >= L) {
        trace_end(p.trace);
        return;
    }
    const int kend = min(L, kbeg + p.CH);
    const size_t head_off = ((size_t)a * p.n_kvh + g) * (size_t)p.kv_cap * 128;
    const uint16_t *Kh = p.Kc + head_off, *Vh = p.Vc + head_off;

    float o[8][3][4];
#pragma unroll
    for (int dt = 0; dt < 8; ++dt)
#pragma unroll
        for (int nt = 0; nt < 3; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                o[dt][nt][e] = 0.f;
    float m[3][2], l[3][2];
#pragma unroll
    for (int nt = 0; nt < 3; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            m[nt][e] = -INFINITY;
            l[nt][e] = 0.f;
        }

    const int ntiles = (kend - kbeg + KT - 1) / KT;
    const int my = ntiles > w ? (ntiles - w + ATT_WARPS - 1) / ATT_WARPS : 0;
    uint8_t *wbuf = smem + (size_t)w * STAGES * 2 * TILE_BYTES;

    const int nq = p.n_qh * 128, nkv = p.n_kvh * 128;
    // per-lane constants of a full tile's copies: chunk (lane & 15) of keys lane/16 + 2i
    // (i = 0..7); keys 8 apart share the swizzle, so 4 offsets cover the 8 rows
    int cp_dst[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        cp_dst[i] = swz((lane >> 4) + 2 * i, lane & 15);
    const int cp_src = (lane >> 4) * 128 + (lane & 15) * 8;  // elements
    auto issue = [&](int it, uint8_t *st) {
        const int kb = kbeg + KT * (w + ATT_WARPS * it);
        if (!(FUSED && kb + KT > len) && kb + KT <= kend) {  // a full tile of cached keys
            const uint16_t *ks = Kh + (size_t)kb * 128 + cp_src, *vs = Vh + (size_t)kb * 128 + cp_src;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                cp_async16(st + cp_dst[i & 3] + (i >> 2) * 2048, ks + 256 * i);
                cp_async16(st + TILE_BYTES + cp_dst[i & 3] + (i >> 2) * 2048, vs + 256 * i);
            }
            return;
        }
        if (FUSED && kb + KT > len) {
            // tile reaches the new positions: cached keys below len, new rows from the projection
#pragma unroll 1
            for (int i = 0; i < 8; ++i) {
                const int idx = lane + 32 * i, kk = idx >> 4, ch = idx & 15, kp = kb + kk;
                if (kp < len || kp >= kend) {
                    const bool ok = kp < kend;
                    const size_t src = (size_t)(ok ? kp : 0) * 128 + ch * 8;
                    cp_async16_zfill(st + swz(kk, ch), Kh + src, ok);
                    cp_async16_zfill(st + TILE_BYTES + swz(kk, ch), Vh + src, ok);
                } else {
                    const float *row = p.qkv + (size_t)(r0 + kp - len) * p.ldqkv + nq + g * 128 + ch * 8;
                    const float4 k0 = *reinterpret_cast<const float4 *>(row);
                    const float4 k1 = *reinterpret_cast<const float4 *>(row + 4);
                    const float4 v0 = *reinterpret_cast<const float4 *>(row + nkv);
                    const float4 v1 = *reinterpret_cast<const float4 *>(row + nkv + 4);
                    const uint4 kw = make_uint4(pack_bf162(k0.x, k0.y), pack_bf162(k0.z, k0.w),
                                                pack_bf162(k1.x, k1.y), pack_bf162(k1.z, k1.w));
                    const uint4 vw = make_uint4(pack_bf162(v0.x, v0.y), pack_bf162(v0.z, v0.w),
                                                pack_bf162(v1.x, v1.y), pack_bf162(v1.z, v1.w));
                    *reinterpret_cast<uint4 *>(st + swz(kk, ch)) = kw;
                    *reinterpret_cast<uint4 *>(st + TILE_BYTES + swz(kk, ch)) = vw;
                    if (rg == 0) {
                        const size_t dst = head_off + (size_t)kp * 128 + ch * 8;
                        *reinterpret_cast<uint4 *>(p.Kw + dst) = kw;
                        *reinterpret_cast<uint4 *>(p.Vw + dst) = vw;
                    }
                }
            }
            return;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int idx = lane + 32 * i, kk = idx >> 4, ch = idx & 15;
            const bool ok = kb + kk < kend;
            const size_t src = (size_t)(ok ? kb + kk : 0) * 128 + ch * 8;
            cp_async16_zfill(st + swz(kk, ch), Kh + src, ok);
            cp_async16_zfill(st + TILE_BYTES + swz(kk, ch), Vh + src, ok);
        }
    };
    // tiles of cached keys only (always the earlier ones) stream before the wait
    auto cached_tile = [&](int it) { return !FUSED || kbeg + KT * (w + ATT_WARPS * it) + KT <= len; };
    auto stage = [&](int i) { return wbuf + (size_t)i * 2 * TILE_BYTES; };
    int pre = 0;
    while (pre < STAGES - 1 && pre < my && cached_tile(pre)) {
        issue(pre, stage(pre));
        cp_async_commit();
        ++pre;
    }
    pdl_wait();
    trace_ready(p.trace);
    for (int it = pre; it < STAGES - 1; ++it) {
        if (it < my)
            issue(it, stage(it));
        cp_async_commit();
    }

    // Q^T fragments: b0 = Q[q][16ks+2c..], b1 = Q[q][16ks+8+2c..] for q = q0 + 8nt + gq
    uint32_t qf[3][8][2];
    int qpos[3][2];  // last visible key of the two query columns this lane owns (per nt)
#pragma unroll
    for (int nt = 0; nt < 3; ++nt) {
        const int qi = q0 + 8 * nt + gq;
        const bool ok = qi < R;
        const int j = ok ? qi / p.G : 0, hl = ok ? qi - j * p.G : 0;
        if (FUSED) {
            const float *qrow = p.qkv + (size_t)(r0 + j) * p.ldqkv + (g * p.G + hl) * 128;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const float2 f0 = ok ? *reinterpret_cast<const float2 *>(qrow + 16 * ks + 2 * c) : make_float2(0.f, 0.f);
                const float2 f1 = ok ? *reinterpret_cast<const float2 *>(qrow + 16 * ks + 8 + 2 * c) : make_float2(0.f, 0.f);
                qf[nt][ks][0] = pack_bf162(f0.x, f0.y);
                qf[nt][ks][1] = pack_bf162(f1.x, f1.y);
            }
        } else {
            const uint16_t *qrow = p.Q + ((size_t)(r0 + j) * p.n_qh + g * p.G + hl) * 128;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                qf[nt][ks][0] = ok ? *reinterpret_cast<const uint32_t *>(qrow + 16 * ks + 2 * c) : 0u;
                qf[nt][ks][1] = ok ? *reinterpret_cast<const uint32_t *>(qrow + 16 * ks + 8 + 2 * c) : 0u;
            }
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int qc = q0 + 8 * nt + 2 * c + e;
            qpos[nt][e] = qc < R ? len + qc / p.G : -1;
        }
    }


    int cur = 0, nxt = STAGES - 1;  // ring slots of tile it and of tile it + STAGES - 1
    for (int it = 0; it < my; ++it) {
        if (it + STAGES - 1 < my)
            issue(it + STAGES - 1, stage(nxt));
        nxt = nxt + 1 == STAGES ? 0 : nxt + 1;
        cp_async_commit();
        cp_async_wait<STAGES - 1>();
        __syncwarp();
        const uint8_t *Ks = stage(cur);
        cur = cur + 1 == STAGES ? 0 : cur + 1;
        const uint8_t *Vs = Ks + TILE_BYTES;
        const int kb = kbeg + KT * (w + ATT_WARPS * it);

        float s[3][4];
#pragma unroll
        for (int nt = 0; nt < 3; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                s[nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t a0, a1, a2, a3;
            const int key = (lane & 7) + 8 * ((lane >> 3) & 1), ch = 2 * ks + (lane >> 4);
            ldsm_x4(a0, a1, a2, a3, Ks + swz(key, ch));
#pragma unroll
            for (int nt = 0; nt < 3; ++nt)
                mma_bf16(s[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
        }
        // Online softmax against a reference maximum m per query column that moves only
        // when a score passes it by more than M_SLACK (log2 units), so most tiles need no
        // cross-lane reduction and no rescale (P <= 2^8, far inside bf16's range; the
        // reference cancels in every merge). Masks only on tiles past the cached keys.
        const bool interior = kb + KT <= kend && kb + KT <= len;
        float v[3][4];
        bool over = false;
#pragma unroll
        for (int nt = 0; nt < 3; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float v0 = s[nt][e] * p.scale_log2, v1 = s[nt][e + 2] * p.scale_log2;
                if (!interior) {
                    const int k0 = kb + gq, k1 = kb + gq + 8;
                    v0 = (k0 < kend && k0 <= qpos[nt][e]) ? v0 : -INFINITY;
                    v1 = (k1 < kend && k1 <= qpos[nt][e]) ? v1 : -INFINITY;
                }
                over |= fmaxf(v0, v1) > m[nt][e] + M_SLACK;
                v[nt][e] = v0;
                v[nt][e + 2] = v1;
            }
        if (__any_sync(0xffffffffu, over)) {
#pragma unroll
            for (int nt = 0; nt < 3; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float mx = fmaxf(v[nt][e], v[nt][e + 2]);
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    const float mn = fmaxf(m[nt][e], mx);
                    const float corr = mn == -INFINITY ? 1.f : ex2_approx(m[nt][e] - mn);
                    m[nt][e] = mn;
                    l[nt][e] *= corr;
#pragma unroll
                    for (int dt = 0; dt < 8; ++dt) {
                        o[dt][nt][e] *= corr;
                        o[dt][nt][e + 2] *= corr;
                    }
                }
        }
        uint32_t bh[3][2], bl[3][2];
#pragma unroll
        for (int nt = 0; nt < 3; ++nt) {
            float pv[4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const bool none = m[nt][e] == -INFINITY;
                pv[e] = none ? 0.f : ex2_approx(v[nt][e] - m[nt][e]);
                pv[e + 2] = none ? 0.f : ex2_approx(v[nt][e + 2] - m[nt][e]);
                l[nt][e] += pv[e] + pv[e + 2];
            }
            // P^T fragment (keys x queries) via an in-register transpose, as bf16 hi + lo
            const uint32_t h0 = pack_bf162(pv[0], pv[1]), h1 = pack_bf162(pv[2], pv[3]);
            const uint32_t l0 = pack_bf162(pv[0] - bf16_to_f((uint16_t)(h0 & 0xFFFF)),
                                           pv[1] - bf16_to_f((uint16_t)(h0 >> 16)));
            const uint32_t l1 = pack_bf162(pv[2] - bf16_to_f((uint16_t)(h1 & 0xFFFF)),
                                           pv[3] - bf16_to_f((uint16_t)(h1 >> 16)));
            bh[nt][0] = movmatrix_t(h0);
            bh[nt][1] = movmatrix_t(h1);
            bl[nt][0] = movmatrix_t(l0);
            bl[nt][1] = movmatrix_t(l1);
        }
#pragma unroll
        for (int dt = 0; dt < 8; ++dt) {
            uint32_t a0, a1, a2, a3;
            const int key = (lane & 7) + 8 * (lane >> 4), ch = 2 * dt + ((lane >> 3) & 1);
            ldsm_x4_t(a0, a1, a2, a3, Vs + swz(key, ch));
#pragma unroll
            for (int nt = 0; nt < 3; ++nt) {
                mma_bf16(o[dt][nt], a0, a1, a2, a3, bh[nt][0], bh[nt][1]);
                mma_bf16(o[dt][nt], a0, a1, a2, a3, bl[nt][0], bl[nt][1]);
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();

    // row sums over the 8 lanes sharing a query column
#pragma unroll
    for (int nt = 0; nt < 3; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float v = l[nt][e];
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            l[nt][e] = v;
        }
    __syncthreads();  // all warps done with their stages: reuse shared memory
    float *sO = reinterpret_cast<float *>(smem);          // [4][QG][128]
    float *sM = sO + ATT_WARPS * QG * 128;                // [4][QG]
    float *sL = sM + ATT_WARPS * QG;                      // [4][QG]
#pragma unroll
    for (int dt = 0; dt < 8; ++dt)
#pragma unroll
        for (int nt = 0; nt < 3; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int d = 16 * dt + gq + 8 * (e >> 1), q = 8 * nt + 2 * c + (e & 1);
                sO[((size_t)w * QG + q) * 128 + d] = o[dt][nt][e];
            }
    if (gq == 0) {
#pragma unroll
        for (int nt = 0; nt < 3; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                sM[w * QG + 8 * nt + 2 * c + e] = m[nt][e];
                sL[w * QG + 8 * nt + 2 * c + e] = l[nt][e];
            }
    }
    __syncthreads();
    const size_t pidx = (((size_t)a * p.n_kvh + g) * p.n_rg + rg) * p.max_splits + sp;
    float *out = p.part + pidx * PART_FLOATS;
    const int nqv = min(QG, R - q0);  // real query vectors of this group (the rest is padding)
    for (int idx = tid; idx < nqv * 128; idx += blockDim.x) {
        const int q = idx >> 7;
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < ATT_WARPS; ++ww)
            M = fmaxf(M, sM[ww * QG + q]);
        float acc = 0.f;
        if (M != -INFINITY)
#pragma unroll
            for (int ww = 0; ww < ATT_WARPS; ++ww)
                acc += exp2f(sM[ww * QG + q] - M) * sO[((size_t)ww * QG + q) * 128 + (idx & 127)];
        out[idx] = acc;
    }
    if (tid < nqv) {
        float M = -INFINITY, Lsum = 0.f;
        for (int ww = 0; ww < ATT_WARPS; ++ww)
            M = fmaxf(M, sM[ww * QG + tid]);
        if (M != -INFINITY)
            for (int ww = 0; ww < ATT_WARPS; ++ww)
                Lsum += exp2f(sM[ww * QG + tid] - M) * sL[ww * QG + tid];
        out[QG * 128 + tid] = M;
        out[QG * 128 + QG + tid] = Lsum;
    }
    trace_end(p.trace);
}

// One CTA per (query vector, row group, agent*kv-head); thread = dimension.
__global__ void __launch_bounds__(128) k_attn_combine(AttnArgs p, uint16_t *O)
{
    const int q = blockIdx.x, rg = blockIdx.y, ag = blockIdx.z;
    const int a = ag / p.n_kvh, g = ag - a * p.n_kvh;
    const int d = threadIdx.x;
    pdl_trigger();
    pdl_wait();
    const int r0 = p.ars[a], na = p.ars[a + 1] - r0;
    const int R = na * p.G;
    const int qi = rg * QG + q;
    if (qi >= R)
        return;
    const int L = min(p.lens[a] + na, p.kv_cap);
    const int nsp = (L + p.CH - 1) / p.CH;
    const size_t base = (((size_t)a * p.n_kvh + g) * p.n_rg + rg) * p.max_splits;
    float M = -INFINITY;
    for (int s = 0; s < nsp; ++s)
        M = fmaxf(M, p.part[(base + s) * PART_FLOATS + QG * 128 + q]);
    float acc = 0.f, Ls = 0.f;
    if (M != -INFINITY)
        for (int s = 0; s < nsp; ++s) {
            const float *pp = p.part + (base + s) * PART_FLOATS;
            const float wgt = exp2f(pp[QG * 128 + q] - M);
            acc += wgt * pp[q * 128 + d];
            Ls += wgt * pp[QG * 128 + QG + q];
        }
    const int j = qi / p.G, hl = qi - j * p.G;
    O[((size_t)(r0 + j) * p.n_qh + g * p.G + hl) * 128 + d] = f_to_bf16(Ls > 0.f ? acc / Ls : 0.f);
}

// ------------------------------------------------------------- host side

AttnPlan attn_plan(int n_agents, int n_qh, int n_kvh, int kv_cap, int max_rows_per_agent)
{
    AttnPlan pl;
    pl.G = n_qh / n_kvh;
    pl.n_rg = (max_rows_per_agent * pl.G + QG - 1) / QG;
    // one wave: two resident CTAs per SM (registers and shared memory allow two)
    const int pairs = n_agents * n_kvh * pl.n_rg;
    // Short caches: at most one CTA per SM, and the split small enough that each
    // warp's tiles (16 keys each, 4 warps) all fit its 6-stage ring, so every
    // cached key is in flight before the kernel waits for its queries.
    {
        int sp = QAD_ATTN_SHORT_CTAS_PER_SM * num_sms() / pairs;
        if (sp < 1)
            sp = 1;
        int ch = (kv_cap + sp - 1) / sp;
        ch = ((ch + 63) / 64) * 64;
        // two CTAs per SM only fit with the 3-deep ring
        const int st = QAD_ATTN_SHORT_CTAS_PER_SM > 1 ? ATT_STAGES_LONG : ATT_STAGES_SHORT;
        if ((ch / KT + ATT_WARPS - 1) / ATT_WARPS <= st - 1) {
            pl.CH = ch;
            pl.stages = st;
            pl.max_splits = (kv_cap + ch - 1) / ch;
            pl.part_bytes = (size_t)n_agents * n_kvh * pl.n_rg * pl.max_splits * PART_FLOATS * sizeof(float);
            return pl;
        }
    }
    pl.stages = ATT_STAGES_LONG;
    const int target = 2 * num_sms();
    int splits = target / pairs;
    if (splits < 1)
        splits = 1;
    int ch = (kv_cap + splits - 1) / splits;
    ch = ((ch + 63) / 64) * 64;
    if (ch < QAD_ATTN_MIN_SPLIT_KEYS)  // short caches: fewer, longer splits (less partial traffic)
        ch = QAD_ATTN_MIN_SPLIT_KEYS;
    pl.CH = ch;
    pl.max_splits = (kv_cap + ch - 1) / ch;
    pl.part_bytes = (size_t)n_agents * n_kvh * pl.n_rg * pl.max_splits * PART_FLOATS * sizeof(float);
    return pl;
}

size_t attn_smem_bytes(int nstages)
{
    const size_t stages = (size_t)ATT_WARPS * nstages * 2 * TILE_BYTES;
    const size_t merge = ((size_t)ATT_WARPS * QG * 128 + 2 * ATT_WARPS * QG) * sizeof(float);
    return stages > merge ? stages : merge;
}

template <bool FUSED, int STAGES>
static int launch_split_kernel_t(const AttnPlan &pl, const AttnArgs &p, int n_agents, cudaStream_t s, bool pdl)
{
    const size_t smem = attn_smem_bytes(STAGES);
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        int rc = cuda_check(
            cudaFuncSetAttribute(k_decode_attn<FUSED, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
            "cudaFuncSetAttribute(attn)");
        if (rc)
            return rc;
        if (dev >= 0 && dev < 64)
            attr_set[dev] = true;
    }
    dim3 grid(pl.max_splits, pl.n_rg, n_agents * p.n_kvh);
    cudaError_t e = pdl ? launch_pdl(k_decode_attn<FUSED, STAGES>, grid, dim3(128), smem, s, p)
                        : (k_decode_attn<FUSED, STAGES><<<grid, 128, smem, s>>>(p), cudaGetLastError());
    return cuda_check(e, "attn launch");
}

template <bool FUSED>
static int launch_split_kernel(const AttnPlan &pl, const AttnArgs &p, int n_agents, cudaStream_t s, bool pdl)
{
    return pl.stages == ATT_STAGES_SHORT ? launch_split_kernel_t<FUSED, ATT_STAGES_SHORT>(pl, p, n_agents, s, pdl)
                                         : launch_split_kernel_t<FUSED, ATT_STAGES_LONG>(pl, p, n_agents, s, pdl);
}

static AttnArgs attn_args(const AttnPlan &pl, const int *lens, const int *ars, int kv_cap, int n_qh, int n_kvh,
                          float scale, float *part)
{
    AttnArgs p = {};
    p.lens = lens;
    p.ars = ars;
    p.n_kvh = n_kvh;
    p.kv_cap = kv_cap;
    p.n_qh = n_qh;
    p.G = pl.G;
    p.CH = pl.CH;
    p.n_rg = pl.n_rg;
    p.max_splits = pl.max_splits;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.part = part;
    return p;
}

int launch_attn_fused(const AttnPlan &pl, const float *qkv, int ldqkv, uint16_t *Kc, uint16_t *Vc, const int *lens,
                      const int *ars, int n_agents, int kv_cap, int n_qh, int n_kvh, float scale, float *part,
                      cudaStream_t s, bool pdl, unsigned long long *trace)
{
    AttnArgs p = attn_args(pl, lens, ars, kv_cap, n_qh, n_kvh, scale, part);
    p.trace = trace;
    p.qkv = qkv;
    p.ldqkv = ldqkv;
    p.Kc = Kc;
    p.Vc = Vc;
    p.Kw = Kc;
    p.Vw = Vc;
    return launch_split_kernel<true>(pl, p, n_agents, s, pdl);
}

AttnPartView attn_part_view(const AttnPlan &pl, const float *part, const int *ars, const int *lens, int kv_cap,
                            int n_qh, int n_kvh)
{
    AttnPartView v;
    v.part = part;
    v.ars = ars;
    v.lens = lens;
    v.n_kvh = n_kvh;
    v.G = pl.G;
    v.n_rg = pl.n_rg;
    v.max_splits = pl.max_splits;
    v.CH = pl.CH;
    v.kv_cap = kv_cap;
    v.n_qh = n_qh;
    return v;
}

int launch_attn(const AttnPlan &pl, const uint16_t *Q, const uint16_t *Kc, const uint16_t *Vc, const int *lens,
                const int *ars, int n_agents, int kv_cap, int n_qh, int n_kvh, float scale, uint16_t *O, float *part,
                cudaStream_t s, bool pdl)
{
    AttnArgs p = attn_args(pl, lens, ars, kv_cap, n_qh, n_kvh, scale, part);
    p.Q = Q;
    p.Kc = Kc;
    p.Vc = Vc;
    int rc = launch_split_kernel<false>(pl, p, n_agents, s, pdl);
    if (rc)
        return rc;
    return launch_attn_combine(pl, part, lens, ars, n_agents, kv_cap, n_qh, n_kvh, O, s, pdl);
}

int launch_attn_combine(const AttnPlan &pl, const float *part, const int *lens, const int *ars, int n_agents,
                        int kv_cap, int n_qh, int n_kvh, uint16_t *O, cudaStream_t s, bool pdl)
{
    AttnArgs p = attn_args(pl, lens, ars, kv_cap, n_qh, n_kvh, 1.f, const_cast<float *>(part));
    dim3 g2(QG, pl.n_rg, n_agents * n_kvh);
    cudaError_t e = pdl ? launch_pdl(k_attn_combine, g2, dim3(128), 0, s, p, O)
                        : (k_attn_combine<<<g2, 128, 0, s>>>(p, O), cudaGetLastError());
    return cuda_check(e, "attn combine launch");
}

}  // namespace qad

extern "C" size_t qad_decode_attn_ws_bytes(int n_agents, int n_qh, int n_kvh, int kv_cap, int max_rows_per_agent)
{
    if (n_agents <= 0 || n_kvh <= 0 || n_qh <= 0 || n_qh % n_kvh || kv_cap <= 0 || max_rows_per_agent <= 0)
        return 0;
    return qad::attn_plan(n_agents, n_qh, n_kvh, kv_cap, max_rows_per_agent).part_bytes;
}

extern "C" int qad_decode_attn(const uint16_t *Q, const uint16_t *Kc, const uint16_t *Vc, const int *lens,
                               const int *agent_row_start, int n_agents, int max_rows_per_agent, int kv_cap, int n_qh,
                               int n_kvh, int hd, float scale, uint16_t *O, void *ws, size_t ws_bytes, void *stream)
{
    if (!Q || !Kc || !Vc || !lens || !agent_row_start || !O || !ws || n_agents <= 0 || kv_cap <= 0 || n_qh <= 0 ||
        n_kvh <= 0 || max_rows_per_agent <= 0)
        return qad::fail(QAD_ERR_INVALID, "qad_decode_attn: null pointer or non-positive size");
    if (hd != 128 || n_qh % n_kvh || max_rows_per_agent * (n_qh / n_kvh) > 96 || max_rows_per_agent > QAD_MAX_ROWS)
        return qad::fail(QAD_ERR_UNSUPPORTED,
                         "qad_decode_attn: need hd == 128, n_qh %% n_kvh == 0, rows*group <= 96 (hd=%d n_qh=%d n_kvh=%d "
                         "rows=%d)",
                         hd, n_qh, n_kvh, max_rows_per_agent);
    if (((uintptr_t)Kc | (uintptr_t)Vc) & 15)
        return qad::fail(QAD_ERR_INVALID, "qad_decode_attn: caches must be 16-byte aligned");
    qad::AttnPlan pl = qad::attn_plan(n_agents, n_qh, n_kvh, kv_cap, max_rows_per_agent);
    if (ws_bytes < pl.part_bytes)
        return qad::fail(QAD_ERR_WORKSPACE, "qad_decode_attn: workspace %zu < %zu bytes", ws_bytes, pl.part_bytes);
    return qad::launch_attn(pl, Q, Kc, Vc, lens, agent_row_start, n_agents, kv_cap, n_qh, n_kvh, scale, O,
                            (float *)ws, (cudaStream_t)stream, false);
}
