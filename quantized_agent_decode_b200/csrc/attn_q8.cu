// attn_q8.cu -- the decode attention of attn.cu over a q8_0 KV cache, and the
// q8_0 quantiser.
//
// [dual-4090 page] = rebasdaily.com 2026-09-10, llama.cpp agent concurrency on
// two RTX 4090s: its tests keep the KV cache in q8_0. q8_0 is read here as the
// llama.cpp block format: 32 values share one fp16 scale d = amax / 127 (fp32
// division, then rounded to fp16) and each value is the int8 round(x * (1/d)),
// ties away from zero. The cache is stored as two planes per tensor: codes
// [agent][kv-head][position][128] int8 and scales [agent][kv-head][position][4]
// fp16, so a key row is 136 bytes instead of 256.
//
// The math is the bf16 kernel's (split-KV, swap-AB tensor-core products, online
// softmax in fp32, partial records merged by the o-projection prep); what
// differs is how the operands reach the MMAs:
//   S: A = the key codes as exact fp16 integers, B = Q rounded to bf16 and then
//      converted to fp16 (exact in fp16's normal range). One MMA pair covers one
//      32-value block, and its fp32 result is multiplied by that key's block
//      scale: S = sum_b d_b * (q_b . Q_b), every product exact.
//   O: A = V^T as fp16 d * q (one rounding, relative error <= 2^-11), B = P as
//      fp16 scaled by 2^15 (relative error <= 2^-11 for P >= 2^-29, absolute
//      <= 2^-40 below), so probabilities far below the maximum still count.
// The key index inside a block and the order of the output dimensions are
// permuted so that each lane reads its codes with 8- and 16-byte shared-memory
// loads (the sum over k and the choice of MMA rows are order-free); the
// partial records use the natural order.
// The cross-lane reduction of a tile's maximum and the rescale of the running
// output run only when some score passes the running maximum, and the
// causal/tail masks only on tiles that reach past the cached length.
#include "attn.cuh"

namespace qad {

namespace {

constexpr int QG = ATT_QG;
constexpr int KT = 16;                       // keys per tile
constexpr int NW = 4;                        // warps per CTA
constexpr int TILE = KT * 128;               // int8 codes of one tile (2 KB)
constexpr int SCB = KT * 8;                  // fp16 scales of one tile (128 B)
constexpr int STAGE = 2 * TILE + 2 * SCB;    // K codes | V codes | K scales | V scales
constexpr int STAGES_SHORT = 6;
constexpr int STAGES_LONG = 5;
constexpr float P_LOG2_SCALE = 15.f;         // P enters the PV product as fp16 2^(v - m + 15) <= 2^15

struct Q8Args {
    const uint16_t *Q;          // standalone: bf16 Q [M][n_qh][128]
    const float *qkv;           // fused: fp32 q | k | v rows [M][ldqkv]
    int ldqkv;
    const int8_t *Kq, *Vq;
    const uint16_t *Kd, *Vd;
    int8_t *Kqw, *Vqw;          // fused: cache planes written at the new positions
    uint16_t *Kdw, *Vdw;
    const int *lens, *ars;
    int n_kvh, kv_cap, n_qh, G, CH, n_rg, max_splits;
    float scale_log2;
    float *part;
    unsigned long long *trace;
};

// 16-byte chunk j (0..7) of key row kk (0..15) of a code tile. The XOR pattern
// keeps three access patterns free of bank conflicts: cp.async writing a row's
// 8 chunks, 8-byte reads of chunk pairs {2b, 2b+1} by keys 0..3 (or 4..7), and
// 16-byte reads of one chunk by keys {0,2,4,6} (or the odd ones).
__device__ __forceinline__ int q8f(int k) { return ((((k ^ (k >> 2)) & 1) | (k & 2)) << 1); }
__device__ __forceinline__ int q8sw(int kk, int j) { return kk * 128 + ((j ^ q8f(kk & 7)) << 4); }

// Bytes 0 and 2 of v (signed) -> fp16x2 of their values: 0x64 above (byte ^ 0x80)
// is 1024 + (q + 128); subtracting 1152 leaves q exactly.
__device__ __forceinline__ uint32_t s8x2_to_h2(uint32_t v) { return hsub2((v & 0x00FF00FFu) ^ 0x64806480u, H2_1152); }

// q8_0 of 8 values whose 32-value block spans 4 consecutive lanes: returns the
// 8 codes packed little-endian and the block's fp16 scale bits. All lanes of the
// warp must call it (the block maximum is a 4-lane shuffle reduction).
__device__ __forceinline__ uint2 q8_quant8(const float (&x)[8], uint16_t &dbits)
{
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        amax = fmaxf(amax, fabsf(x[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const float d = __fdiv_rn(amax, 127.f);
    const float id = d != 0.f ? __fdiv_rn(1.f, d) : 0.f;
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int q = (int)roundf(__fmul_rn(x[i], id));
        w[i >> 2] |= (uint32_t)(q & 0xFF) << (8 * (i & 3));
    }
    dbits = __half_as_ushort(__float2half_rn(d));
    return make_uint2(w[0], w[1]);
}

template <bool FUSED, int STAGES>
__global__ void __launch_bounds__(128, 2) k_decode_attn_q8(Q8Args p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int sp = blockIdx.x, rg = blockIdx.y, ag = blockIdx.z;
    const int a = ag / p.n_kvh, g = ag - a * p.n_kvh;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, gq = lane >> 2, c = lane & 3;
    trace_start(p.trace);
    pdl_trigger();
    // agent offsets, lengths and cached tiles are step constants: read before the wait
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
    const size_t head = ((size_t)a * p.n_kvh + g) * (size_t)p.kv_cap;  // first key row of (agent, kv-head)
    const int8_t *Kh = p.Kq + head * 128, *Vh = p.Vq + head * 128;
    const uint16_t *Kdh = p.Kd + head * 4, *Vdh = p.Vd + head * 4;

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
    const int my = ntiles > w ? (ntiles - w + NW - 1) / NW : 0;
    uint8_t *wbuf = smem + (size_t)w * STAGES * STAGE;
    const int nq = p.n_qh * 128, nkv = p.n_kvh * 128;

    // per-lane constants of the copies: chunk (lane & 7) of keys lane/8 + 4i (i = 0..3)
    const int cp_src = (lane >> 3) * 128 + (lane & 7) * 16;
    const int cp_dst0 = q8sw(lane >> 3, lane & 7), cp_dst1 = q8sw((lane >> 3) + 4, lane & 7);
    const int sc_dst = 2 * TILE + (lane >> 4) * SCB + (lane & 15) * 8;
    const uint16_t *sc_src = (lane < 16 ? Kdh : Vdh) + (lane & 15) * 4;
    auto issue = [&](int it, uint8_t *st) {
        const int kb = kbeg + KT * (w + NW * it);
        const bool mixed = FUSED && kb + KT > len;  // the tile holds new positions (taken from the projection)
        if (!mixed && kb + KT <= kend) {            // a full tile of cached keys
            const int8_t *ks = Kh + (size_t)kb * 128 + cp_src, *vs = Vh + (size_t)kb * 128 + cp_src;
            cp_async16(st + cp_dst0, ks);
            cp_async16(st + cp_dst1, ks + 512);
            cp_async16(st + cp_dst0 + 1024, ks + 1024);
            cp_async16(st + cp_dst1 + 1024, ks + 1536);
            cp_async16(st + TILE + cp_dst0, vs);
            cp_async16(st + TILE + cp_dst1, vs + 512);
            cp_async16(st + TILE + cp_dst0 + 1024, vs + 1024);
            cp_async16(st + TILE + cp_dst1 + 1024, vs + 1536);
            cp_async8_zfill(st + sc_dst, sc_src + (size_t)kb * 4, true);
            return;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int idx = lane + 32 * i, kk = idx >> 3, j = idx & 7, kp = kb + kk;
            if (!mixed || kp < len || kp >= kend) {
                const bool ok = kp < kend;
                const size_t src = (size_t)(ok ? kp : 0) * 128 + j * 16;
                cp_async16_zfill(st + q8sw(kk, j), Kh + src, ok);
                cp_async16_zfill(st + TILE + q8sw(kk, j), Vh + src, ok);
            }
        }
        {
            const int kk = lane & 15, kp = kb + kk;
            if (!mixed || kp < len || kp >= kend) {
                const bool ok = kp < kend;
                const size_t src = (size_t)(ok ? kp : 0) * 4;
                if (lane < 16)
                    cp_async8_zfill(st + 2 * TILE + kk * 8, Kdh + src, ok);
                else
                    cp_async8_zfill(st + 2 * TILE + SCB + kk * 8, Vdh + src, ok);
            }
        }
        if constexpr (FUSED) {
        if (!mixed)
            return;
        // new positions: quantise the fp32 k, v rows; the row-group-0 CTA also
        // writes them to the cache. Two keys per pass, 8 values per lane.
#pragma unroll 1
        for (int i = 0; i < KT / 2; ++i) {
            const int kk = 2 * i + (lane >> 4), ch = lane & 15, kp = kb + kk;
            const bool isnew = kp >= len && kp < kend;
            if (!__any_sync(0xffffffffu, isnew))
                continue;
            float kx[8], vx[8];
            if (isnew) {
                const float *row = p.qkv + (size_t)(r0 + kp - len) * p.ldqkv + nq + g * 128 + ch * 8;
                const float4 k0 = *reinterpret_cast<const float4 *>(row);
                const float4 k1 = *reinterpret_cast<const float4 *>(row + 4);
                const float4 v0 = *reinterpret_cast<const float4 *>(row + nkv);
                const float4 v1 = *reinterpret_cast<const float4 *>(row + nkv + 4);
                kx[0] = k0.x, kx[1] = k0.y, kx[2] = k0.z, kx[3] = k0.w;
                kx[4] = k1.x, kx[5] = k1.y, kx[6] = k1.z, kx[7] = k1.w;
                vx[0] = v0.x, vx[1] = v0.y, vx[2] = v0.z, vx[3] = v0.w;
                vx[4] = v1.x, vx[5] = v1.y, vx[6] = v1.z, vx[7] = v1.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    kx[e] = vx[e] = 0.f;
            }
            uint16_t kdb, vdb;
            const uint2 kc = q8_quant8(kx, kdb);
            const uint2 vc = q8_quant8(vx, vdb);
            if (isnew) {
                const int off = q8sw(kk, ch >> 1) + (ch & 1) * 8;
                *reinterpret_cast<uint2 *>(st + off) = kc;
                *reinterpret_cast<uint2 *>(st + TILE + off) = vc;
                if ((ch & 3) == 0) {
                    *reinterpret_cast<uint16_t *>(st + 2 * TILE + kk * 8 + (ch >> 2) * 2) = kdb;
                    *reinterpret_cast<uint16_t *>(st + 2 * TILE + SCB + kk * 8 + (ch >> 2) * 2) = vdb;
                }
                if (rg == 0) {
                    *reinterpret_cast<uint2 *>(p.Kqw + (head + kp) * 128 + ch * 8) = kc;
                    *reinterpret_cast<uint2 *>(p.Vqw + (head + kp) * 128 + ch * 8) = vc;
                    if ((ch & 3) == 0) {
                        p.Kdw[(head + kp) * 4 + (ch >> 2)] = kdb;
                        p.Vdw[(head + kp) * 4 + (ch >> 2)] = vdb;
                    }
                }
            }
        }
        }
    };
    auto cached_tile = [&](int it) { return !FUSED || kbeg + KT * (w + NW * it) + KT <= len; };
    auto stage = [&](int i) { return wbuf + (size_t)i * STAGE; };
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

    // Q^T fragments, k permuted: for block b and half h the lane holds
    // Q[q][32b + 8c + 4h + 0..3] (b0 = first two, b1 = last two) for q = q0 + 8nt + gq.
    uint32_t qf[3][4][2][2];
    int qpos[3][2];
#pragma unroll
    for (int nt = 0; nt < 3; ++nt) {
        const int qi = q0 + 8 * nt + gq;
        const bool ok = qi < R;
        const int j = ok ? qi / p.G : 0, hl = ok ? qi - j * p.G : 0;
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float f[4] = {0.f, 0.f, 0.f, 0.f};
                const int k = 32 * b + 8 * c + 4 * h;
                if (ok) {
                    if (FUSED) {
                        const float4 v = *reinterpret_cast<const float4 *>(
                            p.qkv + (size_t)(r0 + j) * p.ldqkv + (g * p.G + hl) * 128 + k);
                        // Q is rounded to bf16 as in every other path
                        f[0] = bf16_to_f(f_to_bf16(v.x));
                        f[1] = bf16_to_f(f_to_bf16(v.y));
                        f[2] = bf16_to_f(f_to_bf16(v.z));
                        f[3] = bf16_to_f(f_to_bf16(v.w));
                    } else {
                        const uint2 v = *reinterpret_cast<const uint2 *>(
                            p.Q + ((size_t)(r0 + j) * p.n_qh + g * p.G + hl) * 128 + k);
                        f[0] = bf16_to_f((uint16_t)(v.x & 0xFFFF));
                        f[1] = bf16_to_f((uint16_t)(v.x >> 16));
                        f[2] = bf16_to_f((uint16_t)(v.y & 0xFFFF));
                        f[3] = bf16_to_f((uint16_t)(v.y >> 16));
                    }
                }
                qf[nt][b][h][0] = pack_half2(f[0], f[1]);
                qf[nt][b][h][1] = pack_half2(f[2], f[3]);
            }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int qc = q0 + 8 * nt + 2 * c + e;
            qpos[nt][e] = qc < R ? len + qc / p.G : -1;
        }
    }

    // per-lane shared-memory offsets of the fragment loads (see q8sw)
    int offK[4];
#pragma unroll
    for (int b = 0; b < 4; ++b)
        offK[b] = q8sw(gq, 2 * b + (c >> 1)) + (c & 1) * 8;
    const int offV0 = TILE + q8sw(2 * c, gq), offV1 = TILE + q8sw(2 * c + 1, gq);
    const int offVd = 2 * TILE + SCB + 2 * c * 8 + (gq >> 1) * 2;
    int cur = 0, nxt = STAGES - 1;  // ring slots of tile it and of tile it + STAGES - 1
    for (int it = 0; it < my; ++it) {
        if (it + STAGES - 1 < my)
            issue(it + STAGES - 1, stage(nxt));
        nxt = nxt + 1 == STAGES ? 0 : nxt + 1;
        cp_async_commit();
        cp_async_wait<STAGES - 1>();
        __syncwarp();
        const uint8_t *st = stage(cur);
        cur = cur + 1 == STAGES ? 0 : cur + 1;
        const int kb = kbeg + KT * (w + NW * it);

        // S^T = K Q^T, one MMA pair per 32-value block, scaled per key and block
        const uint2 dks0 = lds_v2(st + 2 * TILE + gq * 8), dks1 = lds_v2(st + 2 * TILE + (gq + 8) * 8);
        const float kd0[4] = {half_lo(dks0.x), half_hi(dks0.x), half_lo(dks0.y), half_hi(dks0.y)};
        const float kd1[4] = {half_lo(dks1.x), half_hi(dks1.x), half_lo(dks1.y), half_hi(dks1.y)};
        float s[3][4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const uint2 x0 = lds_v2(st + offK[b]), x1 = lds_v2(st + offK[b] + 8 * 128);
            const uint32_t u00 = x0.x ^ 0x80808080u, u01 = x0.y ^ 0x80808080u;
            const uint32_t u10 = x1.x ^ 0x80808080u, u11 = x1.y ^ 0x80808080u;
            const uint32_t A0[4] = {hsub2(prmt(u00, 0x64646464u, 0x4140u), H2_1152), hsub2(prmt(u10, 0x64646464u, 0x4140u), H2_1152),
                                    hsub2(prmt(u00, 0x64646464u, 0x4342u), H2_1152), hsub2(prmt(u10, 0x64646464u, 0x4342u), H2_1152)};
            const uint32_t A1[4] = {hsub2(prmt(u01, 0x64646464u, 0x4140u), H2_1152), hsub2(prmt(u11, 0x64646464u, 0x4140u), H2_1152),
                                    hsub2(prmt(u01, 0x64646464u, 0x4342u), H2_1152), hsub2(prmt(u11, 0x64646464u, 0x4342u), H2_1152)};
#pragma unroll
            for (int nt = 0; nt < 3; ++nt) {
                float t[4];
                mma_f16_zero(t, A0[0], A0[1], A0[2], A0[3], qf[nt][b][0][0], qf[nt][b][0][1]);
                mma_f16(t, A1[0], A1[1], A1[2], A1[3], qf[nt][b][1][0], qf[nt][b][1][1]);
                if (b == 0) {
                    s[nt][0] = kd0[0] * t[0];
                    s[nt][1] = kd0[0] * t[1];
                    s[nt][2] = kd1[0] * t[2];
                    s[nt][3] = kd1[0] * t[3];
                } else {
                    s[nt][0] = fmaf(kd0[b], t[0], s[nt][0]);
                    s[nt][1] = fmaf(kd0[b], t[1], s[nt][1]);
                    s[nt][2] = fmaf(kd1[b], t[2], s[nt][2]);
                    s[nt][3] = fmaf(kd1[b], t[3], s[nt][3]);
                }
            }
        }

        // Online softmax: the cross-lane reduction of the tile maximum and the rescale
        // run only when some score passes the running maximum m (once m is established,
        // most tiles skip both). P enters the MMA as fp16 2^(v - m + 15) <= 2^15; fp16
        // keeps 11 bits down to 2^-29 of the maximum, and the common factor cancels in
        // every merge. Masks run only on tiles that reach past the cached keys.
        const bool interior = kb + KT <= kend && kb + KT <= len;
        float v[3][4];
        bool over = false;
#pragma unroll
        for (int nt = 0; nt < 3; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float v0 = s[nt][e] * p.scale_log2, v1 = s[nt][e + 2] * p.scale_log2;
                if (!interior) {
                    const int k0 = kb + gq, k1 = k0 + 8;
                    v0 = (k0 < kend && k0 <= qpos[nt][e]) ? v0 : -INFINITY;
                    v1 = (k1 < kend && k1 <= qpos[nt][e]) ? v1 : -INFINITY;
                }
                over |= fmaxf(v0, v1) > m[nt][e];
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
        uint32_t ph[3][2];
#pragma unroll
        for (int nt = 0; nt < 3; ++nt) {
            float pv[4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const bool none = m[nt][e] == -INFINITY;
                const float mb = m[nt][e] - P_LOG2_SCALE;
                pv[e] = none ? 0.f : ex2_approx(v[nt][e] - mb);
                pv[e + 2] = none ? 0.f : ex2_approx(v[nt][e + 2] - mb);
                l[nt][e] += pv[e] + pv[e + 2];
            }
            // P^T fragment (keys x queries) via an in-register transpose, fp16
            ph[nt][0] = movmatrix_t(pack_half2(pv[0], pv[1]));
            ph[nt][1] = movmatrix_t(pack_half2(pv[2], pv[3]));
        }

        // O^T += V^T P^T. M-tile dt, row gq is output dimension 16 gq + 2 dt,
        // row gq + 8 is 16 gq + 2 dt + 1; K = keys 2c, 2c+1, 2c+8, 2c+9 (natural).
        // keys 2c+8, 2c+9 sit 1024 bytes after keys 2c, 2c+1 (same swizzle); this lane's 16
        // dimensions lie in block gq / 2, whose scales are 2 bytes at offVd in each key's 8
        const uint4 R0 = lds_v4(st + offV0), R1 = lds_v4(st + offV1);
        const uint4 R2 = lds_v4(st + offV0 + 1024), R3 = lds_v4(st + offV1 + 1024);
        const uint32_t d01 = (uint32_t)*reinterpret_cast<const uint16_t *>(st + offVd) |
                             (uint32_t)*reinterpret_cast<const uint16_t *>(st + offVd + 8) << 16;
        const uint32_t d89 = (uint32_t)*reinterpret_cast<const uint16_t *>(st + offVd + 64) |
                             (uint32_t)*reinterpret_cast<const uint16_t *>(st + offVd + 72) << 16;
        const uint32_t W0[4] = {R0.x, R0.y, R0.z, R0.w}, W1[4] = {R1.x, R1.y, R1.z, R1.w};
        const uint32_t W2[4] = {R2.x, R2.y, R2.z, R2.w}, W3[4] = {R3.x, R3.y, R3.z, R3.w};
#pragma unroll
        for (int dt = 0; dt < 8; ++dt) {
            const int wi = dt >> 1;
            const uint32_t sa = (dt & 1) ? 0x0602u : 0x0400u, sbb = (dt & 1) ? 0x0703u : 0x0501u;
            const uint32_t a0 = hmul2(s8x2_to_h2(prmt(W0[wi], W1[wi], sa)), d01);
            const uint32_t a1 = hmul2(s8x2_to_h2(prmt(W0[wi], W1[wi], sbb)), d01);
            const uint32_t a2 = hmul2(s8x2_to_h2(prmt(W2[wi], W3[wi], sa)), d89);
            const uint32_t a3 = hmul2(s8x2_to_h2(prmt(W2[wi], W3[wi], sbb)), d89);
#pragma unroll
            for (int nt = 0; nt < 3; ++nt)
                mma_f16(o[dt][nt], a0, a1, a2, a3, ph[nt][0], ph[nt][1]);
        }
        __syncwarp();
    }
    cp_async_wait<0>();

#pragma unroll
    for (int nt = 0; nt < 3; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float t = l[nt][e];
            t += __shfl_xor_sync(0xffffffffu, t, 4);
            t += __shfl_xor_sync(0xffffffffu, t, 8);
            t += __shfl_xor_sync(0xffffffffu, t, 16);
            l[nt][e] = t;
        }
    __syncthreads();  // every warp is done with its stages: reuse shared memory
    float *sO = reinterpret_cast<float *>(smem);  // [4][QG][128]
    float *sM = sO + NW * QG * 128;               // [4][QG]
    float *sL = sM + NW * QG;                     // [4][QG]
#pragma unroll
    for (int dt = 0; dt < 8; ++dt)
#pragma unroll
        for (int nt = 0; nt < 3; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int d = 16 * gq + 2 * dt + (e >> 1), q = 8 * nt + 2 * c + (e & 1);
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
    float *out = p.part + pidx * ATT_PART_FLOATS;
    const int nqv = min(QG, R - q0);
    for (int idx = tid; idx < nqv * 128; idx += blockDim.x) {
        const int q = idx >> 7;
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww)
            M = fmaxf(M, sM[ww * QG + q]);
        float acc = 0.f;
        if (M != -INFINITY)
#pragma unroll
            for (int ww = 0; ww < NW; ++ww)
                acc += exp2f(sM[ww * QG + q] - M) * sO[((size_t)ww * QG + q) * 128 + (idx & 127)];
        out[idx] = acc;
    }
    if (tid < nqv) {
        float M = -INFINITY, Lsum = 0.f;
        for (int ww = 0; ww < NW; ++ww)
            M = fmaxf(M, sM[ww * QG + tid]);
        if (M != -INFINITY)
            for (int ww = 0; ww < NW; ++ww)
                Lsum += exp2f(sM[ww * QG + tid] - M) * sL[ww * QG + tid];
        out[QG * 128 + tid] = M;
        out[QG * 128 + QG + tid] = Lsum;
    }
    trace_end(p.trace);
}

// q8_0 of n values (n % 32 == 0): 8 values per lane, 4 lanes per block.
template <bool BF16_IN>
__global__ void __launch_bounds__(256) k_q8_0_quantize(const void *__restrict__ x, long long n,
                                                       int8_t *__restrict__ q, uint16_t *__restrict__ d)
{
    const long long groups = n / 8;
    const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    const int lane = threadIdx.x & 31;
    for (long long base = warp * 32; base < groups; base += nwarps * 32) {
        const long long gi = base + lane;
        const bool ok = gi < groups;
        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (ok) {
            if (BF16_IN) {
                const uint4 r = *reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(x) + gi * 8);
                const uint32_t wv[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    v[2 * i] = bf16_to_f((uint16_t)(wv[i] & 0xFFFF));
                    v[2 * i + 1] = bf16_to_f((uint16_t)(wv[i] >> 16));
                }
            } else {
                const float4 a = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(x) + gi * 8);
                const float4 b = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(x) + gi * 8 + 4);
                v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
            }
        }
        uint16_t db;
        const uint2 codes = q8_quant8(v, db);
        if (ok) {
            *reinterpret_cast<uint2 *>(q + gi * 8) = codes;
            if ((gi & 3) == 0)
                d[gi >> 2] = db;
        }
    }
}

size_t q8_smem_bytes(int stages)
{
    const size_t st = (size_t)NW * stages * STAGE;
    const size_t merge = ((size_t)NW * QG * 128 + 2 * NW * QG) * sizeof(float);
    return st > merge ? st : merge;
}

template <bool FUSED, int STAGES>
int launch_q8_t(const AttnPlan &pl, const Q8Args &p, int n_agents, cudaStream_t s, bool pdl)
{
    const size_t smem = q8_smem_bytes(STAGES);
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        int rc = cuda_check(cudaFuncSetAttribute(k_decode_attn_q8<FUSED, STAGES>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                            "cudaFuncSetAttribute(attn q8)");
        if (rc)
            return rc;
        if (dev >= 0 && dev < 64)
            attr_set[dev] = true;
    }
    dim3 grid(pl.max_splits, pl.n_rg, n_agents * p.n_kvh);
    cudaError_t e = pdl ? launch_pdl(k_decode_attn_q8<FUSED, STAGES>, grid, dim3(128), smem, s, p)
                        : (k_decode_attn_q8<FUSED, STAGES><<<grid, 128, smem, s>>>(p), cudaGetLastError());
    return cuda_check(e, "attn q8 launch");
}

template <bool FUSED>
int launch_q8(const AttnPlan &pl, const Q8Args &p, int n_agents, cudaStream_t s, bool pdl)
{
    // the plan's short form sizes splits for a 6-deep ring
    return pl.stages == STAGES_SHORT ? launch_q8_t<FUSED, STAGES_SHORT>(pl, p, n_agents, s, pdl)
                          : launch_q8_t<FUSED, STAGES_LONG>(pl, p, n_agents, s, pdl);
}

Q8Args q8_args(const AttnPlan &pl, const int *lens, const int *ars, int kv_cap, int n_qh, int n_kvh, float scale,
               float *part)
{
    Q8Args p = {};
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

}  // namespace

size_t kv_q8_scale_offset(int n_agents, int n_kvh, int kv_cap)
{
    const size_t codes = (size_t)n_agents * n_kvh * kv_cap * 128;
    return (codes + 255) & ~(size_t)255;
}

int launch_attn_q8_fused(const AttnPlan &pl, const float *qkv, int ldqkv, int8_t *Kq, uint16_t *Kd, int8_t *Vq,
                         uint16_t *Vd, const int *lens, const int *ars, int n_agents, int kv_cap, int n_qh, int n_kvh,
                         float scale, float *part, cudaStream_t s, bool pdl, unsigned long long *trace)
{
    Q8Args p = q8_args(pl, lens, ars, kv_cap, n_qh, n_kvh, scale, part);
    p.trace = trace;
    p.qkv = qkv;
    p.ldqkv = ldqkv;
    p.Kq = p.Kqw = Kq;
    p.Vq = p.Vqw = Vq;
    p.Kd = p.Kdw = Kd;
    p.Vd = p.Vdw = Vd;
    return launch_q8<true>(pl, p, n_agents, s, pdl);
}

int launch_attn_q8(const AttnPlan &pl, const uint16_t *Q, const int8_t *Kq, const uint16_t *Kd, const int8_t *Vq,
                   const uint16_t *Vd, const int *lens, const int *ars, int n_agents, int kv_cap, int n_qh, int n_kvh,
                   float scale, uint16_t *O, float *part, cudaStream_t s, bool pdl)
{
    Q8Args p = q8_args(pl, lens, ars, kv_cap, n_qh, n_kvh, scale, part);
    p.Q = Q;
    p.Kq = Kq;
    p.Vq = Vq;
    p.Kd = Kd;
    p.Vd = Vd;
    int rc = launch_q8<false>(pl, p, n_agents, s, pdl);
    if (rc)
        return rc;
    return launch_attn_combine(pl, part, lens, ars, n_agents, kv_cap, n_qh, n_kvh, O, s, pdl);
}

}  // namespace qad

extern "C" size_t qad_kv_cache_bytes(int kv_format, int n_agents, int n_kvh, int kv_cap, int hd)
{
    if (n_agents <= 0 || n_kvh <= 0 || kv_cap <= 0 || hd != 128)
        return 0;
    if (kv_format == QAD_KV_BF16)
        return (size_t)n_agents * n_kvh * kv_cap * hd * 2;
    if (kv_format == QAD_KV_Q8_0)
        return qad::kv_q8_scale_offset(n_agents, n_kvh, kv_cap) + (size_t)n_agents * n_kvh * kv_cap * (hd / 32) * 2;
    return 0;
}

extern "C" int qad_q8_0_quantize(const void *x, int x_is_bf16, long long n, int8_t *q, uint16_t *d, void *stream)
{
    if (!x || !q || !d || n < 0)
        return qad::fail(QAD_ERR_INVALID, "qad_q8_0_quantize: null pointer or negative size");
    if (n % 32)
        return qad::fail(QAD_ERR_UNSUPPORTED, "qad_q8_0_quantize: n (%lld) must be a multiple of 32", n);
    if (((uintptr_t)x | (uintptr_t)q) & 15 || (uintptr_t)d & 1)
        return qad::fail(QAD_ERR_INVALID, "qad_q8_0_quantize: x and q must be 16-byte aligned, d 2-byte");
    if (n == 0)
        return 0;
    const long long warps = (n / 8 + 31) / 32;
    const int grid = (int)(warps < 4L * 148 * 8 ? (warps + 7) / 8 : 4L * 148);
    cudaStream_t s = (cudaStream_t)stream;
    if (x_is_bf16)
        qad::k_q8_0_quantize<true><<<grid, 256, 0, s>>>(x, n, q, d);
    else
        qad::k_q8_0_quantize<false><<<grid, 256, 0, s>>>(x, n, q, d);
    return qad::cuda_check(cudaGetLastError(), "q8_0 quantize launch");
}

extern "C" int qad_decode_attn_q8(const uint16_t *Q, const int8_t *Kq, const uint16_t *Kd, const int8_t *Vq,
                                  const uint16_t *Vd, const int *lens, const int *agent_row_start, int n_agents,
                                  int max_rows_per_agent, int kv_cap, int n_qh, int n_kvh, int hd, float scale,
                                  uint16_t *O, void *ws, size_t ws_bytes, void *stream)
{
    if (!Q || !Kq || !Kd || !Vq || !Vd || !lens || !agent_row_start || !O || !ws || n_agents <= 0 || kv_cap <= 0 ||
        n_qh <= 0 || n_kvh <= 0 || max_rows_per_agent <= 0)
        return qad::fail(QAD_ERR_INVALID, "qad_decode_attn_q8: null pointer or non-positive size");
    if (hd != 128 || n_qh % n_kvh || max_rows_per_agent * (n_qh / n_kvh) > 96 || max_rows_per_agent > QAD_MAX_ROWS)
        return qad::fail(QAD_ERR_UNSUPPORTED,
                         "qad_decode_attn_q8: need hd == 128, n_qh %% n_kvh == 0, rows*group <= 96 (hd=%d n_qh=%d "
                         "n_kvh=%d rows=%d)",
                         hd, n_qh, n_kvh, max_rows_per_agent);
    if (((uintptr_t)Kq | (uintptr_t)Vq) & 15 || ((uintptr_t)Kd | (uintptr_t)Vd) & 7 || (uintptr_t)Q & 7)
        return qad::fail(QAD_ERR_INVALID,
                         "qad_decode_attn_q8: codes must be 16-byte aligned, scales and Q 8-byte aligned");
    qad::AttnPlan pl = qad::attn_plan(n_agents, n_qh, n_kvh, kv_cap, max_rows_per_agent);
    if (ws_bytes < pl.part_bytes)
        return qad::fail(QAD_ERR_WORKSPACE, "qad_decode_attn_q8: workspace %zu < %zu bytes", ws_bytes, pl.part_bytes);
    return qad::launch_attn_q8(pl, Q, Kq, Kd, Vq, Vd, lens, agent_row_start, n_agents, kv_cap, n_qh, n_kvh, scale, O,
                               (float *)ws, (cudaStream_t)stream, false);
}
