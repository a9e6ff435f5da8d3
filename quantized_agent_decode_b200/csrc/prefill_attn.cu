// prefill_attn.cu -- causal attention of one agent's prompt chunk (C rows at
// positions len .. len+C-1) over that agent's cache (keys 0 .. len+C-1, the
// chunk's own k, v already appended): row j sees keys 0 .. len+j.
//
// [OpenJet page] = rebasdaily.com 2026-10-29, "OpenJet ... multi-agent
// serving", section 真正重要的是少互相堵车: a 20K-token prompt is processed
// while the other agents keep decoding; each chunk of it attends causally over
// the agent's own KV cache. It is the decode attention's definition with
// C ~ 2048 rows instead of 3.
#include <cuda.h>

#include "attn.cuh"

namespace qad {

struct PrefillArgs {
    const uint16_t *Q, *Kc, *Vc;
    uint16_t *O;
    int len, C, kv_cap, n_qh, n_kvh, G;
    float scale_log2;
};

// ------------------------------------------------------------- tcgen05 form
//
// CTA = two blocks of 128 query vectors (A and B, adjacent rows) of one
// kv-head, so every K/V tile brought into shared memory serves 256 query
// vectors (the kernel is bound by re-reading each kv-head's K/V prefix through
// L2 once per CTA); heavy (late) pairs first. Ten warps: softmax warps 0-3 own
// block A and 4-7 block B (thread = query vector = TMEM lane; warp w reaches
// lanes 32 (w & 3)..), a producer warp (TMA) and an MMA warp (one thread
// issues tcgen05.mma). Keys go in 64-key tiles through a 3-deep ring:
//  * K and V arrive as one TMA box each through a 3-D view of the cache (8
//    dims, key, 16-dim chunk) that lands as [dim chunk][key][8 dims], the
//    K-major no-swizzle operand layout (8-row x 16-byte core matrices) of B in
//    S = Q K^T. Q is loaded once in the same layout.
//  * TMEM: S_A, S_B (64 columns each), O_A, O_B (128 each).
//  * The MMA thread alternates the blocks: S_X(j+1) as soon as block X's
//    softmax has read S_X(j), then PV_X(j) once it has written P_X(j), so the
//    tensor core works on one block while the other block's softmax runs.
//  * A softmax thread keeps a reference maximum that moves (with a rescale of
//    its O row in TMEM) only when a score passes it by more than 2^8, skips the
//    masks on tiles below every row's causal limit, and writes P = 2^(s - m + 7)
//    (at most 2^15) as fp16 in the A-operand layout [key chunk][row][8 keys]:
//    one rounding of at most 2^-11, and no subnormal loss above P = 2^-21. All
//    eight warps transpose each V tile with ldmatrix.trans into the K-major B
//    layout [key chunk][dim][8 keys], converting bf16 to fp16 on the way (exact
//    for finite values inside fp16's range; double-buffered; keys past the
//    causal end are zeroed, so cache slots beyond the chunk never reach a
//    product). S = Q K^T stays bf16 x bf16 (exact products), PV is fp16 x fp16,
//    both accumulate in fp32; the row sum uses the same 2^7 factor.
// Every mbarrier wait is bounded; on a timeout the CTA records a status, stops
// issuing, waits for its own copies and MMAs, frees TMEM and exits.
namespace pt {
constexpr int ROWS = 128, KT = 64, NS = 3;  // rows per block, keys per tile, K/V ring depth
constexpr int QB = ROWS * 128 * 2;          // 32 KB: one block's Q
constexpr int KB = KT * 128 * 2;            // 16 KB: one K or V tile, one Vt, one P
constexpr int THREADS = 32 * 10;
constexpr float M_SLACK = 8.f;
constexpr float P_LOG2_SCALE = 7.f;         // P enters the PV product as 2^(s - m + 7) <= 2^15
constexpr size_t SMEM = 128 + 2 * (size_t)QB + (2 * NS + 4) * (size_t)KB + 256;  // Q[2], K/V[NS], Vt[2], P[2]
enum { ST_KV = 1, ST_S = 2, ST_P = 3, ST_PV = 4, ST_DONE = 5, ST_VT = 6 };
}  // namespace pt

__device__ int g_prefill_status;
// Test hook (qad_debug_stall): v > 0 makes the producer of CTA (0, 0) issue no
// K/V tile from its tile v - 1 on, so that CTA's pipeline waits run out.
__device__ int g_prefill_stall;

struct PfMaps {
    CUtensorMap k, v;  // [n_kvh * kv_cap][128] bf16 as (8 dims, key, dim chunk), boxes of 64 keys
};

__global__ void __launch_bounds__(pt::THREADS, 1) k_prefill_attn_tc(const __grid_constant__ PfMaps maps, PrefillArgs p)
{
    using namespace pt;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~(uintptr_t)127);
    uint8_t *QS = smem, *KS = QS + 2 * QB, *VS = KS + NS * KB, *VT = VS + NS * KB, *PS = VT + 2 * KB;
    uint64_t *bar = reinterpret_cast<uint64_t *>(PS + 2 * KB);
    uint64_t *kv_full = bar, *kv_free = bar + NS, *s_full = bar + 2 * NS, *s_free = s_full + 2, *p_full = s_free + 2,
             *pv_done = p_full + 2, *vt_full = pv_done + 2, *vt_free = vt_full + 2, *done = vt_free + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
    __shared__ int s_bad;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kvh = blockIdx.y;
    const int R = p.C * p.G;
    const int npair = (R + 2 * ROWS - 1) / (2 * ROWS);
    const int v0 = (npair - 1 - (int)blockIdx.x) * 2 * ROWS;  // late pairs (more keys) first
    const int j_last = min(p.C - 1, (v0 + 2 * ROWS - 1) / p.G);
    const int kend = p.len + j_last + 1;
    const int ntiles = (kend + KT - 1) / KT;

    if (threadIdx.x == 0) {
        s_bad = 0;
        for (int i = 0; i < NS; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_free[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], 128);
            mbar_init(&p_full[i], 128);
            mbar_init(&pv_done[i], 1);
            mbar_init(&vt_full[i], 256);
            mbar_init(&vt_free[i], 1);
        }
        mbar_init(done, 1);
        mbar_fence_init();
    }
    // Q of both blocks (zero past the chunk), [block][dim chunk][row][8 dims]
    if (warp < 8) {
        const int r = threadIdx.x, v = v0 + r;
        const bool ok = v < R;
        const int j = ok ? v / p.G : 0, hl = ok ? v - j * p.G : 0;
        const uint16_t *qrow = p.Q + ((size_t)j * p.n_qh + kvh * p.G + hl) * 128;
        uint8_t *qb = QS + (r >> 7) * QB + (r & 127) * 16;
#pragma unroll
        for (int dc = 0; dc < 16; ++dc)
            cp_async16_zfill(qb + dc * 2048, qrow + 8 * dc, ok);
        cp_async_commit();
        cp_async_wait<0>();
        fence_proxy_async();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 512);  // S_A 0..63, S_B 64..127, O_A 128..255, O_B 256..383
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&](int code) {
        atomicExch(&g_prefill_status, code);
        atomicExch(&s_bad, 1);
    };
    auto bad = [&]() { return *(volatile int *)&s_bad != 0; };

    if (warp == 8) {
        // ------------------------------------------------ producer: K and V tiles by TMA
        if (lane == 0) {
            const int stall = blockIdx.x == 0 && blockIdx.y == 0 ? *(volatile int *)&g_prefill_stall - 1 : -1;
            int j = 0;
            for (; j < ntiles && !bad() && j != stall; ++j) {
                const int s = j % NS;
                if (j >= NS && !mbar_wait(&kv_free[s], ((j / NS) - 1) & 1)) {
                    fail(ST_KV);
                    break;
                }
                mbar_arrive_expect_tx(&kv_full[s], 2 * KB);
                const int y = kvh * p.kv_cap + j * KT;
                tma_load_3d(KS + s * KB, &maps.k, 0, y, 0, &kv_full[s]);
                tma_load_3d(VS + s * KB, &maps.v, 0, y, 0, &kv_full[s]);
            }
            for (int k = max(0, j - NS); k < j; ++k)  // every issued copy lands before teardown
                if (!mbar_wait(&kv_full[k % NS], (k / NS) & 1, 20000))
                    fail(ST_KV);
        }
    } else if (warp == 9) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16(ROWS, KT), idesc_o = umma_idesc_f16(ROWS, 128);
            bool issued = false;
            auto issue_s = [&](int X, int j) {
                const uint32_t qb = smem_u32(QS + X * QB), kb = smem_u32(KS + (j % NS) * KB);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_f16_ss(tmem + 64 * X, umma_desc_k_noswz(qb + ks * 4096, 2048, 128),
                                umma_desc_k_noswz(kb + ks * 2048, 1024, 128), idesc_s, ks > 0);
                umma_commit(&s_full[X]);
                issued = true;
            };
            auto issue_pv = [&](int X, int j) {
                const uint32_t pb = smem_u32(PS + X * KB), vb = smem_u32(VT + (j & 1) * KB);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_f16_ss(tmem + 128 + 128 * X, umma_desc_k_noswz(pb + ks * 4096, 2048, 128),
                                umma_desc_k_noswz(vb + ks * 4096, 2048, 128), idesc_o, (j | ks) != 0);
                umma_commit(&pv_done[X]);
            };
            if (mbar_wait(&kv_full[0], 0)) {
                tc_fence_after();
                issue_s(0, 0);
                issue_s(1, 0);
            } else {
                fail(ST_S);
            }
            for (int j = 0; j < ntiles && !bad(); ++j) {
                const bool more = j + 1 < ntiles;
                if (more && !mbar_wait(&kv_full[(j + 1) % NS], ((j + 1) / NS) & 1)) {
                    fail(ST_KV);
                    break;
                }
                bool ok = true;
                for (int X = 0; X < 2 && ok; ++X) {
                    if (more) {  // the next S of this block once its softmax has read the current one
                        if (!mbar_wait(&s_free[X], j & 1)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_s(X, j + 1);
                    }
                    if (!mbar_wait(&p_full[X], j & 1) || (X == 0 && !mbar_wait(&vt_full[j & 1], (j >> 1) & 1))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_pv(X, j);
                }
                if (!ok) {
                    fail(ST_P);
                    break;
                }
                umma_commit(&vt_free[j & 1]);   // both PV products of tile j read Vt[j & 1]
                mbar_arrive(&kv_free[j % NS]);  // S_A(j), S_B(j) were read and V_j transposed
            }
            if (issued) {  // every MMA this thread issued completes before TMEM is freed
                umma_commit(done);
                if (!mbar_wait(done, 0, 20000))
                    fail(ST_DONE);
            }
        }
    } else {
        // ------------------------------------------------ softmax warps
        const int X = warp >> 2, quarter = warp & 3;
        const int r = 32 * quarter + lane, v = v0 + X * ROWS + r;
        const bool live = v < R;
        const int jrow = live ? v / p.G : 0;
        const int lim = live ? p.len + jrow : -1;            // last visible key
        const int lim_blk = min(p.len + (v0 + X * ROWS) / p.G, kend - 1);  // the block's smallest limit
        const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
        const uint32_t tS = tmem + 64 * X + lane_off, tO = tmem + 128 + 128 * X + lane_off;
        uint8_t *PX = PS + X * KB;
        float m = -INFINITY, l = 0.f;
        for (int j = 0; j < ntiles && !bad(); ++j) {
            const int s = j % NS, kb = j * KT;
            // this warp's share of the V transpose: dim chunks 2w, 2w+1, both 32-key groups
            if (!__all_sync(0xffffffffu, mbar_wait(&kv_full[s], (j / NS) & 1)) ||
                (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&vt_free[j & 1], ((j >> 1) - 1) & 1)))) {
                fail(ST_VT);
                break;
            }
            const uint8_t *Vs = VS + s * KB;
            uint8_t *Vt = VT + (j & 1) * KB;
#pragma unroll
            for (int dd = 0; dd < 2; ++dd) {
                const int dc = 2 * warp + dd;
#pragma unroll
                for (int kg = 0; kg < 2; ++kg) {
                    uint32_t t4[4];
                    ldsm_x4_t(t4[0], t4[1], t4[2], t4[3], Vs + dc * 1024 + (32 * kg + lane) * 16);
#pragma unroll
                    for (int mi = 0; mi < 4; ++mi) {
                        const int kc = 4 * kg + mi, key = kb + 8 * kc + 2 * (lane & 3);
                        uint32_t val = t4[mi];
                        if (key >= kend)
                            val = 0u;
                        else if (key + 1 >= kend)
                            val &= 0xFFFFu;
                        *reinterpret_cast<uint32_t *>(Vt + kc * 2048 + (8 * dc + (lane >> 2)) * 16 + (lane & 3) * 4) =
                            bf162_to_h2(val);
                    }
                }
            }
            fence_proxy_async();
            mbar_arrive(&vt_full[j & 1]);
            // the S row of this block
            if (!__all_sync(0xffffffffu, mbar_wait(&s_full[X], j & 1))) {
                fail(ST_S);
                break;
            }
            tc_fence_after();
            float x[KT];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc)
                tmem_ld_x32(tS + 32 * cc, reinterpret_cast<uint32_t *>(x + 32 * cc));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&s_free[X]);
            // scores in the log2 domain, rounded once: the maximum and every exponent below use the same
            // values, so s - m is exact where it matters and P <= 2^15 holds whatever the scores' size
            // (computing the maximum and the exponents with different roundings lets s - m exceed the slack
            // by the scores' rounding error, which is large once |s| is large). Tiles below every row's
            // causal limit skip the mask.
            const bool interior = kb + KT - 1 <= lim_blk;
            float mx = -INFINITY;
            if (interior) {
#pragma unroll
                for (int i = 0; i < KT; ++i) {
                    x[i] *= p.scale_log2;
                    mx = fmaxf(mx, x[i]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < KT; ++i) {
                    const int key = kb + i;
                    x[i] = (key < kend && key <= lim) ? x[i] * p.scale_log2 : -INFINITY;
                    mx = fmaxf(mx, x[i]);
                }
            }
            const bool resc = __any_sync(0xffffffffu, mx > m + M_SLACK);
            float corr = 1.f;
            if (resc) {
                const float mn = fmaxf(m, mx);
                corr = mn == -INFINITY ? 1.f : ex2_approx(m - mn);
                m = mn;
            }
            const bool none = m == -INFINITY;
            uint32_t pw[KT / 2];
            float psum = 0.f;
#pragma unroll
            for (int i = 0; i < KT / 2; ++i) {
                const float p0 = none ? 0.f : ex2_approx((x[2 * i] - m) + P_LOG2_SCALE);
                const float p1 = none ? 0.f : ex2_approx((x[2 * i + 1] - m) + P_LOG2_SCALE);
                psum += p0 + p1;
                pw[i] = pack_half2(p0, p1);
            }
            l = l * corr + psum;
            // this block's previous PV product must be done before O is rescaled or P rewritten
            if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(&pv_done[X], (j - 1) & 1))) {
                fail(ST_PV);
                break;
            }
            tc_fence_after();
            if (resc && j > 0) {
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t ov[32];
                    tmem_ld_x32(tO + 32 * cc, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        ov[i] = __float_as_uint(__uint_as_float(ov[i]) * corr);
                    tmem_st_x32(tO + 32 * cc, ov);
                }
                tmem_wait_st();
            }
#pragma unroll
            for (int kc = 0; kc < 8; ++kc)
                *reinterpret_cast<uint4 *>(PX + kc * 2048 + r * 16) =
                    make_uint4(pw[4 * kc], pw[4 * kc + 1], pw[4 * kc + 2], pw[4 * kc + 3]);
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(&p_full[X]);
        }
        // epilogue: O / l -> bf16
        if (!bad() && __all_sync(0xffffffffu, mbar_wait(&pv_done[X], (ntiles - 1) & 1))) {
            tc_fence_after();
            const int hl = live ? v - jrow * p.G : 0;
            uint16_t *orow = p.O + ((size_t)jrow * p.n_qh + kvh * p.G + hl) * 128;
            const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t ov[32];
                tmem_ld_x32(tO + 32 * cc, ov);
                tmem_wait_ld();
                if (live)
#pragma unroll
                    for (int i = 0; i < 32; i += 8)
                        *reinterpret_cast<uint4 *>(orow + 32 * cc + i) = make_uint4(
                            pack_bf162(__uint_as_float(ov[i]) * inv, __uint_as_float(ov[i + 1]) * inv),
                            pack_bf162(__uint_as_float(ov[i + 2]) * inv, __uint_as_float(ov[i + 3]) * inv),
                            pack_bf162(__uint_as_float(ov[i + 4]) * inv, __uint_as_float(ov[i + 5]) * inv),
                            pack_bf162(__uint_as_float(ov[i + 6]) * inv, __uint_as_float(ov[i + 7]) * inv));
            }
        } else if (!bad()) {
            fail(ST_PV);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

int launch_prefill_attn(const uint16_t *Q, const uint16_t *Kc, const uint16_t *Vc, int len, int C, int kv_cap,
                        int n_qh, int n_kvh, float scale, uint16_t *O, cudaStream_t s)
{
    PrefillArgs a;
    a.Q = Q;
    a.Kc = Kc;
    a.Vc = Vc;
    a.O = O;
    a.len = len;
    a.C = C;
    a.kv_cap = kv_cap;
    a.n_qh = n_qh;
    a.n_kvh = n_kvh;
    a.G = n_qh / n_kvh;
    a.scale_log2 = scale * 1.4426950408889634f;
    PfMaps maps;
    int rc = encode_tmap_kmajor_bf16(&maps.k, Kc, (uint64_t)n_kvh * kv_cap, pt::KT);
    if (!rc)
        rc = encode_tmap_kmajor_bf16(&maps.v, Vc, (uint64_t)n_kvh * kv_cap, pt::KT);
    if (rc)
        return rc;
    static bool done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !done[dev]) {
        rc = cuda_check(cudaFuncSetAttribute(k_prefill_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)pt::SMEM),
                        "cudaFuncSetAttribute(prefill attn tc)");
        if (rc)
            return rc;
        if (dev >= 0 && dev < 64)
            done[dev] = true;
    }
    dim3 grid((C * a.G + 2 * pt::ROWS - 1) / (2 * pt::ROWS), n_kvh);
    k_prefill_attn_tc<<<grid, pt::THREADS, pt::SMEM, s>>>(maps, a);
    return cuda_check(cudaGetLastError(), "prefill attn launch");
}

}  // namespace qad

extern "C" int qad_prefill_attn(const uint16_t *Q, const uint16_t *Kc, const uint16_t *Vc, int len, int C, int kv_cap,
                                int n_qh, int n_kvh, int hd, float scale, uint16_t *O, void *stream)
{
    if (!Q || !Kc || !Vc || !O || C <= 0 || len < 0 || kv_cap <= 0 || n_qh <= 0 || n_kvh <= 0)
        return qad::fail(QAD_ERR_INVALID, "qad_prefill_attn: null pointer or non-positive size");
    if (hd != 128 || n_qh % n_kvh)
        return qad::fail(QAD_ERR_UNSUPPORTED, "qad_prefill_attn: need hd == 128 and n_qh %% n_kvh == 0");
    if ((long long)len + C > kv_cap)
        return qad::fail(QAD_ERR_INVALID, "qad_prefill_attn: len + C = %lld exceeds kv_cap %d", (long long)len + C,
                         kv_cap);
    if ((long long)C * (n_qh / n_kvh) > (1LL << 30))
        return qad::fail(QAD_ERR_UNSUPPORTED, "qad_prefill_attn: chunk too large");
    if (((uintptr_t)Q | (uintptr_t)Kc | (uintptr_t)Vc | (uintptr_t)O) & 15)
        return qad::fail(QAD_ERR_INVALID, "qad_prefill_attn: Q, caches and O must be 16-byte aligned");
    return qad::launch_prefill_attn(Q, Kc, Vc, len, C, kv_cap, n_qh, n_kvh, scale, O, (cudaStream_t)stream);
}

namespace qad {
int prefill_set_stall(int at)
{
    const int v = at < 0 ? 0 : at + 1;
    return cuda_check(cudaMemcpyToSymbol(g_prefill_stall, &v, sizeof(int)), "prefill stall hook");
}
}  // namespace qad

extern "C" int qad_prefill_status(int reset)
{
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, qad::g_prefill_status, sizeof(int));
    if (e != cudaSuccess)
        return qad::cuda_check(e, "qad_prefill_status");
    if (reset && v) {
        const int z = 0;
        e = cudaMemcpyToSymbol(qad::g_prefill_status, &z, sizeof(int));
        if (e != cudaSuccess)
            return qad::cuda_check(e, "qad_prefill_status reset");
    }
    return v;
}
