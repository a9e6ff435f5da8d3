// prefill_attn.cu -- causal attention of one agent's prompt chunk (C rows at
// positions len .. len+C-1) over that agent's cache (keys 0 .. len+C-1, the
// chunk's own k, v already appended): row j sees keys 0 .. len+j.
//
// [OpenJet page] = rebasdaily.com 2026-10-29, "OpenJet ... multi-agent
// serving", section 真正重要的是少互相堵车: a 20K-token prompt is processed
// while the other agents keep decoding; each chunk of it attends causally over
// the agent's own KV cache. It is the decode attention's definition with
// C ~ 2048 rows instead of 3.
//
// Design (sm_100a warp MMAs, flash-attention style):
//  * CTA = 64 query vectors of one kv-head (vector v = row j * G + local head,
//    so the G heads sharing a kv-head are adjacent and one causal limit covers
//    whole rows), 4 warps of 16 vectors. Q stays in registers as the A
//    operand of S = Q K^T (m16n8k16 bf16, fp32 accumulate).
//  * K and V stream through a double-buffered shared-memory ring in 64-key
//    tiles (cp.async, 16-byte chunks XOR-swizzled so ldmatrix is conflict
//    free); K feeds S via ldmatrix, V feeds O += P V via ldmatrix.trans.
//  * Online softmax in fp32 (exp2 with the scale folded in); P is rounded to
//    bf16 once and used straight from the S accumulator registers as the A
//    operand of the PV product.
#include "attn.cuh"

namespace qad {

namespace pf {
constexpr int QV = 64;      // query vectors per CTA
constexpr int KT = 64;      // keys per tile
constexpr int STAGES = 2;
constexpr int TILE = KT * 128 * 2;  // 16 KB per K (or V) tile
constexpr float M_SLACK = 8.f;      // scores may pass the reference maximum by 2^8
}  // namespace pf

struct PrefillArgs {
    const uint16_t *Q, *Kc, *Vc;
    uint16_t *O;
    int len, C, kv_cap, n_qh, n_kvh, G;
    float scale_log2;
};

__device__ __forceinline__ int pswz(int key, int chunk) { return key * 256 + ((chunk ^ (key & 7)) << 4); }

__global__ void __launch_bounds__(128) k_prefill_attn(PrefillArgs p)
{
    using namespace pf;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
    const int kvh = blockIdx.y;
    const int R = p.C * p.G;            // query vectors of this kv-head
    const int v0 = blockIdx.x * QV;     // first vector of the CTA
    const int wv = v0 + 16 * w;         // first vector of this warp
    const int j_last = min(p.C - 1, (v0 + QV - 1) / p.G);
    const int kend = p.len + j_last + 1;  // keys any vector of the CTA can see
    const int ntiles = (kend + KT - 1) / KT;
    const size_t head_off = (size_t)kvh * p.kv_cap * 128;
    const uint16_t *Kh = p.Kc + head_off, *Vh = p.Vc + head_off;

    // Q fragments (A operand) of this warp's 16 vectors: rows g and g + 8
    uint32_t qf[8][4];
    int lim[2];  // last visible key of each of the two vectors this lane holds
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int v = wv + g + 8 * r;
        const bool ok = v < R;
        const int j = ok ? v / p.G : 0, hl = ok ? v - j * p.G : 0;
        lim[r] = ok ? p.len + j : -1;
        const uint16_t *qrow = p.Q + ((size_t)j * p.n_qh + kvh * p.G + hl) * 128;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qf[ks][r] = ok ? *reinterpret_cast<const uint32_t *>(qrow + 16 * ks + 2 * c) : 0u;
            qf[ks][2 + r] = ok ? *reinterpret_cast<const uint32_t *>(qrow + 16 * ks + 8 + 2 * c) : 0u;
        }
    }
    float o[16][4];
#pragma unroll
    for (int nd = 0; nd < 16; ++nd)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            o[nd][e] = 0.f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};

    auto issue = [&](int t) {
        uint8_t *st = smem + (size_t)(t % STAGES) * 2 * TILE;
        const int kb = t * KT;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int idx = tid + 128 * i, key = idx >> 4, ch = idx & 15;
            const bool ok = kb + key < kend;
            const size_t src = (size_t)(ok ? kb + key : 0) * 128 + ch * 8;
            cp_async16_zfill(st + pswz(key, ch), Kh + src, ok);
            cp_async16_zfill(st + TILE + pswz(key, ch), Vh + src, ok);
        }
    };
    issue(0);
    cp_async_commit();
    for (int t = 0; t < ntiles; ++t) {
        if (t + 1 < ntiles)
            issue(t + 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const uint8_t *Ks = smem + (size_t)(t % STAGES) * 2 * TILE;
        const uint8_t *Vs = Ks + TILE;
        const int kb = t * KT;

        // S = Q K^T for 64 keys (8 n-tiles)
        float s[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                s[nt][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 8; ks += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(b0, b1, b2, b3, Ks + pswz(8 * nt + (lane & 7), 2 * ks + (lane >> 3)));
                mma_bf16(s[nt], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b0, b1);
                mma_bf16(s[nt], qf[ks + 1][0], qf[ks + 1][1], qf[ks + 1][2], qf[ks + 1][3], b2, b3);
            }
        }
        // Online softmax; rows r = 0 (vector g) and 1 (vector g + 8). The reference
        // maximum m moves (cross-lane reduction, rescale of o and l) only when a score
        // passes it by more than M_SLACK log2 units, so P <= 2^8 (well inside bf16's
        // range) and most tiles skip the reduction and the rescale.
        const bool need_mask = kb + KT - 1 > p.len + (wv / p.G) || kb + KT > kend;
        bool over = false;
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float x = s[nt][2 * r + e] * p.scale_log2;
                    if (need_mask && kb + 8 * nt + 2 * c + e > lim[r])
                        x = -INFINITY;
                    s[nt][2 * r + e] = x;
                    over |= x > m[r] + M_SLACK;
                }
        if (__any_sync(0xffffffffu, over)) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                float mx = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
                    mx = fmaxf(mx, fmaxf(s[nt][2 * r], s[nt][2 * r + 1]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float mn = fmaxf(m[r], mx);
                const float corr = mn == -INFINITY ? 1.f : ex2_approx(m[r] - mn);
                m[r] = mn;
                l[r] *= corr;
#pragma unroll
                for (int nd = 0; nd < 16; ++nd) {
                    o[nd][2 * r] *= corr;
                    o[nd][2 * r + 1] *= corr;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const bool none = m[r] == -INFINITY;
            float sum = 0.f;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float pv = none ? 0.f : ex2_approx(s[nt][2 * r + e] - m[r]);
                    s[nt][2 * r + e] = pv;
                    sum += pv;
                }
            l[r] += sum;
        }
        // O += P V: P (bf16) straight from the S registers, V^T via ldmatrix.trans
#pragma unroll
        for (int kt = 0; kt < 4; ++kt) {
            const uint32_t a0 = pack_bf162(s[2 * kt][0], s[2 * kt][1]);
            const uint32_t a1 = pack_bf162(s[2 * kt][2], s[2 * kt][3]);
            const uint32_t a2 = pack_bf162(s[2 * kt + 1][0], s[2 * kt + 1][1]);
            const uint32_t a3 = pack_bf162(s[2 * kt + 1][2], s[2 * kt + 1][3]);
#pragma unroll
            for (int nd = 0; nd < 16; nd += 2) {
                uint32_t b0, b1, b2, b3;
                const int i = lane >> 3;
                ldsm_x4_t(b0, b1, b2, b3, Vs + pswz(16 * kt + 8 * (i & 1) + (lane & 7), nd + (i >> 1)));
                mma_bf16(o[nd], a0, a1, a2, a3, b0, b1);
                mma_bf16(o[nd + 1], a0, a1, a2, a3, b2, b3);
            }
        }
        __syncthreads();  // the next issue() overwrites this stage
    }
    cp_async_wait<0>();

    // normalise and store (bf16): lane holds dims 8 nd + 2c, +1 of vectors g, g + 8
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        float tot = l[r];
        tot += __shfl_xor_sync(0xffffffffu, tot, 1);
        tot += __shfl_xor_sync(0xffffffffu, tot, 2);
        const int v = wv + g + 8 * r;
        if (v >= R)
            continue;
        const int j = v / p.G, hl = v - j * p.G;
        const float inv = tot > 0.f ? 1.f / tot : 0.f;
        uint16_t *orow = p.O + ((size_t)j * p.n_qh + kvh * p.G + hl) * 128;
#pragma unroll
        for (int nd = 0; nd < 16; ++nd)
            *reinterpret_cast<uint32_t *>(orow + 8 * nd + 2 * c) = pack_bf162(o[nd][2 * r] * inv, o[nd][2 * r + 1] * inv);
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
    const size_t smem = (size_t)pf::STAGES * 2 * pf::TILE;
    static bool done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !done[dev]) {
        int rc = cuda_check(cudaFuncSetAttribute(k_prefill_attn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                            "cudaFuncSetAttribute(prefill attn)");
        if (rc)
            return rc;
        if (dev >= 0 && dev < 64)
            done[dev] = true;
    }
    dim3 grid((C * a.G + pf::QV - 1) / pf::QV, n_kvh);
    k_prefill_attn<<<grid, 128, smem, s>>>(a);
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
