// dense.cu -- the prefill-chunk GEMM: Y[m][n] = sum_k w[n][k] x[m][k] for a
// chunk of M ~ 2060 activation rows (2048 prompt tokens of one agent plus the
// 12 decode rows) against the same Q4_K / Q6_K-like weights as the decode step.
//
// [OpenJet page] = rebasdaily.com 2026-10-29, "OpenJet ... multi-agent
// serving", section 真正重要的是少互相堵车: a 20K-token prompt arrives while
// other agents decode; its chunks run through the same weights. At M = 2060
// the product is compute-bound (~2 FLOP per weight per row), so it belongs
// on the 5th-generation tensor cores.
//
// Design (sm_100a, one CTA per SM, persistent): rounds of output tiles go one
// tile per CTA (tile c + r * grid: the CTAs of a round work on neighbouring
// tiles and share their weights and activations in L2). When the last round
// is partial and would leave many CTAs idle for many blocks, its tiles are cut
// into (tile, 256-k block) units and split evenly over all CTAs instead
// (stream-K); see dense_schedule:
//  * Output tile = 128 weight rows x 256 activation rows. The accumulator
//    D[128][256] fp32 lives in TMEM (256 columns); one elected thread issues
//    tcgen05.mma kind::f16 (M=128, N=256, K=16) with both operands in shared
//    memory (K-major, no swizzle: 8-row x 16-byte core matrices).
//  * A producer warp streams the raw quantized blocks of the tile's 128 rows
//    by TMA (one block of 256 k per stage) and the activation tiles (256 rows
//    x 64 k fp16, already in core-matrix order) by one bulk copy per k-step.
//  * Eight dequant warps turn each 64-wide k-step of the raw blocks into fp16
//    weights in core-matrix order (one weight row per thread, one 32-wide half
//    of the k-step per warp). Each weight (d*sc*q - dmin*m for Q4_K,
//    d*sc*(q-32) for Q6_K) is formed in fp32 with packed f32x2 operations and
//    rounded to fp16 once, so an operand is within 2^-11 of its weight.
//  * Two accumulators (512 TMEM columns): four epilogue warps read one tile
//    segment (the run's part of a tile) out of TMEM, apply the activation row
//    scales and store Y while the MMAs of the next segment run. A tile whose
//    blocks are split between CTAs was zeroed by the prep kernel and each of
//    its segments is added into Y (fp32 atomics); a whole tile is stored.
//  * Activations enter as fp16 of x * 2^e_m (per-row power of two putting the
//    row's max |x| in [2^14, 2^15)); a prep kernel writes them straight into
//    the tile order the bulk copies want, zero-padding M to whole tiles.
//  * Every mbarrier wait is bounded; on a timeout the CTA records a status,
//    skips the rest of its work, waits for its own copies and MMAs, frees its
//    TMEM and exits.
#include <cuda.h>

#include "dense.cuh"
#include "gemm.cuh"

namespace qad {

__device__ int g_dense_status;
// Test hook (qad_debug_stall): v > 0 makes the producer of CTA 0 issue no copy
// from its activation step v - 1 on, so that CTA's pipeline waits run out.
__device__ int g_dense_stall;

namespace dn {
constexpr int TN = 128;            // weight rows per tile (MMA M)
constexpr int TM = 256;            // activation rows per tile (MMA N)
constexpr int KS = 64;             // k per pipeline step
constexpr int SR = 2;              // raw-block stages
constexpr int SB = 3;              // activation-tile stages
constexpr int SA = 3;              // dequantized-weight stages
constexpr int B_BYTES = TM * KS * 2;   // 32 KB
constexpr int A_BYTES = TN * KS * 2;   // 16 KB
constexpr int DQW = 8;             // dequant warps: two per weight-row quarter (k halves)
constexpr int EPW = 4;             // epilogue warps (one per TMEM lane quarter)
constexpr int THREADS = 32 * (2 + DQW + EPW);  // + producer, MMA issuer
constexpr int Q6A = 208;
template <int FMT>
struct Raw {
    static constexpr int W = TN * (FMT == 4 ? 144 : Q6A);
    static constexpr int D = FMT == 4 ? 0 : TN * 16;
    static constexpr int COPY = W + D;
    static constexpr int BYTES = (COPY + 1023) / 1024 * 1024;
};
template <int FMT>
constexpr size_t smem_bytes()
{
    return 1024 /* alignment slack */ + (size_t)SR * Raw<FMT>::BYTES + (size_t)SB * B_BYTES + (size_t)SA * A_BYTES +
           256 /* barriers + tmem slot */;
}
enum { ST_RAW = 1, ST_B = 2, ST_A = 3, ST_ACC = 4, ST_DONE = 5 };
}  // namespace dn

struct DenseArgs {
    int N, K, M, mt, nt, nblk;
    int tiles;            // mt * nt
    int rounds;           // rounds of tiles (tile c + r * grid < tiles, r < rounds)
    int sk_units;         // units of the last round split over all CTAs (0: none)
    const uint16_t *x16;  // activation tiles (dense_x16 layout)
    const float *rs;      // per activation row 2^-e (0 past M)
    float *Y;
    int ldy;
};

// Segment i of this CTA's work: blocks b0 .. b1-1 of tile t. Rounds first (whole
// tiles), then (SK) the CTA's share [u0, u1) of the last round's units, cut at
// tile boundaries. False when there is no segment i. The kernel is compiled
// twice: without SK it holds none of the split-tile code.
template <bool SK>
__device__ __forceinline__ bool dense_segment(const DenseArgs &a, int i, int &t, int &b0, int &b1)
{
    if (!SK || i < a.rounds) {
        t = (int)blockIdx.x + i * (int)gridDim.x;
        b0 = 0;
        b1 = a.nblk;
        return t < a.tiles && (SK || i < a.rounds);
    }
    const int j = i - a.rounds;
    const int u0 = (int)((long long)blockIdx.x * a.sk_units / gridDim.x);
    const int u1 = (int)((long long)(blockIdx.x + 1) * a.sk_units / gridDim.x);
    const int u = j == 0 ? u0 : (u0 / a.nblk + j) * a.nblk;
    if (u >= u1)
        return false;
    t = a.rounds * (int)gridDim.x + u / a.nblk;
    b0 = u % a.nblk;
    b1 = min(a.nblk, b0 + (u1 - u));
    return true;
}

// Epilogue of one tile segment for this thread's weight column ng: the 256
// accumulator columns (activation rows) times their row scales, stored into Y
// (a whole tile) or added into it (ADD: a segment of a zeroed, split tile).
template <bool ADD>
__device__ __forceinline__ void dense_store_tile(const DenseArgs &a, uint32_t tacc, const float (&rsv)[dn::TM / 32],
                                                 int mt, int ng, int lane)
{
    const bool col_ok = ng < a.N;
#pragma unroll
    for (int j = 0; j < dn::TM / 16; ++j) {
        uint32_t v[16];
        tmem_ld_x16(tacc + 16 * j, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int mm = 16 * j + i, m = mt * dn::TM + mm;
            const float r = __shfl_sync(0xffffffffu, rsv[mm / 32], mm % 32);
            if (m < a.M && col_ok) {
                if (ADD)
                    atomicAdd(a.Y + (size_t)m * a.ldy + ng, __uint_as_float(v[i]) * r);
                else
                    a.Y[(size_t)m * a.ldy + ng] = __uint_as_float(v[i]) * r;
            }
        }
    }
}

// Activation tile layout: [m_tile][k-step][k-chunk 8][256 rows][8 fp16]; one
// (m_tile, k-step) is 32 KB contiguous, i.e. exactly the B operand of one
// k-step in core-matrix order (chunk stride 4096 B, 8-row stride 128 B).
// The prep kernel (one CTA per activation row r) writes row r into those tiles
// and zeroes, in row r of Y, the last-round tiles whose units the GEMM's CTAs
// split (a CTA boundary c * sk_units / grid inside the tile): their segments
// are added into Y. Tile t = (n-tile t / n_mt, m-tile t % n_mt).
__global__ void __launch_bounds__(256) k_prep_dense(const uint16_t *__restrict__ X, int ldx, int M, int K,
                                                    uint16_t *__restrict__ x16, float *__restrict__ rs,
                                                    float *__restrict__ Y, int N, int n_mt, int t_sk, int sk_units,
                                                    int grid)
{
    __shared__ float red[8];
    const int r = blockIdx.x, tid = threadIdx.x;
    const int mt = r / dn::TM, rr = r % dn::TM, ksteps = K / dn::KS;
    const bool live = r < M;
    const int nblk = K / 256;
    if (live && sk_units > 0)
        for (int c = 1 + tid; c < grid; c += 256) {
            const int u = (int)((long long)c * sk_units / grid), t = t_sk + u / nblk;
            if (u % nblk == 0 || t % n_mt != mt)
                continue;
            const int n0 = (t / n_mt) * dn::TN, n1 = min(N, n0 + dn::TN);
            for (int n = n0; n < n1; ++n)
                Y[(size_t)r * N + n] = 0.f;
        }
    float mx = 0.f;
    if (live)
        for (int q = tid; q < K / 8; q += 256) {
            const uint4 v = *reinterpret_cast<const uint4 *>(X + (size_t)r * ldx + 8 * q);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                mx = fmaxf(mx, fabsf(bf16_to_f((uint16_t)(w[i] & 0xFFFF))));
                mx = fmaxf(mx, fabsf(bf16_to_f((uint16_t)(w[i] >> 16))));
            }
        }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((tid & 31) == 0)
        red[tid >> 5] = mx;
    __syncthreads();
    mx = 0.f;
    for (int i = 0; i < 8; ++i)
        mx = fmaxf(mx, red[i]);
    int e = 0;
    if (mx > 0.f) {
        int E;
        frexpf(mx, &E);  // mx in [2^(E-1), 2^E)
        e = min(126, max(-126, 15 - E));
    }
    const float sc = ldexpf(1.f, e);
    if (tid == 0)
        rs[r] = live ? ldexpf(1.f, -e) : 0.f;
    for (int q = tid; q < K / 8; q += 256) {
        uint4 o = make_uint4(0u, 0u, 0u, 0u);
        if (live) {
            const uint4 v = *reinterpret_cast<const uint4 *>(X + (size_t)r * ldx + 8 * q);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t h[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                h[i] = pack_half2(bf16_to_f((uint16_t)(w[i] & 0xFFFF)) * sc, bf16_to_f((uint16_t)(w[i] >> 16)) * sc);
            o = make_uint4(h[0], h[1], h[2], h[3]);
        }
        const int ks = q / 8, ch = q % 8;
        const size_t off = ((((size_t)mt * ksteps + ks) * 8 + ch) * dn::TM + rr) * 8;
        *reinterpret_cast<uint4 *>(x16 + off) = o;
    }
}

// 32 fp16 weights of row n for k-step kk (0..3) of a Q4_K block: half 0 = the
// low nibbles (k 0..31 of the step, chunks 0..3), half 1 = the high nibbles
// (k 32..63, chunks 4..7); chunk c of the A stage sits at c * 2048 + n * 16.
// Each weight w = d*sc*q - dmin*m is formed in fp32 by one fused multiply-add
// (q, d*sc and dmin*m are exact there, so it rounds once, by at most 2^-24 |w|)
// and rounded to fp16 once: the operand differs from w by at most
// (2^-11 + 2^-24) |w|, or 2^-25 in fp16's subnormal range.
__device__ __forceinline__ void dequant_q4(const uint8_t *blk, int kk, int half, uint8_t *A, int n)
{
    const uint4 h = lds_v4(blk);
    const float d = half_lo(h.x), dmin = half_hi(h.x);
    // byte i of the 12 packed scale/min bytes (h.y, h.z, h.w)
    auto byte = [&](int i) { return ((i < 4 ? h.y : i < 8 ? h.z : h.w) >> (8 * (i & 3))) & 0xFFu; };
    const int j = 2 * kk + half;  // sub-block
    float sc, mn;
    if (j < 4) {
        sc = (float)(byte(j) & 63);
        mn = (float)(byte(j + 4) & 63);
    } else {
        sc = (float)((byte(j + 4) & 0xF) | ((byte(j - 4) >> 6) << 4));
        mn = (float)((byte(j + 4) >> 4) | ((byte(j) >> 6) << 4));
    }
    const float ds = d * sc, dm = -dmin * mn;  // exact in fp32 (at most 17 significant bits)
    const float2 DS = make_float2(ds, ds), DM = make_float2(dm, dm);
    const float2 OFF = make_float2(-8388608.f, -8388608.f);  // -2^23
    const uint4 q0 = lds_v4(blk + 16 + 32 * kk), q1 = lds_v4(blk + 32 + 32 * kk);
    const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t o[4];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const uint32_t w = qw[2 * c + u];
            const uint32_t v = (half ? (w >> 4) : w) & 0x0F0F0F0Fu;  // four 4-bit quants as bytes
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {
                const float2 q = fadd2(make_float2(byte_f23(v, 2 * pr), byte_f23(v, 2 * pr + 1)), OFF);
                const float2 wv = ffma2(q, DS, DM);
                o[2 * u + pr] = pack_half2(wv.x, wv.y);
            }
        }
        *reinterpret_cast<uint4 *>(A + (4 * half + c) * 2048 + n * 16) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Q6_K-like (packed plane A, d from the D tile): k-step kk = half h, group sel;
// `part` 0 writes k 0..31 of the step (chunks 0..3), part 1 k 32..63.
// w = d*sc*(q-32) is exact in fp32 (at most 18 + 5 significant bits) and is
// rounded to fp16 once (at most 2^-11 |w|, or 2^-25 in the subnormal range).
__device__ __forceinline__ void dequant_q6(const uint8_t *blk, float d, int kk, int part, uint8_t *A, int n)
{
    const int h = kk >> 1, sel = kk & 1;
    const uint2 sw = lds_v2(blk + 192 + 8 * h);
    float2 DS[2];
#pragma unroll
    for (int g = 0; g < 2; ++g) {  // 16-weight groups of the part: scales 4 sel + 2 part + g
        const int i = 2 * part + g;  // byte i of word sel (int8)
        const int scv = (int)(int8_t)(uint8_t)((sel ? sw.y : sw.x) >> (8 * i));
        const float ds = d * (float)scv;  // exact (at most 18 significant bits)
        DS[g] = make_float2(ds, ds);
    }
    const float2 OFF = make_float2(-8388640.f, -8388640.f);  // -(2^23 + 32): byte_f23(q) + OFF = q - 32
    {  // part 0: k 0..31 (ql[l], qh bits 4sel); part 1: k 32..63 (ql[l+32], qh bits 4sel+2)
        const uint8_t *ql = blk + 64 * h + 32 * part;
        const uint8_t *qh = blk + 128 + 32 * h;
        const int sh = 4 * sel + 2 * part;
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) {  // chunk = 4 part + c2: k 8 c2 .. 8 c2 + 7 of the part
            const uint2 L = lds_v2(ql + 8 * c2), Hh = lds_v2(qh + 8 * c2);
            const uint32_t lw[2] = {L.x, L.y}, hw[2] = {Hh.x, Hh.y};
            uint32_t o[4];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint32_t q = ((lw[u] >> (4 * sel)) & 0x0F0F0F0Fu) | (((hw[u] >> sh) & 0x03030303u) << 4);
#pragma unroll
                for (int pr = 0; pr < 2; ++pr) {
                    const float2 qm = fadd2(make_float2(byte_f23(q, 2 * pr), byte_f23(q, 2 * pr + 1)), OFF);
                    const float2 wv = fmul2(qm, DS[c2 >> 1]);
                    o[2 * u + pr] = pack_half2(wv.x, wv.y);
                }
            }
            *reinterpret_cast<uint4 *>(A + (4 * part + c2) * 2048 + n * 16) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}


template <int FMT, bool SK>
__global__ void __launch_bounds__(dn::THREADS, 1) k_dense_gemm(const __grid_constant__ WeightMapsBlob mapsb, DenseArgs a)
{
    using namespace dn;
    using R = Raw<FMT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *RAW = smem;
    uint8_t *BS = RAW + SR * R::BYTES;
    uint8_t *AS = BS + SB * B_BYTES;
    uint64_t *bar = reinterpret_cast<uint64_t *>(AS + SA * A_BYTES);
    uint64_t *raw_full = bar, *raw_empty = bar + SR, *b_full = bar + 2 * SR, *b_empty = b_full + SB;
    uint64_t *a_full = b_empty + SB, *a_empty = a_full + SA, *acc_full = a_empty + SA, *acc_empty = acc_full + 2;
    uint64_t *done = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
    __shared__ int s_bad;
    const CUtensorMap *mw = reinterpret_cast<const CUtensorMap *>(mapsb.bytes);
    const CUtensorMap *md = mw + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        s_bad = 0;
        for (int i = 0; i < SR; ++i) {
            mbar_init(&raw_full[i], 1);
            mbar_init(&raw_empty[i], DQW);
        }
        for (int i = 0; i < SB; ++i) {
            mbar_init(&b_full[i], 1);
            mbar_init(&b_empty[i], 1);
        }
        for (int i = 0; i < SA; ++i) {
            mbar_init(&a_full[i], DQW);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], EPW);
        }
        mbar_init(done, 1);
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);  // two 256-column accumulators
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&](int code) {
        atomicExch(&g_dense_status, code);
        atomicExch(&s_bad, 1);
    };
    auto bad = [&]() { return *(volatile int *)&s_bad != 0; };

    if (warp == 0) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            const int stall = blockIdx.x == 0 ? *(volatile int *)&g_dense_stall - 1 : -1;
            int bk = 0, ks = 0, t, b0, b1;
            for (int sg = 0; !bad() && ks != stall && dense_segment<SK>(a, sg, t, b0, b1); ++sg) {
                const int nt = t / a.mt, mt = t % a.mt;
                for (int blk = b0; blk < b1 && !bad() && ks != stall; ++blk) {
                    const int s = bk % SR;
                    if (bk >= SR && !mbar_wait(&raw_empty[s], ((bk / SR) - 1) & 1)) {
                        fail(ST_RAW);
                        break;
                    }
                    uint8_t *st = RAW + s * R::BYTES;
                    mbar_arrive_expect_tx(&raw_full[s], (uint32_t)R::COPY);
                    tma_load_2d(st, mw, blk * (FMT == 4 ? 144 : Q6A), nt * TN, &raw_full[s]);
                    if (FMT == 6)
                        tma_load_2d(st + R::W, md, blk & ~7, nt * TN, &raw_full[s]);
                    ++bk;
                    for (int kk = 0; kk < 4 && ks != stall; ++kk) {
                        const int sb = ks % SB;
                        if (ks >= SB && !mbar_wait(&b_empty[sb], ((ks / SB) - 1) & 1)) {
                            fail(ST_B);
                            break;
                        }
                        mbar_arrive_expect_tx(&b_full[sb], (uint32_t)B_BYTES);
                        bulk_g2s(BS + sb * B_BYTES, a.x16 + ((size_t)mt * (4 * a.nblk) + 4 * blk + kk) * (B_BYTES / 2),
                                 B_BYTES, &b_full[sb]);
                        ++ks;
                    }
                }
            }
            // every issued copy lands before teardown
            for (int k = max(0, bk - SR); k < bk; ++k)
                if (!mbar_wait(&raw_full[k % SR], (k / SR) & 1, 20000))
                    fail(ST_RAW);
            for (int k = max(0, ks - SB); k < ks; ++k)
                if (!mbar_wait(&b_full[k % SB], (k / SB) & 1, 20000))
                    fail(ST_B);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_f16(TN, TM);
            int ks = 0, tc = 0, t, b0, b1;
            bool issued = false;
            for (; !bad() && dense_segment<SK>(a, tc, t, b0, b1); ++tc) {
                const int acc = tc & 1;
                if (tc >= 2) {  // the epilogue has drained this accumulator's previous segment
                    if (!mbar_wait(&acc_empty[acc], ((tc >> 1) - 1) & 1)) {
                        fail(ST_ACC);
                        break;
                    }
                    tc_fence_after();
                }
                for (int k = 4 * b0; k < 4 * b1; ++k, ++ks) {
                    const int sa = ks % SA, sb = ks % SB;
                    if (!mbar_wait(&a_full[sa], (ks / SA) & 1) || !mbar_wait(&b_full[sb], (ks / SB) & 1)) {
                        fail(ST_A);
                        break;
                    }
                    tc_fence_after();
                    const uint32_t abase = smem_u32(AS + sa * A_BYTES), bbase = smem_u32(BS + sb * B_BYTES);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint64_t ad = umma_desc_k_noswz(abase + j * 2 * (TN * 16), TN * 16, 128);
                        const uint64_t bd = umma_desc_k_noswz(bbase + j * 2 * (TM * 16), TM * 16, 128);
                        umma_f16_ss(tmem + 256 * acc, ad, bd, idesc, k != 4 * b0 || j != 0);
                    }
                    issued = true;
                    umma_commit(&a_empty[sa]);
                    umma_commit(&b_empty[sb]);
                }
                if (bad())
                    break;
                umma_commit(&acc_full[acc]);
            }
            // every MMA this thread issued has completed before TMEM is freed
            if (issued) {
                umma_commit(done);
                if (!mbar_wait(done, 0, 20000))
                    fail(ST_DONE);
            }
        }
    } else if (warp < 2 + DQW) {
        // ------------------------------------------------ dequant (weight row n, one k half)
        const int dw = warp - 2, quarter = dw & 3, half = dw >> 2;
        const int n = 32 * quarter + lane;
        int bk = 0, ks = 0, t, b0, b1;
        for (int sg = 0; !bad() && dense_segment<SK>(a, sg, t, b0, b1); ++sg) {
            for (int blk = b0; blk < b1 && !bad(); ++blk, ++bk) {
                const int s = bk % SR;
                if (!__all_sync(0xffffffffu, mbar_wait(&raw_full[s], (bk / SR) & 1))) {
                    fail(ST_RAW);
                    break;
                }
                const uint8_t *st = RAW + s * R::BYTES;
                float d6 = 0.f;
                if (FMT == 6) {
                    const uint32_t dwd = lds_u32(st + R::W + n * 16 + (blk & 6) * 2);
                    d6 = __half2float(__ushort_as_half((unsigned short)(dwd >> ((blk & 1) * 16))));
                }
                for (int kk = 0; kk < 4; ++kk, ++ks) {
                    const int sa = ks % SA;
                    if (ks >= SA && !__all_sync(0xffffffffu, mbar_wait(&a_empty[sa], ((ks / SA) - 1) & 1))) {
                        fail(ST_A);
                        break;
                    }
                    uint8_t *A = AS + sa * A_BYTES;
                    if (FMT == 4)
                        dequant_q4(st + n * 144, kk, half, A, n);
                    else
                        dequant_q6(st + n * Q6A, d6, kk, half, A, n);
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&a_full[sa]);
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&raw_empty[s]);
            }
        }
    } else {
        // ------------------------------------------------ epilogue: D[n][m] * 2^-e_m -> Y[m][n]
        const int quarter = warp & 3;  // TMEM lanes 32 quarter .. + 31 (this warp's access window)
        const int n = 32 * quarter + lane;
        int tc = 0, t, b0, b1;
        for (; !bad() && dense_segment<SK>(a, tc, t, b0, b1); ++tc) {
            const bool whole = !SK || (b0 == 0 && b1 == a.nblk);  // else the tile was zeroed: add the segment
            const int nt = t / a.mt, mt = t % a.mt, acc = tc & 1;
            float rsv[TM / 32];  // row scales of this tile's 256 activation rows, 8 per lane
#pragma unroll
            for (int i = 0; i < TM / 32; ++i)
                rsv[i] = a.rs[mt * TM + 32 * i + lane];
            if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[acc], (tc >> 1) & 1))) {
                fail(ST_ACC);
                break;
            }
            tc_fence_after();
            const uint32_t tacc = tmem + 256 * acc + ((uint32_t)(32 * quarter) << 16);
            if (whole)
                dense_store_tile<false>(a, tacc, rsv, mt, nt * TN + n, lane);
            else if (SK)
                dense_store_tile<true>(a, tacc, rsv, mt, nt * TN + n, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&acc_empty[acc]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------- host side

// Tensor maps of the weights with 128-row boxes: [0] the Q4_K matrix or the
// Q6_K plane A, [1] the Q6_K plane D.
int make_dense_maps(int fmt, const void *W, int N, int K, WeightMapsBlob *out)
{
    static_assert(sizeof(WeightMapsBlob) >= 2 * sizeof(CUtensorMap), "blob too small");
    CUtensorMap *m = reinterpret_cast<CUtensorMap *>(out->bytes);
    const int nblk = K / 256;
    if (fmt == 4)
        return encode_tmap_2d(&m[0], W, 1, (uint64_t)nblk * 144, (uint64_t)N, (uint64_t)nblk * 144, 144, dn::TN);
    int rc = encode_tmap_2d(&m[0], W, 1, (uint64_t)nblk * dn::Q6A, (uint64_t)N, (uint64_t)nblk * dn::Q6A, dn::Q6A,
                            dn::TN);
    if (rc)
        return rc;
    const int nblk8 = (nblk + 7) & ~7;
    const uint8_t *D = (const uint8_t *)W + (size_t)N * nblk * dn::Q6A;
    return encode_tmap_2d(&m[1], D, 2, (uint64_t)nblk8, (uint64_t)N, (uint64_t)nblk8 * 2, 8, dn::TN);
}

size_t dense_ws_bytes(int K, int M)
{
    const size_t mpad = (size_t)(M + dn::TM - 1) / dn::TM * dn::TM;
    return mpad * (size_t)K * 2 + ((mpad * 4 + 255) & ~(size_t)255);
}

// The schedule. Rounds of one tile per CTA; if the last round is partial, its
// tiles are split over all CTAs (stream-K) only when the CTAs it would leave
// idle, times its blocks, come to more than DENSE_SK_MIN_IDLE units per CTA:
// the split tiles' fp32 atomic additions cost about that much. Measured at
// M = 2060 (two rounds plus 64 of 148 tiles): the split took the Q6_K down
// projection (68 blocks) from 580 to 508 us, but cost gate|up (20 blocks, 80
// of 148) 783 -> 838 us, q|k|v 206 -> 242 and o (24 blocks) 185 -> 194.
constexpr int DENSE_SK_MIN_IDLE = 20;
struct DenseSchedule {
    int grid, rounds, sk_units;
};
static DenseSchedule dense_schedule(int tiles, int nblk)
{
    const int sms = num_sms();
    const long long units = (long long)tiles * nblk;
    const int g_sk = units < sms ? (int)units : sms;
    const int rem = tiles % g_sk;
    if (rem > 0 && (long long)(g_sk - rem) * nblk > (long long)DENSE_SK_MIN_IDLE * g_sk)
        return {g_sk, tiles / g_sk, rem * nblk};
    const int g = tiles < sms ? tiles : sms;
    return {g, (tiles + g - 1) / g, 0};
}

template <int FMT, bool SK>
static int launch_dense_t(const WeightMapsBlob &maps, const DenseArgs &a, int grid, cudaStream_t s)
{
    const size_t smem = dn::smem_bytes<FMT>();
    static bool done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !done[dev]) {
        int rc = cuda_check(
            cudaFuncSetAttribute(k_dense_gemm<FMT, SK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
            "cudaFuncSetAttribute(dense)");
        if (rc)
            return rc;
        if (dev >= 0 && dev < 64)
            done[dev] = true;
    }
    k_dense_gemm<FMT, SK><<<grid, dn::THREADS, smem, s>>>(maps, a);
    return cuda_check(cudaGetLastError(), "dense gemm launch");
}

int launch_dense(int fmt, const void *W, int N, int K, const uint16_t *X, int M, float *Y, void *ws,
                 cudaStream_t s)
{
    WeightMapsBlob maps;
    int rc = make_dense_maps(fmt, W, N, K, &maps);
    if (rc)
        return rc;
    const int mt = (M + dn::TM - 1) / dn::TM, ntl = (N + dn::TN - 1) / dn::TN, tiles = mt * ntl;
    const DenseSchedule sch = dense_schedule(tiles, K / 256);
    uint16_t *x16 = (uint16_t *)ws;
    float *rs = (float *)((char *)ws + (size_t)mt * dn::TM * K * 2);
    k_prep_dense<<<mt * dn::TM, 256, 0, s>>>(X, K, M, K, x16, rs, Y, N, mt, sch.rounds * sch.grid, sch.sk_units,
                                             sch.grid);
    rc = cuda_check(cudaGetLastError(), "dense prep launch");
    if (rc)
        return rc;
    DenseArgs a;
    a.N = N;
    a.K = K;
    a.M = M;
    a.mt = mt;
    a.nt = ntl;
    a.nblk = K / 256;
    a.tiles = tiles;
    a.rounds = sch.rounds;
    a.sk_units = sch.sk_units;
    a.x16 = x16;
    a.rs = rs;
    a.Y = Y;
    a.ldy = N;
    if (sch.sk_units > 0)
        return fmt == 4 ? launch_dense_t<4, true>(maps, a, sch.grid, s) : launch_dense_t<6, true>(maps, a, sch.grid, s);
    return fmt == 4 ? launch_dense_t<4, false>(maps, a, sch.grid, s) : launch_dense_t<6, false>(maps, a, sch.grid, s);
}

}  // namespace qad

// ------------------------------------------------------------- C ABI

extern "C" size_t qad_dense_gemm_ws_bytes(int K, int M)
{
    if (K <= 0 || K % 256 || M <= 0)
        return 0;
    return qad::dense_ws_bytes(K, M);
}

namespace qad {
int dense_set_stall(int at)
{
    const int v = at < 0 ? 0 : at + 1;
    return cuda_check(cudaMemcpyToSymbol(g_dense_stall, &v, sizeof(int)), "dense stall hook");
}
}  // namespace qad

extern "C" int qad_dense_status(int reset)
{
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, qad::g_dense_status, sizeof(int));
    if (e != cudaSuccess)
        return qad::cuda_check(e, "qad_dense_status");
    if (reset && v) {
        const int z = 0;
        e = cudaMemcpyToSymbol(qad::g_dense_status, &z, sizeof(int));
        if (e != cudaSuccess)
            return qad::cuda_check(e, "qad_dense_status reset");
    }
    return v;
}

static int dense_entry(int fmt, const void *W, int N, int K, const uint16_t *X, int M, float *Y, void *ws,
                       size_t ws_bytes, void *stream)
{
    const char *name = fmt == 4 ? "qad_q4k_gemm_dense" : "qad_q6k_gemm_dense";
    if (!W || !X || !Y || !ws || N <= 0 || K <= 0 || M <= 0)
        return qad::fail(QAD_ERR_INVALID, "%s: null pointer or non-positive size (N=%d K=%d M=%d)", name, N, K, M);
    if (K % 256 || K > 65536 || N > (1 << 24))
        return qad::fail(QAD_ERR_UNSUPPORTED, "%s: need K %% 256 == 0, K <= 65536 (K=%d N=%d)", name, K, N);
    if (((uintptr_t)W | (uintptr_t)X) & 15 || (uintptr_t)ws & 255)
        return qad::fail(QAD_ERR_INVALID, "%s: W and X must be 16-byte aligned, ws 256-byte aligned", name);
    if (ws_bytes < qad::dense_ws_bytes(K, M))
        return qad::fail(QAD_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", name, ws_bytes, qad::dense_ws_bytes(K, M));
    return qad::launch_dense(fmt, W, N, K, X, M, Y, ws, (cudaStream_t)stream);
}

extern "C" int qad_q4k_gemm_dense(const void *W, int N, int K, const uint16_t *X, int M, float *Y, void *ws,
                                  size_t ws_bytes, void *stream)
{
    return dense_entry(4, W, N, K, X, M, Y, ws, ws_bytes, stream);
}

extern "C" int qad_q6k_gemm_dense(const void *W, int N, int K, const uint16_t *X, int M, float *Y, void *ws,
                                  size_t ws_bytes, void *stream)
{
    return dense_entry(6, W, N, K, X, M, Y, ws, ws_bytes, stream);
}
