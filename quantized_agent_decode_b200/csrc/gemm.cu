// gemm.cu -- the shared weight pass: skinny (M <= 16) dequant-GEMM over Q4_K
// and Q6_K-like weights, Y[r][n] = sum_k w[n][k] x[r][k].
//
// [OpenJet page] = rebasdaily.com 2026-10-29, "OpenJet ... multi-agent
// serving", section 只搬一次权重 (move the weights once): the rows of all
// active agents are stacked into one batch, the quantized weights are read
// from memory once per step and every weight just read is used for all rows.
// The page's own cost model is that weight read (16.7 GB / 936 GB/s ~ 18 ms
// on its GPU), so this kernel is an HBM stream with the decode and the
// multiply-accumulate hidden under it.
//
// Design (sm_100a):
//  * A prep kernel forms the activation rows exactly as the step defines them
//    (the bf16 input, RMSNorm of the residual, silu(gate)*up or the merged
//    attention output) and writes, per 256-wide block, a record holding them as
//    fp16 of x * 2^e(r,b) in the tensor core's operand layout, with a power of
//    two per (row, block) so every bf16 value converts exactly.
//  * The GEMM (k_qgemm_tc, below) streams each unit (128 weight rows x one
//    block) by TMA into a ring of shared-memory stages; every quantized byte
//    leaves HBM exactly once. Sixteen decode warps turn a unit into EXACT fp16
//    operands in tensor memory: for Q4_K, A = sc_j * q (<= 945) with the mins
//    entering through one more small product against per-sub-block activation
//    sums; for Q6_K, A = sc * (q - 32). The fp16 values come from the
//    "1024 + q" exponent trick (OR of the nibble into the mantissa of 1024.0)
//    and one fused multiply-add that applies the scale.
//  * One thread issues tcgen05.mma (M = 128 weight rows, N = 16 activation
//    rows, K = 16) with A in tensor memory and the record in shared memory, so
//    the multiply costs the decoding warps no instructions; four epilogue warps
//    apply the block's d, dmin and the row scales.
//  * Work is split stream-K style over a persistent grid (one CTA per SM):
//    each CTA takes a contiguous run of units and adds a tile's partial sums
//    into Y with fp32 atomics when its run leaves the tile.
//  * Programmatic dependent launch: the weights are requested before
//    griddepcontrol.wait, so the weight stream starts while the producer of the
//    activations is still finishing.
#include <cuda.h>

#include <mutex>

#include "dense.cuh"
#include "gemm.cuh"


namespace qad {

// Set by a GEMM whose pipeline wait timed out (1: a consumer, 2: the producer);
// read and cleared by qad_device_status().
__device__ int g_gemm_status;
// Test hook (qad_debug_stall): v > 0 makes the record producer of CTA 0 issue no
// operand copy from its unit v - 1 on, so that CTA's pipeline waits run out.
__device__ int g_gemm_stall;

// ------------------------------------------------------------- operand records
// e(r,b) puts the block's largest |x| in [512, 1024): fp16 holds every bf16
// value of the block exactly unless it is 2^24 times smaller than that max.
static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t frag_bytes(int K, int) { return align256((size_t)(K / 256) * REC_BYTES); }

FragBuf frag_carve(void *ws, int, int)
{
    FragBuf f;
    f.rec = (uint8_t *)ws;
    return f;
}

// ------------------------------------------------------------- prep kernel

struct PrepArgs {
    PrepSrc src;
    int K, M;
    FragBuf fb;
    unsigned long long *trace;
};

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float round_half(float v) { return __half2float(__float2half_rn(v)); }


// Zero the next GEMM's output (its atomics accumulate into it); this CTA's share.
__device__ __forceinline__ void zero_next_output(const PrepSrc &S)
{
    if (S.zero) {
        const long long nct = (long long)gridDim.x * gridDim.y, ct = (long long)blockIdx.y * gridDim.x + blockIdx.x;
        const long long per = ((S.zero_n + nct - 1) / nct + 3) & ~3LL;
        const long long z0 = ct * per, z1 = min(S.zero_n, z0 + per);
        if ((S.zero_n & 3) == 0 && ((uintptr_t)S.zero & 15) == 0) {
            for (long long i = z0 + 4 * (long long)threadIdx.x; i < z1; i += 4 * 256)
                *reinterpret_cast<float4 *>(S.zero + i) = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
            for (long long i = z0 + threadIdx.x; i < z1; i += 256)
                S.zero[i] = 0.f;
        }
    }
}

// Grid (ceil(nblk / 4), 16): CTA (x, r) forms row r's blocks 4x..4x+3, one
// 64-thread quarter per block, thread t of a quarter owning columns 4t..4t+3.
// The values are formed exactly as the GEMM must see them (bf16: the input
// itself, RMSNorm of the fp32 residual, silu(gate)*up, or the merged
// attention output), then scaled per (row, block) into the fp16 record.
template <int FMT>
__global__ void __launch_bounds__(256) k_prep(PrepArgs a)
{
    __shared__ float red[8];
    __shared__ float s_inv;
    const int r = blockIdx.y, tid = threadIdx.x, q = tid >> 6, t = tid & 63;
    const int K = a.K, nblk = K >> 8;
    const int b = 4 * blockIdx.x + q;
    const PrepSrc &S = a.src;
    trace_start(a.trace);
    pdl_trigger();
    const bool live = r < a.M;
    const bool act = live && b < nblk;
    const int k = 256 * b + 4 * t;
    // PREP_ATTN: which agent / query vector / partial records this thread merges.
    // Agent offsets and lengths are constant for the whole step, so they are read
    // before waiting on the previous kernel.
    const float *att_base = nullptr;
    int att_nsp = 0, att_qq = 0, att_d = 0;
    if (S.kind == PREP_ATTN && act) {
        const AttnPartView &P = S.att;
        int ag = 0;
        while (ag + 1 < S.n_agents && P.ars[ag + 1] <= r)
            ++ag;
        const int na = P.ars[ag + 1] - P.ars[ag], j = r - P.ars[ag];
        const int head = k >> 7, g = head / P.G, hl = head - g * P.G;
        const int qi = j * P.G + hl, rg = qi / ATT_QG;
        att_qq = qi - rg * ATT_QG;
        att_d = k & 127;
        att_nsp = (min(P.lens[ag] + na, P.kv_cap) + P.CH - 1) / P.CH;
        att_base = P.part + ((((size_t)ag * P.n_kvh + g) * P.n_rg + rg) * P.max_splits) * ATT_PART_FLOATS;
    }
    pdl_wait();
    trace_ready(a.trace);
    float4 own = make_float4(0.f, 0.f, 0.f, 0.f);  // RMSNorm: this thread's 4 values, kept from the sum pass
    if (S.kind == PREP_RMSNORM && live) {
        // the whole row's mean square, recomputed by every CTA of the row in the same
        // order; float4 index 256 * blockIdx.x + tid is this thread's own k .. k+3
        const float4 *h4 = reinterpret_cast<const float4 *>(S.xf + (size_t)r * S.ldx);
        const int mine = 256 * blockIdx.x + tid;
        float ss = 0.f;
        for (int i = tid; i < (K >> 2); i += 256) {
            const float4 v = h4[i];
            if (i == mine)
                own = v;
            ss = fmaf(v.x, v.x, ss);
            ss = fmaf(v.y, v.y, ss);
            ss = fmaf(v.z, v.z, ss);
            ss = fmaf(v.w, v.w, ss);
        }
        ss = warp_sum(ss);
        if ((tid & 31) == 0)
            red[tid >> 5] = ss;
        __syncthreads();
        if (tid == 0) {
            float tot = 0.f;
            for (int w = 0; w < 8; ++w)
                tot += red[w];
            s_inv = 1.f / sqrtf(tot / (float)K + S.eps);
        }
        __syncthreads();
    }
    uint16_t v[4] = {0, 0, 0, 0};
    if (act) {
        if (S.kind == PREP_BF16) {
            const uint2 w = *reinterpret_cast<const uint2 *>(S.xb + (size_t)r * S.ldx + k);
            v[0] = (uint16_t)(w.x & 0xFFFF);
            v[1] = (uint16_t)(w.x >> 16);
            v[2] = (uint16_t)(w.y & 0xFFFF);
            v[3] = (uint16_t)(w.y >> 16);
        } else if (S.kind == PREP_RMSNORM) {
            const float inv = s_inv;
            v[0] = f_to_bf16(own.x * inv);
            v[1] = f_to_bf16(own.y * inv);
            v[2] = f_to_bf16(own.z * inv);
            v[3] = f_to_bf16(own.w * inv);
        } else if (S.kind == PREP_SILU) {
            const float *gp = S.xf + (size_t)r * S.ldx;
            const float4 g = *reinterpret_cast<const float4 *>(gp + k);
            const float4 u = *reinterpret_cast<const float4 *>(gp + K + k);
            v[0] = f_to_bf16(silu_mul(g.x, u.x));
            v[1] = f_to_bf16(silu_mul(g.y, u.y));
            v[2] = f_to_bf16(silu_mul(g.z, u.z));
            v[3] = f_to_bf16(silu_mul(g.w, u.w));
        } else {
            // merge the key splits of query vector (row r, head k / 128), dims k%128 .. +3:
            // the global max first, then the weighted sums (the loads of each pass are
            // independent of one another, so they overlap)
            float Mx = -INFINITY;
            for (int sp = 0; sp < att_nsp; ++sp)
                Mx = fmaxf(Mx, att_base[(size_t)sp * ATT_PART_FLOATS + ATT_QG * 128 + att_qq]);
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            float Ls = 0.f;
            if (Mx != -INFINITY)
                for (int sp = 0; sp < att_nsp; ++sp) {
                    const float *pp = att_base + (size_t)sp * ATT_PART_FLOATS;
                    const float wgt = exp2f(pp[ATT_QG * 128 + att_qq] - Mx);
                    const float4 o = *reinterpret_cast<const float4 *>(pp + att_qq * 128 + att_d);
                    acc.x += wgt * o.x;
                    acc.y += wgt * o.y;
                    acc.z += wgt * o.z;
                    acc.w += wgt * o.w;
                    Ls += wgt * pp[ATT_QG * 128 + ATT_QG + att_qq];
                }
            const bool pos = Ls > 0.f;
            v[0] = f_to_bf16(pos ? acc.x / Ls : 0.f);
            v[1] = f_to_bf16(pos ? acc.y / Ls : 0.f);
            v[2] = f_to_bf16(pos ? acc.z / Ls : 0.f);
            v[3] = f_to_bf16(pos ? acc.w / Ls : 0.f);
        }
        if (S.dbg)
            *reinterpret_cast<uint2 *>(S.dbg + (size_t)r * S.ld_dbg + k) =
                make_uint2(v[0] | (uint32_t)v[1] << 16, v[2] | (uint32_t)v[3] << 16);
    }
    float x[4];
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[i] = bf16_to_f(v[i]);
        mx = fmaxf(mx, fabsf(x[i]));
    }
    // max over the block's two warps
    mx = warp_max(mx);
    if ((tid & 31) == 0)
        red[tid >> 5] = mx;
    __syncthreads();
    mx = fmaxf(red[2 * q], red[2 * q + 1]);
    int e = 0;
    if (mx > 0.f) {
        int E;
        frexpf(mx, &E);  // mx in [2^(E-1), 2^E)
        e = min(126, max(-126, 10 - E));
    }
    if (b >= nblk) {
        zero_next_output(S);
        trace_end(a.trace);
        return;
    }
    const float sc = ldexpf(1.f, e);
    uint8_t *rec = a.fb.rec + (size_t)b * REC_BYTES;
    const float h0 = round_half(x[0] * sc), h1 = round_half(x[1] * sc), h2 = round_half(x[2] * sc),
                h3 = round_half(x[3] * sc);
    // MMA positions 4t .. 4t+3 (k chunk t / 2, half t & 1 of the row's 16 bytes) hold columns 4t + {0,2,1,3}
    *reinterpret_cast<uint2 *>(rec + (t >> 1) * 256 + r * 16 + (t & 1) * 8) =
        make_uint2(pack_half2(h0, h2), pack_half2(h1, h3));
    if (FMT == 4) {
        // sub-block j = t >> 3 is the 8 lanes t & ~7 .. +7 (fp32 sum of its fp16 values)
        float sj = (h0 + h1) + (h2 + h3);
        sj += __shfl_xor_sync(0xffffffffu, sj, 1);
        sj += __shfl_xor_sync(0xffffffffu, sj, 2);
        sj += __shfl_xor_sync(0xffffffffu, sj, 4);
        const float sj1 = __shfl_down_sync(0xffffffffu, sj, 8);  // sub-block j + 1
        if ((t & 15) == 0) {
            const int j = t >> 3;  // even
            const float hi0 = round_half(sj), hi1 = round_half(sj1);
            *reinterpret_cast<uint32_t *>(rec + REC_S_OFF + r * 16 + 2 * j) = pack_half2(hi0, hi1);
            *reinterpret_cast<uint32_t *>(rec + REC_S_OFF + 256 + r * 16 + 2 * j) = pack_half2(sj - hi0, sj1 - hi1);
        }
    }
    if (t == 0)
        reinterpret_cast<float *>(rec + REC_RS_OFF)[r] = live ? ldexpf(1.f, -e) : 0.f;
    zero_next_output(S);  // last: the next GEMM's output is not read by this kernel
    trace_end(a.trace);
}

// ------------------------------------------------------------- GEMM kernel (tcgen05)
//
// One CTA per SM, persistent over a contiguous run of units (stream-K); a unit
// is a tile of 128 weight rows x one 256-wide block. The weights of a unit are
// decoded once, in registers, into exact fp16 tensor-core operands that go
// straight to tensor memory, and the 5th-generation tensor core multiplies
// them with the block's 16-row activation operand:
//
//   weight producer (1 thread)  TMA: 128 rows x one block -> raw stage   [SR-deep ring]
//   record producer (1 thread)  bulk copy: the block's operand record    [SB-deep ring]
//   16 decode warps             raw stage -> A = sc*q (Q4_K) or sc*(q-32) (Q6_K) as fp16
//                               in TMEM: two groups of 8 take alternate units; warp w
//                               covers lane quarter w & 3 (thread = weight row = TMEM
//                               lane) and k half (w >> 2) & 1       [2 A buffers x 2 halves]
//   2 MMA warps                 per unit 16 x tcgen05.mma M=128 N=16 K=16 (A from TMEM,
//                               B from shared memory) into the unit's accumulator, plus
//                               for Q4_K one more for the mins (A = m_j, B = sub-block
//                               sums); warp k takes the units of decode group k, the
//                               whole warp runs the loop and one elected lane issues
//   4 epilogue warps            y = d * acc - dmin * acc_mins (per row), times the
//                               activation row scales, summed over the tile's blocks
//                               in registers, added into Y with fp32 atomics when the
//                               run leaves the tile                       [NACC slots]
//
// A decode warp does 128 weights of each of its 32 rows per unit: per-unit
// synchronisation (one raw-stage wait, one A-half wait, a few arrivals) costs
// several hundred cycles, so a warp's share of a unit must be large, and two
// groups keep two units in flight in the two A buffers TMEM has room for.
// The k order inside the operands: A column c of a block holds the weights at
// k = 4 (c / 2) + (c & 1) + {0, 2} (the pair a nibble mask gives without
// shifting), so MMA position 4 t + {0, 1, 2, 3} carries block position
// 4 t + {0, 2, 1, 3}; the record builder writes the activations in that order.
// Every mbarrier wait is bounded: on a timeout the CTA records a status, stops
// issuing, waits for its own copies and MMAs, frees its tensor memory and
// exits.

namespace tg {
constexpr int TILE = 128;                      // weight rows per unit (MMA M, TMEM lanes)
constexpr int NCOL = 16;                       // activation rows (MMA N)
constexpr int DW = 16;                         // decode warps: 2 groups x 2 k halves x 4 lane quarters
constexpr int EW = 4;                          // epilogue warps
constexpr int NG = 2;                          // decode groups = MMA warps = A buffers
constexpr int W_PROD = DW + EW, W_REC = W_PROD + 1, W_MMA = W_REC + 1;
constexpr int THREADS = 32 * (W_MMA + NG);
constexpr int NACC = 4;                        // TMEM accumulator slots
constexpr int SB = 4;                          // operand-record stages
constexpr int ND = 8;                          // ring of per-unit d, dmin (decode -> epilogue)
static_assert(NACC % NG == 0 && SB % NG == 0, "a group's units use fixed slots and stages");
static_assert(ND >= NG + NACC, "a d slot is rewritten only after its epilogue has read it");
constexpr uint32_t COL_A = 0;                  // A buffers: 128 columns each (256 fp16 per row)
constexpr uint32_t COL_MA = 128 * NG;          // mins operand: 8 columns per A buffer
constexpr uint32_t COL_ACC = 288;              // accumulator slots: 16 (product) + 16 (mins) columns
static_assert(COL_MA + 8 * NG <= COL_ACC && COL_ACC + 32 * NACC <= 512, "TMEM map");
constexpr int Q6A = 208;                       // plane A bytes per Q6_K block
template <int FMT>
struct Stg {
    static constexpr int SR = FMT == 4 ? 8 : 6;             // raw weight stages (even: a stage keeps one group)
    static constexpr int ROW = FMT == 4 ? 144 : Q6A;
    static constexpr int W = TILE * ROW;                    // weight bytes per unit
    static constexpr int D = FMT == 4 ? 0 : TILE * 16;      // Q6_K: 8 fp16 d per row (aligned group of 8 blocks)
    static constexpr int RAW = (W + D + 127) / 128 * 128;
    static constexpr int NBAR = 2 * SR + 2 * SB + 4 * NG + 2 * NACC + ND + NG;
    static constexpr size_t SMEM = 128 + (size_t)SR * RAW + (size_t)SB * REC_BYTES + (size_t)ND * TILE * 8 + 8 * NBAR + 16;
    static_assert(SR % NG == 0, "raw stages alternate between the decode groups");
    static_assert(SMEM <= 232448, "shared memory per CTA");
};
enum { ST_RAW = 1, ST_REC = 2, ST_A = 3, ST_ACC = 4, ST_DONE = 5 };
}  // namespace tg

struct WeightMaps {
    CUtensorMap w;  // Q4_K matrix, or Q6_K plane A
    CUtensorMap d;  // Q6_K plane D (unused for Q4_K)
};

struct GemmArgs {
    int N, nblk, M, ldy, units;
    const uint8_t *rec;  // operand records, REC_BYTES apart
    float *Y;
    unsigned long long *trace;
};

// (v, v) as fp16 pair from byte i of w (an integer 0..255): 1024 + v built in the
// mantissa, 1024 subtracted exactly.
__device__ __forceinline__ uint32_t byte_h2(uint32_t w, uint32_t i)
{
    return hsub2(prmt(w, 0x64u, 0x4040u | i | (i << 8)), H2_1024);
}

// Q4_K: 64 weights of this thread's row (k part p = quant bytes 32p .. 32p + 31,
// sub-blocks 2p (low nibbles) and 2p + 1 (high nibbles)) as 32 exact fp16 pairs
// sc_j * q in column order (16 h + 2 i + s: h = high nibble, i = quant word,
// s = the word shifted by one byte).
__device__ __forceinline__ void decode_q4(const uint8_t *blk, int p, uint32_t (&out)[32])
{
    const uint4 h = lds_v4(blk);
    const uint32_t scA = h.y & 0x3F3F3F3Fu;                                    // sc_0..3
    const uint32_t scB = (h.w & 0x0F0F0F0Fu) | ((h.y >> 2) & 0x30303030u);     // sc_4..7
    const uint32_t scw = p < 2 ? scA : scB;
    const uint32_t bo = 2u * (uint32_t)(p & 1);
    const uint32_t SC0 = byte_h2(scw, bo);                                     // (sc_2p, sc_2p)
    const uint32_t NG0 = hmul2(SC0, H2_NEG1024);
    // the high nibble enters as 1024 + 16 q: scale sc / 16, offset -64 sc
    const uint32_t SC1 = hfma2(prmt(scw, 0x64u, 0x4040u | (bo + 1) | ((bo + 1) << 8)), H2_SIXTEENTH, H2_NEG64);
    const uint32_t NG1 = hmul2(SC1, H2_NEG1024);
    const uint4 qa = lds_v4(blk + 16 + 32 * p), qb = lds_v4(blk + 32 + 32 * p);
    const uint32_t w8[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t w = w8[i], ws = w >> 8;
        out[2 * i] = hfma2(and_or(w, 0x000F000Fu, H2_1024), SC0, NG0);
        out[2 * i + 1] = hfma2(and_or(ws, 0x000F000Fu, H2_1024), SC0, NG0);
        out[16 + 2 * i] = hfma2(and_or(w, 0x00F000F0u, H2_1024), SC1, NG1);
        out[16 + 2 * i + 1] = hfma2(and_or(ws, 0x00F000F0u, H2_1024), SC1, NG1);
    }
}

// Q4_K mins operand of this thread's row: (m_0, m_1) .. (m_6, m_7) twice (K = 16:
// the first 8 meet the high parts of the sub-block sums, the last 8 the low parts).
__device__ __forceinline__ void decode_q4_mins(const uint8_t *blk, uint32_t (&mm)[8])
{
    const uint4 h = lds_v4(blk);
    const uint32_t mA = h.z & 0x3F3F3F3Fu;                                     // m_0..3
    const uint32_t mB = ((h.w >> 4) & 0x0F0F0F0Fu) | ((h.z >> 2) & 0x30303030u);  // m_4..7
    mm[0] = hsub2(prmt(mA, 0x64u, 0x4140u), H2_1024);
    mm[1] = hsub2(prmt(mA, 0x64u, 0x4342u), H2_1024);
    mm[2] = hsub2(prmt(mB, 0x64u, 0x4140u), H2_1024);
    mm[3] = hsub2(prmt(mB, 0x64u, 0x4342u), H2_1024);
    mm[4] = mm[0];
    mm[5] = mm[1];
    mm[6] = mm[2];
    mm[7] = mm[3];
}

// Q6_K-like: this thread's k part p (half hh = p >> 1, l range 16 (p & 1) ..
// + 15) gives 64 weights in four sub-blocks sb = 8 hh + 2 m + (p & 1), m = 0..3
// (quants at k = 128 hh + 32 m + l); out[8 m + 2 i + s] = sc_sb * (q - 32) as
// fp16 pairs, i = quant word, s = shifted pair. Exact when |sc (q - 32)| <= 2048
// (always for scales in -64..64), else within half an fp16 ulp (2^-11 relative).
__device__ __forceinline__ void decode_q6(const uint8_t *blk, int p, uint32_t (&out)[32])
{
    const int hh = p >> 1, lh = p & 1;
    const uint2 sw = lds_v2(blk + 192 + 8 * hh);  // scales 8 hh .. 8 hh + 7
    const uint32_t sv[2] = {sw.x ^ 0x80808080u, sw.y ^ 0x80808080u};  // biased: sc + 128
    uint32_t SC[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {  // scale index 2 m + lh inside the 8: word m >> 1, byte 2 (m & 1) + lh
        const uint32_t bi = 2u * (uint32_t)(m & 1) + (uint32_t)lh;
        SC[m] = hsub2(prmt(sv[m >> 1], 0x64u, 0x4040u | bi | (bi << 8)), H2_1152);  // (1024 + sc + 128) - 1152
    }
    const uint4 L0 = lds_v4(blk + 64 * hh + 16 * lh), L1 = lds_v4(blk + 64 * hh + 32 + 16 * lh);
    const uint4 HH = lds_v4(blk + 128 + 32 * hh + 16 * lh);
    const uint32_t l0[4] = {L0.x, L0.y, L0.z, L0.w}, l1[4] = {L1.x, L1.y, L1.z, L1.w};
    const uint32_t hw[4] = {HH.x, HH.y, HH.z, HH.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t qt[4];
        qt[0] = (l0[i] & 0x0F0F0F0Fu) | ((hw[i] << 4) & 0x30303030u);
        qt[1] = (l1[i] & 0x0F0F0F0Fu) | ((hw[i] << 2) & 0x30303030u);
        qt[2] = ((l0[i] >> 4) & 0x0F0F0F0Fu) | (hw[i] & 0x30303030u);
        qt[3] = ((l1[i] >> 4) & 0x0F0F0F0Fu) | ((hw[i] >> 2) & 0x30303030u);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            out[8 * m + 2 * i] = hmul2(hsub2(prmt(qt[m], 0x64u, 0x4240u), H2_1056), SC[m]);
            out[8 * m + 2 * i + 1] = hmul2(hsub2(prmt(qt[m], 0x64u, 0x4341u), H2_1056), SC[m]);
        }
    }
}

// Pipeline waits: a waiting warp is suspended in the mbarrier try_wait until the
// phase completes, so it takes no issue slots from the warps doing the work
// (polling with a short sleep between tries measured 2% slower per step).
#define QAD_TG_WAIT(bar, par) mbar_wait(bar, par)
#define QAD_TG_WAIT_SLOW(bar, par) mbar_wait(bar, par)

template <int FMT>
__global__ void __launch_bounds__(tg::THREADS, 1) k_qgemm_tc(const __grid_constant__ WeightMaps maps, GemmArgs a)
{
    using namespace tg;
    using G = Stg<FMT>;
    constexpr int SR = G::SR;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~(uintptr_t)127);
    uint8_t *RAW = smem;
    uint8_t *RECS = RAW + (size_t)SR * G::RAW;
    float2 *DD = reinterpret_cast<float2 *>(RECS + (size_t)SB * REC_BYTES);  // [ND][TILE] (d, dmin) per unit
    uint64_t *bar = reinterpret_cast<uint64_t *>(DD + ND * TILE);
    uint64_t *raw_full = bar, *raw_empty = bar + SR, *b_full = bar + 2 * SR, *b_empty = b_full + SB;
    uint64_t *a_full = b_empty + SB, *a_empty = a_full + 2 * NG;  // [buffer][k half]
    uint64_t *acc_full = a_empty + 2 * NG, *acc_empty = acc_full + NACC, *dd_full = acc_empty + NACC;
    uint64_t *done = dd_full + ND;  // one per MMA warp
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + NG);
    __shared__ int s_bad;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u0 = (int)((long long)blockIdx.x * a.units / gridDim.x);
    const int u1 = (int)((long long)(blockIdx.x + 1) * a.units / gridDim.x);
    const int n_units = u1 - u0;
    if (threadIdx.x == 0) {
        s_bad = 0;
        for (int i = 0; i < SR; ++i) {
            mbar_init(&raw_full[i], 1);
            mbar_init(&raw_empty[i], DW / NG);  // the 8 warps of the stage's group
        }
        for (int i = 0; i < SB; ++i) {
            mbar_init(&b_full[i], 1);
            mbar_init(&b_empty[i], EW);
        }
        for (int i = 0; i < 2 * NG; ++i) {
            mbar_init(&a_full[i], 4);  // the four lane-quarter warps of one k half
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < NACC; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], EW);
        }
        for (int i = 0; i < ND; ++i)
            mbar_init(&dd_full[i], 4);  // the k-half-0 warps of the unit's group
        for (int i = 0; i < NG; ++i)
            mbar_init(&done[i], 1);
        mbar_fence_init();
    }
    if (warp == W_MMA) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    trace_start(a.trace);
    pdl_trigger();
    auto fail = [&](int code) {
        atomicExch(&g_gemm_status, code);
        atomicExch(&s_bad, 1);
    };
    auto bad = [&]() { return *(volatile int *)&s_bad != 0; };

    if (warp == W_PROD) {
        // ------------------------------------------------ weights by TMA (independent of the previous kernel)
        if (lane == 0) {
            int i = 0;
            for (; i < n_units && !bad(); ++i) {
                if (i >= SR && !QAD_TG_WAIT_SLOW(&raw_empty[i % SR], ((i / SR) - 1) & 1)) {
                    fail(ST_RAW);
                    break;
                }
                const int u = u0 + i, t = u / a.nblk, b = u - t * a.nblk;
                uint8_t *st = RAW + (size_t)(i % SR) * G::RAW;
                uint64_t *bb = &raw_full[i % SR];
                mbar_arrive_expect_tx(bb, (uint32_t)(G::W + G::D));
                tma_load_2d(st, &maps.w, b * G::ROW, t * TILE, bb);
                if (FMT == 6)
                    tma_load_2d(st + G::W, &maps.d, b & ~7, t * TILE, bb);
            }
            for (int k = max(0, i - SR); k < i; ++k)  // every issued copy lands before teardown
                if (!mbar_wait(&raw_full[k % SR], (k / SR) & 1, 20000))
                    fail(ST_RAW);
        }
    } else if (warp == W_REC) {
        // ------------------------------------------------ operand records (written by the previous kernel)
        pdl_wait();
        if (a.trace && lane == 0)
            atomicMin(a.trace + 1, gtimer());  // past the dependency wait
        if (lane == 0) {
            const int stall = blockIdx.x == 0 ? *(volatile int *)&g_gemm_stall - 1 : -1;
            int i = 0;
            for (; i < n_units && !bad() && i != stall; ++i) {
                const int b = (u0 + i) % a.nblk, bs = i % SB;
                if (i >= SB && !QAD_TG_WAIT_SLOW(&b_empty[bs], ((i / SB) - 1) & 1)) {
                    fail(ST_REC);
                    break;
                }
                mbar_arrive_expect_tx(&b_full[bs], (uint32_t)REC_BYTES);
                bulk_g2s(RECS + (size_t)bs * REC_BYTES, a.rec + (size_t)b * REC_BYTES, REC_BYTES, &b_full[bs]);
            }
            for (int k = max(0, i - SB); k < i; ++k)
                if (!mbar_wait(&b_full[k % SB], (k / SB) & 1, 20000))
                    fail(ST_REC);
        }
    } else if (warp >= W_MMA) {
        // ------------------------------------------------ MMA warps: warp g multiplies the units of decode group g;
        // the whole warp runs the loop with warp-uniform operands, one elected lane issues
        constexpr uint32_t idesc = umma_idesc_f16(TILE, NCOL);
        const int g = warp - W_MMA;
        const uint32_t at = tmem + COL_A + 128 * g;
        bool issued = false;
        for (int i = g; i < n_units; i += NG) {
            const int bs = i % SB, c = i % NACC;
            bool ok = __all_sync(0xffffffffu, QAD_TG_WAIT(&b_full[bs], (i / SB) & 1)) &&
                      (i < NACC || __all_sync(0xffffffffu, QAD_TG_WAIT(&acc_empty[c], ((i / NACC) - 1) & 1)));
            const uint32_t rb = smem_u32(RECS + (size_t)bs * REC_BYTES);
            const uint64_t bdesc = umma_desc_k_noswz(rb, 256, 128);  // + 32 per 512-byte k step (16-byte units)
            const uint32_t acc = tmem + COL_ACC + 32 * c;
#pragma unroll
            for (int h = 0; h < 2 && ok; ++h) {  // k half h (k steps 8h .. 8h+7) once its four warps wrote it
                if (!__all_sync(0xffffffffu, QAD_TG_WAIT(&a_full[2 * g + h], (i / NG) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (FMT == 4 && h == 0)
                    umma_f16_ts_warp(acc + 16, tmem + COL_MA + 8 * g, bdesc + (REC_S_OFF >> 4), idesc, 0);
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const int k = 8 * h + m;
                    umma_f16_ts_warp(acc, at + 8 * k, bdesc + 32 * k, idesc, k != 0);
                }
                issued = true;
                umma_commit_warp(&a_empty[2 * g + h]);
            }
            if (!ok) {
                fail(ST_A);
                break;
            }
            umma_commit_warp(&acc_full[c]);
        }
        if (issued) {  // every MMA this warp issued completes before TMEM is freed
            umma_commit_warp(&done[g]);
            if (!__all_sync(0xffffffffu, mbar_wait(&done[g], 0, 20000)))
                fail(ST_DONE);
        }
    } else if (warp < DW) {
        // ------------------------------------------------ decode: group g, k half h, lane quarter q
        const int g = warp >> 3, h = (warp >> 2) & 1, q = warp & 3;
        const int row = 32 * q + lane;
        const uint32_t lanes = (uint32_t)(32 * q) << 16;
        const uint32_t abase = tmem + lanes + COL_A + 128 * g;
        int b = n_units > g ? (u0 + g) % a.nblk : 0;
        for (int i = g; i < n_units; i += NG) {
            const int s = i % SR;
            if (!__all_sync(0xffffffffu, QAD_TG_WAIT(&raw_full[s], (i / SR) & 1)) ||
                (i >= NG && !__all_sync(0xffffffffu, QAD_TG_WAIT(&a_empty[2 * g + h], ((i / NG) - 1) & 1)))) {
                fail(ST_RAW);
                break;
            }
            tc_fence_after();
            const uint8_t *st = RAW + (size_t)s * G::RAW;
            const uint8_t *blk = st + (size_t)row * G::ROW;
#pragma unroll
            for (int pp = 0; pp < 2; ++pp) {  // the half's two k parts (64 weights each)
                const int p = 2 * h + pp;
                uint32_t out[32];
                if (FMT == 4) {
                    decode_q4(blk, p, out);
                    tmem_st_x32(abase + 32 * p, out);
                } else {
                    decode_q6(blk, p, out);
                    const uint32_t base = abase + 8 * (8 * (p >> 1) + (p & 1));
#pragma unroll
                    for (int m = 0; m < 4; ++m)  // sub-block 8 hh + 2 m + lh: columns 8 sb .. 8 sb + 7
                        tmem_st_x8(base + 16 * m, out + 8 * m);
                }
            }
            if (h == 0) {  // the mins operand and the block's d (and dmin) of this row for the epilogue
                float2 dv;
                if (FMT == 4) {
                    uint32_t mm[8];
                    decode_q4_mins(blk, mm);
                    tmem_st_x8(tmem + lanes + COL_MA + 8 * g, mm);
                    const uint32_t hd = lds_u32(blk);
                    dv = make_float2(half_lo(hd), half_hi(hd));
                } else {
                    const uint32_t dw = lds_u32(st + G::W + row * 16 + (b & 6) * 2);
                    dv = make_float2((b & 1) ? half_hi(dw) : half_lo(dw), 0.f);
                }
                DD[(i % ND) * TILE + row] = dv;
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&a_full[2 * g + h]);
                mbar_arrive(&raw_empty[s]);
                if (h == 0)
                    mbar_arrive(&dd_full[i % ND]);
            }
            b += NG;
            if (b >= a.nblk)
                b -= a.nblk;
        }
    } else {
        // ------------------------------------------------ epilogue: per-block scales, sum over the tile's blocks
        pdl_wait();  // Y was prepared (zeroed) by the previous kernel
        const int q = warp - DW, row = 32 * q + lane;
        const uint32_t lanes = (uint32_t)(32 * q) << 16;
        float tot[NCOL];
#pragma unroll
        for (int r = 0; r < NCOL; ++r)
            tot[r] = 0.f;
        int t = n_units > 0 ? u0 / a.nblk : 0, b = u0 - t * a.nblk;
        for (int i = 0; i < n_units; ++i) {
            const int bs = i % SB, c = i % NACC;
            // d (and dmin) of this row for unit i: published by the unit's k-half-0 decode warps.
            // The slot is rewritten for unit i + ND only after the MMAs of unit i + ND - NG started,
            // which needs this warp's release of unit i + ND - NG - NACC >= i.
            if (!__all_sync(0xffffffffu, QAD_TG_WAIT_SLOW(&dd_full[i % ND], (i / ND) & 1))) {
                fail(ST_RAW);
                break;
            }
            const float2 dv = DD[(i % ND) * TILE + row];
            const float d = dv.x, dmin = dv.y;
            if (!__all_sync(0xffffffffu, QAD_TG_WAIT_SLOW(&acc_full[c], (i / NACC) & 1)) ||
                !__all_sync(0xffffffffu, QAD_TG_WAIT_SLOW(&b_full[bs], (i / SB) & 1))) {
                fail(ST_ACC);
                break;
            }
            tc_fence_after();
            uint32_t acc[16], accm[16];
            tmem_ld_x16(tmem + lanes + COL_ACC + 32 * c, acc);
            if (FMT == 4)
                tmem_ld_x16(tmem + lanes + COL_ACC + 32 * c + 16, accm);
            tmem_wait_ld();
            tc_fence_before();
            const float *RS = reinterpret_cast<const float *>(RECS + (size_t)bs * REC_BYTES + REC_RS_OFF);
            float rs[NCOL];
#pragma unroll
            for (int r = 0; r < NCOL; r += 4) {
                const uint4 v = lds_v4(RS + r);
                rs[r] = __uint_as_float(v.x);
                rs[r + 1] = __uint_as_float(v.y);
                rs[r + 2] = __uint_as_float(v.z);
                rs[r + 3] = __uint_as_float(v.w);
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&acc_empty[c]);
                mbar_arrive(&b_empty[bs]);
            }
#pragma unroll
            for (int r = 0; r < NCOL; ++r) {
                const float y = FMT == 4 ? fmaf(d, __uint_as_float(acc[r]), -dmin * __uint_as_float(accm[r]))
                                         : d * __uint_as_float(acc[r]);
                tot[r] = fmaf(rs[r], y, tot[r]);
            }
            if (++b == a.nblk || i + 1 == n_units) {
                const int n = t * TILE + row;
                if (n < a.N)
#pragma unroll
                    for (int r = 0; r < NCOL; ++r)
                        if (r < a.M)
                            atomicAdd(a.Y + (size_t)r * a.ldy + n, tot[r]);
#pragma unroll
                for (int r = 0; r < NCOL; ++r)
                    tot[r] = 0.f;
                b = 0;
                ++t;
            }
        }
    }
    trace_end(a.trace);
    tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Q6_K-like GGUF blocks -> packed device layout (plane A: first 208 bytes of
// each block; plane D: d, rows padded to a multiple of 8 blocks with zeros).
__global__ void k_q6k_pack(const uint8_t *__restrict__ W, int N, int nblk, uint8_t *__restrict__ P)
{
    const int nblk8 = (nblk + 7) & ~7;
    uint8_t *A = P;
    uint16_t *D = reinterpret_cast<uint16_t *>(P + (size_t)N * nblk * tg::Q6A);
    const long long total = (long long)N * nblk;
    for (long long blk = blockIdx.x * (long long)(blockDim.x / 32) + threadIdx.x / 32; blk < total;
         blk += (long long)gridDim.x * (blockDim.x / 32)) {
        const uint8_t *src = W + blk * 210;
        uint8_t *dst = A + blk * tg::Q6A;
        for (int i = threadIdx.x & 31; i < tg::Q6A; i += 32)
            dst[i] = src[i];
        if ((threadIdx.x & 31) == 0) {
            const long long n = blk / nblk, b = blk - n * nblk;
            D[n * nblk8 + b] = (uint16_t)(src[208] | src[209] << 8);
            if (b == nblk - 1)
                for (int p = nblk; p < nblk8; ++p)
                    D[n * nblk8 + p] = 0;
        }
    }
}

size_t q6k_packed_bytes(long long N, int K)
{
    const int nblk = K / 256, nblk8 = (nblk + 7) & ~7;
    return (size_t)N * nblk * tg::Q6A + (size_t)N * nblk8 * 2;
}

// ------------------------------------------------------------- launchers

template <typename K>
static int set_smem(K kernel, size_t bytes)
{
    return cuda_check(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes),
                      "cudaFuncSetAttribute");
}

int frag_nt(int) { return 2; }

int launch_prep(int fmt, int K, int M, const PrepSrc &src, const FragBuf &fb, cudaStream_t s, bool pdl,
                unsigned long long *trace)
{
    PrepArgs a{src, K, M, fb, trace};
    void (*kern)(PrepArgs) = fmt == 4 ? k_prep<4> : k_prep<6>;
    const dim3 grid((K / 256 + 3) / 4, QAD_MAX_ROWS);
    cudaError_t e = pdl ? launch_pdl(kern, grid, dim3(256), 0, s, a)
                        : (kern<<<grid, 256, 0, s>>>(a), cudaGetLastError());
    return cuda_check(e, "prep launch");
}

int make_weight_maps(int fmt, const void *W, int N, int K, WeightMapsBlob *out)
{
    static_assert(sizeof(WeightMapsBlob) >= sizeof(WeightMaps), "blob too small");
    WeightMaps *m = reinterpret_cast<WeightMaps *>(out);
    const int nblk = K / 256;
    if (fmt == 4)
        return encode_tmap_2d(&m->w, W, 1, (uint64_t)nblk * 144, (uint64_t)N, (uint64_t)nblk * 144, 144, tg::TILE);
    int rc = encode_tmap_2d(&m->w, W, 1, (uint64_t)nblk * tg::Q6A, (uint64_t)N, (uint64_t)nblk * tg::Q6A, tg::Q6A,
                            tg::TILE);
    if (rc)
        return rc;
    const int nblk8 = (nblk + 7) & ~7;
    const uint8_t *D = (const uint8_t *)W + (size_t)N * nblk * tg::Q6A;
    return encode_tmap_2d(&m->d, D, 2, (uint64_t)nblk8, (uint64_t)N, (uint64_t)nblk8 * 2, 8, tg::TILE);
}

int launch_gemm(int fmt, const WeightMapsBlob &maps_blob, int N, int K, int M, const FragBuf &fb, float *Y, int ldy,
                cudaStream_t s, bool pdl, unsigned long long *trace)
{
    const WeightMaps &maps = reinterpret_cast<const WeightMaps &>(maps_blob);
    GemmArgs a;
    a.N = N;
    a.nblk = K / 256;
    a.M = M;
    a.ldy = ldy;
    a.units = ((N + tg::TILE - 1) / tg::TILE) * a.nblk;
    a.rec = fb.rec;
    a.Y = Y;
    a.trace = trace;
    void (*kern)(const WeightMaps, GemmArgs) = fmt == 4 ? k_qgemm_tc<4> : k_qgemm_tc<6>;
    const size_t smem = fmt == 4 ? tg::Stg<4>::SMEM : tg::Stg<6>::SMEM;
    static bool done[64][2] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const int v = fmt == 4 ? 0 : 1;
    if (dev < 0 || dev >= 64 || !done[dev][v]) {
        int rc = set_smem(kern, smem);
        if (rc)
            return rc;
        if (dev >= 0 && dev < 64)
            done[dev][v] = true;
    }
    const int grid = num_sms();
    cudaError_t e = pdl ? launch_pdl(kern, dim3(grid), dim3(tg::THREADS), smem, s, maps, a)
                        : (kern<<<grid, tg::THREADS, smem, s>>>(maps, a), cudaGetLastError());
    return cuda_check(e, "gemm launch");
}

int launch_q6k_pack(const void *W, int N, int K, void *P, cudaStream_t s)
{
    const long long blocks = (long long)N * (K / 256);
    long long grid = (blocks + 7) / 8;
    if (grid > 65535LL * 16)
        grid = 65535LL * 16;
    k_q6k_pack<<<(unsigned)grid, 256, 0, s>>>((const uint8_t *)W, N, K / 256, (uint8_t *)P);
    return cuda_check(cudaGetLastError(), "q6k pack launch");
}

}  // namespace qad

// ------------------------------------------------------------- C ABI

extern "C" int qad_device_status(int reset)
{
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, qad::g_gemm_status, sizeof(int));
    if (e != cudaSuccess)
        return qad::cuda_check(e, "qad_device_status");
    if (reset && v) {
        const int z = 0;
        e = cudaMemcpyToSymbol(qad::g_gemm_status, &z, sizeof(int));
        if (e != cudaSuccess)
            return qad::cuda_check(e, "qad_device_status reset");
    }
    return v;
}

namespace qad {
int gemm_set_stall(int at)
{
    const int v = at < 0 ? 0 : at + 1;
    return cuda_check(cudaMemcpyToSymbol(g_gemm_stall, &v, sizeof(int)), "gemm stall hook");
}
}  // namespace qad

extern "C" int qad_debug_stall(int kernel, int at)
{
    if (kernel == 0)
        return qad::gemm_set_stall(at);
    if (kernel == 1)
        return qad::dense_set_stall(at);
    if (kernel == 2)
        return qad::prefill_set_stall(at);
    return qad::fail(QAD_ERR_INVALID, "qad_debug_stall: unknown kernel %d", kernel);
}

extern "C" size_t qad_gemm_ws_bytes(int K, int M)
{
    if (K <= 0 || K % 256 || M < 1 || M > QAD_MAX_ROWS)
        return 0;
    return qad::frag_bytes(K, 2);  // the larger layout: valid for every backend and row count
}

extern "C" size_t qad_q6k_packed_bytes(long long N, int K)
{
    if (N <= 0 || K <= 0 || K % 256)
        return 0;
    return qad::q6k_packed_bytes(N, K);
}

extern "C" int qad_q6k_pack(const void *W, int N, int K, void *W_packed, void *stream)
{
    if (!W || !W_packed || N <= 0 || K <= 0)
        return qad::fail(QAD_ERR_INVALID, "qad_q6k_pack: null pointer or non-positive size");
    if (K % 256)
        return qad::fail(QAD_ERR_UNSUPPORTED, "qad_q6k_pack: K %% 256 != 0");
    if ((uintptr_t)W_packed & 15)
        return qad::fail(QAD_ERR_INVALID, "qad_q6k_pack: packed weights must be 16-byte aligned");
    return qad::launch_q6k_pack(W, N, K, W_packed, (cudaStream_t)stream);
}

static int gemm_entry(int fmt, const void *W, int N, int K, const uint16_t *X, int M, float *Y, int accumulate,
                      void *ws, size_t ws_bytes, void *stream)
{
    const char *name = fmt == 4 ? "qad_q4k_gemm" : "qad_q6k_gemm";
    if (!W || !X || !Y || !ws || N <= 0 || K <= 0 || M <= 0)
        return qad::fail(QAD_ERR_INVALID, "%s: null pointer or non-positive size (N=%d K=%d M=%d)", name, N, K, M);
    if (M > QAD_MAX_ROWS || K % 256 || K > 65536)
        return qad::fail(QAD_ERR_UNSUPPORTED, "%s: need 1 <= M <= 16 and K %% 256 == 0, K <= 65536 (M=%d K=%d)",
                         name, M, K);
    if ((uintptr_t)ws & 255)
        return qad::fail(QAD_ERR_INVALID, "%s: workspace must be 256-byte aligned", name);
    if ((uintptr_t)W & 15)
        return qad::fail(QAD_ERR_INVALID, "%s: weights must be 16-byte aligned", name);
    if ((uintptr_t)X & 7)
        return qad::fail(QAD_ERR_INVALID, "%s: activations must be 8-byte aligned", name);
    if (ws_bytes < qad_gemm_ws_bytes(K, M))
        return qad::fail(QAD_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", name, ws_bytes, qad_gemm_ws_bytes(K, M));
    qad::WeightMapsBlob maps;
    int rc = qad::make_weight_maps(fmt, W, N, K, &maps);
    if (rc)
        return rc;
    cudaStream_t s = (cudaStream_t)stream;
    qad::FragBuf fb = qad::frag_carve(ws, K, qad::frag_nt(M));
    qad::PrepSrc src = {};
    src.kind = qad::PREP_BF16;
    src.xb = X;
    src.ldx = K;
    if (!accumulate) {
        src.zero = Y;
        src.zero_n = (long long)M * N;
    }
    rc = qad::launch_prep(fmt, K, M, src, fb, s, false);
    if (rc)
        return rc;
    return qad::launch_gemm(fmt, maps, N, K, M, fb, Y, N, s, true);
}

extern "C" int qad_q4k_gemm(const void *W, int N, int K, const uint16_t *X, int M, float *Y, int accumulate, void *ws,
                            size_t ws_bytes, void *stream)
{
    return gemm_entry(4, W, N, K, X, M, Y, accumulate, ws, ws_bytes, stream);
}

extern "C" int qad_q6k_gemm(const void *W, int N, int K, const uint16_t *X, int M, float *Y, int accumulate, void *ws,
                            size_t ws_bytes, void *stream)
{
    return gemm_entry(6, W, N, K, X, M, Y, accumulate, ws, ws_bytes, stream);
}

// ------------------------------------------------------------- allocation-free variant
//
// Some callers cannot allocate device memory when they run this GEMM: servers
// that reserve all of HBM for weights and KV-cache pools at start-up and
// forbid later allocations, code that must not trigger the device-wide
// synchronisation cudaFree can cause while other streams are decoding, and
// plain C integrations that only hold pointers to buffers owned elsewhere.
// For them the activation-fragment scratch lives in a fixed array of device
// memory that every GPU loading this library keeps until the process exits.

// 1 MiB holds the operand records of K <= 30464 (119 blocks of 8,768 bytes) for
// every row count from 1 to 16: the record layout does not depend on M.
static constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)1 << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// The array's host-side name is not a device address: resolve it with the
// device current. Outside stream capture the address is looked up on every call
// (a device reset reloads the module and may move the array); a call made while
// its stream is being captured reuses the address found by an earlier call on
// that device, and fails if there is none.
static void *noalloc_scratch_address(cudaStream_t stream, int *rc)
{
    static void *addr[64] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        *rc = qad::cuda_check(e, "qad_q4k_gemm_noalloc: cudaGetDevice");
        return nullptr;
    }
    if (dev < 0 || dev >= 64) {
        *rc = qad::fail(QAD_ERR_UNSUPPORTED, "qad_q4k_gemm_noalloc: device ordinal %d >= 64", dev);
        return nullptr;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) {
        *rc = qad::cuda_check(e, "qad_q4k_gemm_noalloc: cudaStreamIsCapturing");
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (cap == cudaStreamCaptureStatusNone) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) {
            *rc = qad::cuda_check(e, "qad_q4k_gemm_noalloc: cudaGetSymbolAddress");
            return nullptr;
        }
        addr[dev] = p;
    } else if (!addr[dev]) {
        *rc = qad::fail(QAD_ERR_INVALID,
                        "qad_q4k_gemm_noalloc: first call on device %d made during stream capture; make one call "
                        "before capturing",
                        dev);
        return nullptr;
    }
    *rc = QAD_OK;
    return addr[dev];
}

extern "C" size_t qad_q4k_gemm_noalloc_scratch_bytes(void) { return NOALLOC_SCRATCH_BYTES; }

extern "C" int qad_q4k_gemm_noalloc(const void *W, int N, int K, const uint16_t *X, int M, float *Y, int accumulate,
                                    void *stream)
{
    if (!W || !X || !Y || N <= 0 || K <= 0 || M <= 0)
        return qad::fail(QAD_ERR_INVALID, "qad_q4k_gemm_noalloc: null pointer or non-positive size (N=%d K=%d M=%d)",
                         N, K, M);
    if (M > QAD_MAX_ROWS || K % 256)
        return qad::fail(QAD_ERR_UNSUPPORTED, "qad_q4k_gemm_noalloc: need 1 <= M <= 16 and K %% 256 == 0");
    const size_t need = qad_gemm_ws_bytes(K, M);
    if (need > NOALLOC_SCRATCH_BYTES)
        return qad::fail(QAD_ERR_UNSUPPORTED,
                         "qad_q4k_gemm_noalloc: K=%d with M=%d needs %zu bytes of scratch; the fixed array holds %zu "
                         "(use qad_q4k_gemm with a workspace)",
                         K, M, need, NOALLOC_SCRATCH_BYTES);
    int rc = QAD_OK;
    void *scratch = noalloc_scratch_address((cudaStream_t)stream, &rc);
    if (!scratch)
        return rc;
    return gemm_entry(4, W, N, K, X, M, Y, accumulate, scratch, NOALLOC_SCRATCH_BYTES, stream);
}
