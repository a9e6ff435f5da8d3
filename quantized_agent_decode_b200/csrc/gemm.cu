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
//  * A producer warp streams each unit (a tile of weight rows x one 256-wide
//    block) into a ring of shared-memory stages with one 2-D tensor-map load
//    (TMA), plus one bulk copy of that block's activation record; each stage
//    completes on an mbarrier. Every quantized byte leaves HBM exactly once.
//  * The block is decoded in registers into fp16 tensor-core operands that are
//    EXACT: for Q4_K, A = sc_j * q (<= 945) and the mins enter through a second
//    small MMA against per-sub-block activation sums; for Q6_K, A = sc * (q-32)
//    (|.| <= 4096). The fp16 values come from the "1024 + q" exponent trick (OR
//    of the nibble into the mantissa of 1024.0) followed by one fused
//    multiply-add that applies the scale.
//  * M = 12 rows need ~16 multiply-adds per weight, four times what the FP32
//    pipes deliver at the HBM rate, so the product runs on the tensor cores as
//    m16n8k16 warp MMAs (weights = A, the 16 padded activation rows = B). Each
//    consumer warp owns 32 weight rows (two m16 tiles), so every activation
//    fragment read from shared memory feeds four MMAs.
//  * The activations are prepared once per GEMM (k_prep) into fp16 B
//    fragments in exactly the register order each lane consumes, with a
//    power-of-two scale per (row, block) so fp16's range always holds them.
//  * Work is split stream-K style over a persistent grid (one CTA per SM):
//    each CTA takes a contiguous run of units, its consumer groups take them
//    round-robin and accumulate in registers, adding partial tile sums into Y
//    with fp32 atomics when a group's run leaves a tile.
//  * Programmatic dependent launch: the first units' weights are requested
//    before griddepcontrol.wait, so the weight stream starts while the
//    producer of the activations is still finishing.
#include <cuda.h>

#include <mutex>

#include "gemm.cuh"


namespace qad {

// Set by a GEMM whose pipeline wait timed out (1: a consumer, 2: the producer);
// read and cleared by qad_device_status().
__device__ int g_gemm_status;

// ------------------------------------------------------------- fragment layout
// Activation rows r = 8*nt + g (nt < NT, g < 8); blocks b < nblk; k-steps
// s < 16; lane quad c < 4. One record per block (rec_bytes), so a GEMM unit
// fetches its block's operand with one bulk copy and a warp's 32 lanes read 32
// consecutive entries.
//   X (uint2 units): [s][g][c][nt] = {b0, b1}: the two B registers of the
//       m16n8k16 fragment: b0 = (x[k0], x[k0+2]), b1 = (x[k0+1], x[k0+3]) with
//       k0 = 256 b + frag_k0(s, c), as fp16 of x * 2^e(r,b).
//   S (uint2 units): [g][c][nt] = {(Shi_2c, Shi_2c+1), (Slo_2c, Slo_2c+1)}
//       with S_j the sum of the 32 fp16 activations of Q4_K sub-block j split
//       into two fp16 parts (Q4_K only).
//   RS: 16 floats, 2^-e(r,b) (0 for rows >= M).
// e(r,b) puts the block's largest |x| in [512, 1024): fp16 holds every bf16
// value of the block exactly unless it is 2^24 times smaller than that max.
static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t frag_bytes(int K, int nt) { return align256((size_t)(K / 256) * rec_bytes(4, nt)); }

FragBuf frag_carve(void *ws, int, int)
{
    FragBuf f;
    f.rec = (uint8_t *)ws;
    return f;
}

// Which activation column feeds logical k-slot (s, c). The weight-side decode
// below produces, for lane quad c and k-step s, the weights at within-block
// positions k0, k0+2 (first B register) and k0+1, k0+3 (second).
__host__ __device__ constexpr int frag_k0(int fmt, int s, int c)
{
    // Q4_K: quant bytes 32c..32c+31: word s>>1, low (s even) or high (s odd) nibbles.
    // Q6_K: half c>>1, l-range 16*(c&1); word s>>2; s&3 selects the 32-weight quarter.
    return fmt == 4 ? 64 * c + 4 * (s >> 1) + 32 * (s & 1) : 128 * (c >> 1) + 16 * (c & 1) + 4 * (s >> 2) + 32 * (s & 3);
}

// The inverse: the slot (s, c) whose k0 is 4t (t < 64), so thread t of a block
// reads columns 4t..4t+3 and its loads coalesce. For Q4_K, t >> 3 is the
// sub-block 2c + (s & 1).
__host__ __device__ constexpr int slot_s(int fmt, int t)
{
    return fmt == 4 ? 2 * (t & 7) + ((t >> 3) & 1) : 4 * (t & 3) + ((t & 31) >> 3);
}
__host__ __device__ constexpr int slot_c(int fmt, int t) { return fmt == 4 ? t >> 4 : 2 * (t >> 5) + ((t >> 2) & 1); }

constexpr bool slot_maps_consistent()
{
    for (int fmt = 4; fmt <= 6; fmt += 2)
        for (int t = 0; t < 64; ++t)
            if (frag_k0(fmt, slot_s(fmt, t), slot_c(fmt, t)) != 4 * t || slot_s(fmt, t) > 15 || slot_c(fmt, t) > 3)
                return false;
    return true;
}
static_assert(slot_maps_consistent(), "fragment slot maps must invert frag_k0");

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

// Grid (ceil(nblk / 4), 8*NT): CTA (x, r) forms row r's blocks 4x..4x+3, one
// 64-thread quarter per block, thread t of a quarter owning columns 4t..4t+3.
// The values are formed exactly as the GEMM must see them (bf16: the input
// itself, RMSNorm of the fp32 residual, silu(gate)*up, or the merged
// attention output), then scaled per (row, block) into fp16 fragments.
template <int FMT, int NT>
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
    uint8_t *rec = a.fb.rec + (size_t)b * rec_bytes(FMT, NT);
    const int g = r & 7, nt = r >> 3;
    const int s = slot_s(FMT, t), c = slot_c(FMT, t);
    const float h0 = round_half(x[0] * sc), h1 = round_half(x[1] * sc), h2 = round_half(x[2] * sc),
                h3 = round_half(x[3] * sc);
    reinterpret_cast<uint2 *>(rec)[((s * 8 + g) * 4 + c) * NT + nt] =
        make_uint2(pack_half2(h0, h2), pack_half2(h1, h3));
    if (FMT == 4) {
        // sub-block j = t >> 3 is the 8 lanes t & ~7 .. +7 (fp32 sum of its fp16 values)
        float sj = (h0 + h1) + (h2 + h3);
        sj += __shfl_xor_sync(0xffffffffu, sj, 1);
        sj += __shfl_xor_sync(0xffffffffu, sj, 2);
        sj += __shfl_xor_sync(0xffffffffu, sj, 4);
        const float sj1 = __shfl_down_sync(0xffffffffu, sj, 8);  // sub-block j + 1
        if ((t & 15) == 0) {
            const float hi0 = round_half(sj), hi1 = round_half(sj1);
            reinterpret_cast<uint2 *>(rec + 4096 * NT)[(g * 4 + c) * NT + nt] =
                make_uint2(pack_half2(hi0, hi1), pack_half2(sj - hi0, sj1 - hi1));
        }
    }
    if (t == 0)
        reinterpret_cast<float *>(rec + rec_bytes(FMT, NT) - 64)[r] = live ? ldexpf(1.f, -e) : 0.f;
    zero_next_output(S);  // last: the next GEMM's output is not read by this kernel
    trace_end(a.trace);
}

// ------------------------------------------------------------- GEMM kernels
//
// One CTA per SM: 8 consumer warps + 1 producer warp. A CTA unit is a tile of
// 128 weight rows x one 256-wide block. Units are numbered tile-major with the
// block fastest, and each CTA takes a contiguous run of them (stream-K). For
// each unit the producer issues ONE 2-D tensor-map load (TMA) of the 128
// row-blocks (plus the d plane for Q6_K) and one bulk copy of the block's
// activation fragments into a ring of shared-memory stages, completing on a
// "full" mbarrier; the consumer warps (16 rows each) decode their rows from
// shared memory, run the MMAs and release the stage on an "empty" mbarrier.
// Every wait is bounded: on timeout the warp records a status code and returns.
//
// Q6_K-like weights use the packed device layout of qad_q6k_pack(): plane A
// [N][nblk][208] (ql, qh, int8 scales: the first 208 bytes of each GGUF block,
// so every field is 16-byte aligned) followed by plane D [N][ceil8(nblk)] fp16
// d. 210-byte GGUF blocks cannot be addressed by TMA (16-byte start rule).

constexpr int RW = 32;               // weight rows per consumer warp (two m16 tiles)
constexpr int Q6A_BYTES = 208;       // plane A bytes per Q6_K block

// CG consumer groups of GW warps take units round-robin; each warp owns RW
// weight rows of the unit. Stages are reused every S units and S is a multiple
// of CG, so unit i and unit i + S (the next use of a stage) belong to the same
// group: a group never waits on a stage phase whose predecessor it has not
// itself seen complete (parity waits cannot tell phase u from phase u - 2).
// Consumer groups per CTA (build-time tunables).
#ifndef QAD_Q4_GROUPS
#define QAD_Q4_GROUPS 3
#endif
#ifndef QAD_Q6_GROUPS
#define QAD_Q6_GROUPS 2
#endif
template <int FMT>
struct Cfg {
    static constexpr int GW = 4;                       // warps per consumer group
    static constexpr int CG = FMT == 4 ? QAD_Q4_GROUPS : QAD_Q6_GROUPS;  // consumer groups
    static constexpr int TILE = RW * GW;               // weight rows per unit
    static constexpr int S = 6;                        // pipeline stages
    static constexpr int THREADS = 32 * (CG * GW + 1);
    static constexpr int ROW_BYTES = FMT == 4 ? 144 : Q6A_BYTES;
    static_assert(S % CG == 0, "stage reuse must stay within one consumer group");
};

template <int FMT, int NT>
struct Stage {
    static constexpr int W_BYTES = Cfg<FMT>::TILE * Cfg<FMT>::ROW_BYTES;
    static constexpr int D_BYTES = FMT == 4 ? 0 : Cfg<FMT>::TILE * 16;  // 8 fp16 d per row (aligned group of 8 blocks)
    static constexpr int X_BYTES = 4096 * NT;                          // the block's operand record:
    static constexpr int S_BYTES = FMT == 4 ? 256 * NT : 0;            //   X, S, then 16 row scales
    static constexpr int R_BYTES = rec_bytes(FMT, NT);
    static constexpr int COPY_BYTES = W_BYTES + D_BYTES + R_BYTES;     // what lands per unit
    // every stage starts on a 128-byte boundary (tensor-map copy destinations)
    static constexpr int BYTES = (COPY_BYTES + 127) / 128 * 128;
    static_assert(W_BYTES % 128 == 0 && D_BYTES % 128 == 0 && R_BYTES % 16 == 0, "stage field alignment");
};

template <int FMT, int NT>
constexpr size_t gemm_smem_bytes()
{
    return (size_t)Cfg<FMT>::S * Stage<FMT, NT>::BYTES + 2 * Cfg<FMT>::S * sizeof(uint64_t);
}

struct WeightMaps {
    CUtensorMap w;  // Q4_K matrix, or Q6_K plane A
    CUtensorMap d;  // Q6_K plane D (unused for Q4_K)
};

struct GemmArgs {
    int N, nblk, M, ldy, units;
    const uint8_t *rec;  // operand records, rec_bytes(FMT, NT) apart
    float *Y;
    unsigned long long *trace;
};

enum { ERR_FULL_TIMEOUT = 1, ERR_EMPTY_TIMEOUT = 2 };

// Add a warp's partial sums of 16 weight rows (n0 + g, n0 + g + 8) to Y.
template <int NT>
__device__ __forceinline__ void flush_rows(float (&tot)[NT][4], const GemmArgs &a, int n0, int g, int c)
{
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int n = n0 + g + 8 * (e >> 1);
            const int r = 8 * nt + 2 * c + (e & 1);
            if (n < a.N && r < a.M)
                atomicAdd(a.Y + (size_t)r * a.ldy + n, tot[nt][e]);
            tot[nt][e] = 0.f;
        }
}

template <int NT>
__device__ __forceinline__ void lds_b(const uint8_t *p, uint32_t (&b)[NT][2])
{
    if (NT == 2) {
        const uint4 v = lds_v4(p);
        b[0][0] = v.x;
        b[0][1] = v.y;
        b[NT - 1][0] = v.z;
        b[NT - 1][1] = v.w;
    } else {
        const uint2 v = lds_v2(p);
        b[0][0] = v.x;
        b[0][1] = v.y;
    }
}

__device__ __forceinline__ uint32_t u4w(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Row scales 2^-e(r,b) of the activation rows this lane's accumulators hold.
template <int NT>
__device__ __forceinline__ void lds_rs(const uint8_t *RS, int c, float (&rs)[NT][2])
{
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const float2 v = lds_v2f(RS + 4 * (8 * nt + 2 * c));
        rs[nt][0] = v.x;
        rs[nt][1] = v.y;
    }
}

// One Q4_K block of this warp's 32 weight rows (tiles mt = 0, 1; this lane
// decodes rows 16 mt + g and 16 mt + g + 8, indexed q = 2 mt + rh) against
// all activation rows. W: the warp's first row in the stage; XS/SS/RS: the
// block's operand record.
template <int NT>
__device__ __forceinline__ void q4_block(const uint8_t *W, const uint8_t *XS, const uint8_t *SS, const uint8_t *RS,
                                         int g, int c, uint32_t selT, bool hib, float (&tot)[2][NT][4])
{
    uint32_t SCl[4], NGl[4], SCh[4], NGh[4], AM[4];
    float dd[4], dm[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 h = lds_v4(W + (16 * (q >> 1) + g + 8 * (q & 1)) * 144);
        // scales/mins of sub-blocks 2c and 2c+1 (bytes (2c)&3, +1 of the packed words)
        const uint32_t scA = h.y & 0x3F3F3F3Fu, mA = h.z & 0x3F3F3F3Fu;
        const uint32_t scB = (h.w & 0x0F0F0F0Fu) | ((h.y >> 2) & 0x30303030u);
        const uint32_t mB = ((h.w >> 4) & 0x0F0F0F0Fu) | ((h.z >> 2) & 0x30303030u);
        const uint32_t T = prmt(hib ? scB : scA, hib ? mB : mA, selT);  // [sc_lo, sc_hi, m_lo, m_hi]
        const uint32_t Tl = prmt(T, 0x64u, 0x4040u);                     // 1024 + sc_lo (x2)
        const uint32_t Th = prmt(T, 0x64u, 0x4141u);                     // 1024 + sc_hi (x2)
        const uint32_t Tm = prmt(T, 0x64u, 0x4342u);                     // 1024 + (m_lo, m_hi)
        SCl[q] = hsub2(Tl, H2_1024);                                     // sc_lo
        NGl[q] = hmul2(SCl[q], H2_NEG1024);                              // -1024 sc_lo
        SCh[q] = hfma2(Th, H2_SIXTEENTH, H2_NEG64);                      // sc_hi / 16
        NGh[q] = hmul2(SCh[q], H2_NEG1024);                              // -64 sc_hi
        AM[q] = hsub2(Tm, H2_1024);                                      // (m_lo, m_hi)
        dd[q] = half_lo(h.x);
        dm[q] = half_hi(h.x);
    }
    float acc[2][NT][4];
    const uint8_t *xl = XS + (g * 4 + c) * 8 * NT;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        uint4 qw[4];  // quant words 4 half .. 4 half + 3 of this lane's 32 bytes, per row
#pragma unroll
        for (int q = 0; q < 4; ++q)
            qw[q] = lds_v4(W + (16 * (q >> 1) + g + 8 * (q & 1)) * 144 + 16 + 32 * c + 16 * half);
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const int i = 4 * half + ii;
            uint32_t blo[NT][2], bhi[NT][2];
            lds_b<NT>(xl + (2 * i) * 256 * NT, blo);
            lds_b<NT>(xl + (2 * i + 1) * 256 * NT, bhi);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int q0 = 2 * mt, q1 = 2 * mt + 1;
                const uint32_t w0 = u4w(qw[q0], ii), w1 = u4w(qw[q1], ii);
                const uint32_t w0s = w0 >> 8, w1s = w1 >> 8;
                // low nibbles: sub-block 2c, k-step 2i
                const uint32_t a0 = hfma2(and_or(w0, 0x000F000Fu, H2_1024), SCl[q0], NGl[q0]);
                const uint32_t a1 = hfma2(and_or(w1, 0x000F000Fu, H2_1024), SCl[q1], NGl[q1]);
                const uint32_t a2 = hfma2(and_or(w0s, 0x000F000Fu, H2_1024), SCl[q0], NGl[q0]);
                const uint32_t a3 = hfma2(and_or(w1s, 0x000F000Fu, H2_1024), SCl[q1], NGl[q1]);
                // high nibbles: sub-block 2c+1, k-step 2i+1
                const uint32_t c0 = hfma2(and_or(w0, 0x00F000F0u, H2_1024), SCh[q0], NGh[q0]);
                const uint32_t c1 = hfma2(and_or(w1, 0x00F000F0u, H2_1024), SCh[q1], NGh[q1]);
                const uint32_t c2 = hfma2(and_or(w0s, 0x00F000F0u, H2_1024), SCh[q0], NGh[q0]);
                const uint32_t c3 = hfma2(and_or(w1s, 0x00F000F0u, H2_1024), SCh[q1], NGh[q1]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (i == 0)
                        mma_f16_zero(acc[mt][nt], a0, a1, a2, a3, blo[nt][0], blo[nt][1]);
                    else
                        mma_f16(acc[mt][nt], a0, a1, a2, a3, blo[nt][0], blo[nt][1]);
                    mma_f16(acc[mt][nt], c0, c1, c2, c3, bhi[nt][0], bhi[nt][1]);
                }
            }
        }
    }
    // mins: sum_j m_j * S_j, S split into two fp16 parts along k
    uint32_t sb[NT][2];
    lds_b<NT>(SS + (g * 4 + c) * 8 * NT, sb);
    float rs[NT][2];
    lds_rs<NT>(RS, c, rs);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float accm[4];
            mma_f16_zero(accm, AM[2 * mt], AM[2 * mt + 1], AM[2 * mt], AM[2 * mt + 1], sb[nt][0], sb[nt][1]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int q = 2 * mt + (e >> 1);
                const float y = fmaf(dd[q], acc[mt][nt][e], -dm[q] * accm[e]);
                tot[mt][nt][e] = fmaf(rs[nt][e & 1], y, tot[mt][nt][e]);
            }
        }
}


// One Q6_K-like block (packed layout) of this warp's 32 weight rows. A: the
// warp's first row in plane A of the stage; D: its first row of the d tile.
template <int NT>
__device__ __forceinline__ void q6_block(const uint8_t *A, const uint8_t *D, int bsub, const uint8_t *XS,
                                         const uint8_t *RS, int g, int c, float (&tot)[2][NT][4])
{
    uint32_t SC[4][4];
    float dd[4];
    const int h = c >> 1, lq = 16 * (c & 1);
    const uint32_t j = (uint32_t)(c & 1);
    const uint32_t sel0 = j | 0x40u | (j << 8) | 0x4000u, sel1 = (j + 2) | 0x40u | ((j + 2) << 8) | 0x4000u;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int row = 16 * (q >> 1) + g + 8 * (q & 1);
        const uint8_t *blk = A + row * Q6A_BYTES;
        // int8 scales of sub-blocks 8h + 2t + (c&1): bytes (c&1) + 2t of the 8 scale bytes
        const uint2 sw = lds_v2(blk + 192 + 8 * h);
        const uint32_t s0 = sw.x ^ 0x80808080u, s1 = sw.y ^ 0x80808080u;
        // (sc + 128) + 1024 - 1152 = sc, exact in fp16
        SC[q][0] = hsub2(prmt(s0, 0x64u, sel0), H2_1152);
        SC[q][1] = hsub2(prmt(s0, 0x64u, sel1), H2_1152);
        SC[q][2] = hsub2(prmt(s1, 0x64u, sel0), H2_1152);
        SC[q][3] = hsub2(prmt(s1, 0x64u, sel1), H2_1152);
        const uint32_t dw = lds_u32(D + row * 16 + (bsub & 6) * 2);
        dd[q] = __half2float(__ushort_as_half((unsigned short)(dw >> ((bsub & 1) * 16))));
    }
    float acc[2][NT][4];
    const uint8_t *xl = XS + (g * 4 + c) * 8 * NT;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        uint2 L0[4], L1[4], HH[4];  // words 2 half, 2 half + 1 of ql (two quarters) and qh, per row
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint8_t *blk = A + (16 * (q >> 1) + g + 8 * (q & 1)) * Q6A_BYTES;
            L0[q] = lds_v2(blk + 64 * h + lq + 8 * half);
            L1[q] = lds_v2(blk + 64 * h + 32 + lq + 8 * half);
            HH[q] = lds_v2(blk + 128 + 32 * h + lq + 8 * half);
        }
#pragma unroll
        for (int ii = 0; ii < 2; ++ii) {
            const int i = 2 * half + ii;
            uint32_t qt[4][4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t l0 = ii ? L0[q].y : L0[q].x, l1 = ii ? L1[q].y : L1[q].x;
                const uint32_t hh = ii ? HH[q].y : HH[q].x;
                qt[q][0] = (l0 & 0x0F0F0F0Fu) | ((hh << 4) & 0x30303030u);
                qt[q][1] = (l1 & 0x0F0F0F0Fu) | ((hh << 2) & 0x30303030u);
                qt[q][2] = ((l0 >> 4) & 0x0F0F0F0Fu) | (hh & 0x30303030u);
                qt[q][3] = ((l1 >> 4) & 0x0F0F0F0Fu) | ((hh >> 2) & 0x30303030u);
            }
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int s = 4 * i + t;
                uint32_t bf[NT][2];
                lds_b<NT>(xl + s * 256 * NT, bf);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    const int q0 = 2 * mt, q1 = 2 * mt + 1;
                    // pairs (bytes 0,2) and (bytes 1,3) -> 1024 + q -> q - 32 -> sc*(q-32)
                    const uint32_t a0 = hmul2(hsub2(prmt(qt[q0][t], 0x64u, 0x4240u), H2_1056), SC[q0][t]);
                    const uint32_t a1 = hmul2(hsub2(prmt(qt[q1][t], 0x64u, 0x4240u), H2_1056), SC[q1][t]);
                    const uint32_t a2 = hmul2(hsub2(prmt(qt[q0][t], 0x64u, 0x4341u), H2_1056), SC[q0][t]);
                    const uint32_t a3 = hmul2(hsub2(prmt(qt[q1][t], 0x64u, 0x4341u), H2_1056), SC[q1][t]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (s == 0)
                            mma_f16_zero(acc[mt][nt], a0, a1, a2, a3, bf[nt][0], bf[nt][1]);
                        else
                            mma_f16(acc[mt][nt], a0, a1, a2, a3, bf[nt][0], bf[nt][1]);
                    }
                }
            }
        }
    }
    float rs[NT][2];
    lds_rs<NT>(RS, c, rs);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                tot[mt][nt][e] = fmaf(dd[2 * mt + (e >> 1)] * rs[nt][e & 1], acc[mt][nt][e], tot[mt][nt][e]);
}

template <int FMT, int NT>
__global__ void __launch_bounds__(Cfg<FMT>::THREADS, 1) k_qgemm(const __grid_constant__ WeightMaps maps, GemmArgs a)
{
    extern __shared__ __align__(128) uint8_t smem[];
    using St = Stage<FMT, NT>;
    using Cf = Cfg<FMT>;
    constexpr int S = Cf::S, GW = Cf::GW, CG = Cf::CG, TILE = Cf::TILE;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)S * St::BYTES);
    uint64_t *empty = full + S;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u0 = (int)((long long)blockIdx.x * a.units / gridDim.x);
    const int u1 = (int)((long long)(blockIdx.x + 1) * a.units / gridDim.x);
    const int n_units = u1 - u0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], GW);  // the warps of the consumer group that used the stage
        }
        mbar_fence_init();
    }
    __syncthreads();
    trace_start(a.trace);
    pdl_trigger();

    if (warp == CG * GW) {
        // ------------------------------------------------ producer warp (lane 0 issues)
        if (lane != 0) {
            pdl_wait();
            return;
        }
        auto issue = [&](int i, int t, int b, bool weights, bool frags) {
            uint8_t *st = smem + (size_t)(i % S) * St::BYTES;
            uint64_t *bar = &full[i % S];
            if (weights) {
                mbar_arrive_expect_tx(bar, (uint32_t)St::COPY_BYTES);
                tma_load_2d(st, &maps.w, b * Cf::ROW_BYTES, t * TILE, bar);
                if (FMT == 6)
                    tma_load_2d(st + St::W_BYTES, &maps.d, b & ~7, t * TILE, bar);
            }
            if (frags)
                bulk_g2s(st + St::W_BYTES + St::D_BYTES, a.rec + (size_t)b * St::R_BYTES, St::R_BYTES, bar);
        };
        const int pre = min(S, n_units);
        int t = n_units > 0 ? u0 / a.nblk : 0, b = u0 - t * a.nblk;
        for (int i = 0, tt = t, bb = b; i < pre; ++i) {
            issue(i, tt, bb, true, false);  // weights do not depend on the previous kernel
            if (++bb == a.nblk) {
                bb = 0;
                ++tt;
            }
        }
        pdl_wait();
        int i = 0;
        for (; i < pre; ++i) {
            issue(i, t, b, false, true);
            if (++b == a.nblk) {
                b = 0;
                ++t;
            }
        }
        for (; i < n_units; ++i) {
            if (!mbar_wait(&empty[i % S], ((i / S) - 1) & 1)) {
                atomicExch(&g_gemm_status, ERR_EMPTY_TIMEOUT);
                break;
            }
            issue(i, t, b, true, true);
            if (++b == a.nblk) {
                b = 0;
                ++t;
            }
        }
        // every issued copy lands before this CTA may exit
        for (int k = max(0, i - S); k < i; ++k)
            if (!mbar_wait(&full[k % S], (k / S) & 1, 20000))
                atomicExch(&g_gemm_status, ERR_FULL_TIMEOUT);
        trace_end(a.trace);
        return;
    }

    // ---------------------------------------------------- consumer groups (round-robin units)
    const int grp = warp / GW, wi = warp % GW;
    const int g = lane >> 2, c = lane & 3;
    const int jj = 2 * (c & 1);
    const uint32_t selT = (uint32_t)(jj | ((jj + 1) << 4) | ((jj + 4) << 8) | ((jj + 5) << 12));
    const bool hib = c >= 2;
    pdl_wait();
    trace_ready(a.trace);
    float tot[2][NT][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                tot[mt][nt][e] = 0.f;
    int t = 0, b = 0;
    if (grp < n_units) {
        t = (u0 + grp) / a.nblk;
        b = (u0 + grp) - t * a.nblk;
    }
    for (int i = grp; i < n_units; i += CG) {
        const uint8_t *st = smem + (size_t)(i % S) * St::BYTES;
        if (!mbar_wait(&full[i % S], (i / S) & 1)) {
            if (lane == 0)
                atomicExch(&g_gemm_status, ERR_FULL_TIMEOUT);
            return;
        }
        const uint8_t *XS = st + St::W_BYTES + St::D_BYTES;
        const uint8_t *RS = XS + St::R_BYTES - 64;
        if (FMT == 4)
            q4_block<NT>(st + (size_t)(RW * wi) * 144, XS, XS + St::X_BYTES, RS, g, c, selT, hib, tot);
        else
            q6_block<NT>(st + (size_t)(RW * wi) * Q6A_BYTES, st + St::W_BYTES + (size_t)(RW * wi) * 16, b & 7, XS, RS,
                         g, c, tot);
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[i % S]);
        // next unit of this group: CG blocks further along
        int tn = t, bn = b + CG;
        while (bn >= a.nblk) {
            bn -= a.nblk;
            ++tn;
        }
        if (tn != t || i + CG >= n_units) {
            flush_rows<NT>(tot[0], a, t * TILE + RW * wi, g, c);
            flush_rows<NT>(tot[1], a, t * TILE + RW * wi + 16, g, c);
        }
        t = tn;
        b = bn;
    }
    trace_end(a.trace);
}

// Q4_K form without a producer warp: 4 consumer groups of 4 warps (16 warps,
// so each SM sub-partition runs 4 consumers at the same register budget as 3
// consumers + the producer). Group grp consumes units grp, grp+4, ... through
// its own two ring slots (grp and grp+4 of 8) and refills a slot itself: after
// the group's 4 warps release unit i (one arrival each on the slot's empty
// barrier), lane 0 of the group's first warp issues unit i+8 into it. Before
// the wait on the previous kernel each group requests the weights of its first
// two units; every wait is bounded and reports through g_gemm_status.
#ifndef QAD_Q4_SELF_REFILL
#define QAD_Q4_SELF_REFILL 1
#endif
namespace sr {
constexpr int CG = 4, GW = 4, S = 8, THREADS = 32 * CG * GW;
}
template <int NT>
constexpr size_t gemm_sr_smem_bytes()
{
    return (size_t)sr::S * Stage<4, NT>::BYTES + 2 * sr::S * sizeof(uint64_t);
}

template <int NT>
__global__ void __launch_bounds__(sr::THREADS, 1) k_qgemm_sr(const __grid_constant__ WeightMaps maps, GemmArgs a)
{
    extern __shared__ __align__(128) uint8_t smem[];
    using St = Stage<4, NT>;
    constexpr int S = sr::S, GW = sr::GW, CG = sr::CG, TILE = Cfg<4>::TILE;
    static_assert(S % CG == 0 && TILE == RW * GW, "each group owns S / CG slots; a unit is GW warps of RW rows");
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)S * St::BYTES);
    uint64_t *empty = full + S;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = warp / GW, wi = warp % GW;
    const int u0 = (int)((long long)blockIdx.x * a.units / gridDim.x);
    const int u1 = (int)((long long)(blockIdx.x + 1) * a.units / gridDim.x);
    const int n_units = u1 - u0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], GW);
        }
        mbar_fence_init();
    }
    __syncthreads();
    trace_start(a.trace);
    pdl_trigger();
    const bool leader = wi == 0 && lane == 0;
    auto issue = [&](int i, bool weights, bool frags) {
        const int u = u0 + i, t = u / a.nblk, b = u - t * a.nblk;
        uint8_t *st = smem + (size_t)(i % S) * St::BYTES;
        uint64_t *bar = &full[i % S];
        if (weights) {
            mbar_arrive_expect_tx(bar, (uint32_t)St::COPY_BYTES);
            tma_load_2d(st, &maps.w, b * 144, t * TILE, bar);
        }
        if (frags)
            bulk_g2s(st + St::W_BYTES, a.rec + (size_t)b * St::R_BYTES, St::R_BYTES, bar);
    };
    int issued = -1;  // highest unit this group's leader has requested
    if (leader)
        for (int i = grp; i < n_units && i < S; i += CG) {
            issue(i, true, false);  // weights do not depend on the previous kernel
            issued = i;
        }
    pdl_wait();
    if (leader)
        for (int i = grp; i < n_units && i < S; i += CG)
            issue(i, false, true);
    trace_ready(a.trace);

    const int g = lane >> 2, c = lane & 3;
    const int jj = 2 * (c & 1);
    const uint32_t selT = (uint32_t)(jj | ((jj + 1) << 4) | ((jj + 4) << 8) | ((jj + 5) << 12));
    const bool hib = c >= 2;
    float tot[2][NT][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                tot[mt][nt][e] = 0.f;
    int t = 0, b = 0;
    if (grp < n_units) {
        t = (u0 + grp) / a.nblk;
        b = (u0 + grp) - t * a.nblk;
    }
    int done = grp - CG;  // last unit this warp consumed
    for (int i = grp; i < n_units; i += CG) {
        const uint8_t *st = smem + (size_t)(i % S) * St::BYTES;
        if (!mbar_wait(&full[i % S], (i / S) & 1)) {
            if (lane == 0)
                atomicExch(&g_gemm_status, ERR_FULL_TIMEOUT);
            break;
        }
        const uint8_t *XS = st + St::W_BYTES;
        const uint8_t *RS = XS + St::R_BYTES - 64;
        q4_block<NT>(st + (size_t)(RW * wi) * 144, XS, XS + St::X_BYTES, RS, g, c, selT, hib, tot);
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[i % S]);
        done = i;
        if (leader && i + S < n_units) {
            // the slot's next user is unit i + S of this group: refill it once all GW warps released it
            if (!mbar_wait(&empty[i % S], (i / S) & 1)) {
                atomicExch(&g_gemm_status, ERR_EMPTY_TIMEOUT);
            } else {
                issue(i + S, true, true);
                issued = i + S;
            }
        }
        int tn = t, bn = b + CG;
        while (bn >= a.nblk) {
            bn -= a.nblk;
            ++tn;
        }
        if (tn != t || i + CG >= n_units) {
            flush_rows<NT>(tot[0], a, t * TILE + RW * wi, g, c);
            flush_rows<NT>(tot[1], a, t * TILE + RW * wi + 16, g, c);
        }
        t = tn;
        b = bn;
    }
    // after an error exit, copies this group requested but did not consume land before the CTA exits
    if (leader)
        for (int k = done + CG; k <= issued; k += CG)
            if (!mbar_wait(&full[k % S], (k / S) & 1, 20000))
                atomicExch(&g_gemm_status, ERR_FULL_TIMEOUT);
    trace_end(a.trace);
}

// Q6_K-like GGUF blocks -> packed device layout (plane A: first 208 bytes of
// each block; plane D: d, rows padded to a multiple of 8 blocks with zeros).
__global__ void k_q6k_pack(const uint8_t *__restrict__ W, int N, int nblk, uint8_t *__restrict__ P)
{
    const int nblk8 = (nblk + 7) & ~7;
    uint8_t *A = P;
    uint16_t *D = reinterpret_cast<uint16_t *>(P + (size_t)N * nblk * Q6A_BYTES);
    const long long total = (long long)N * nblk;
    for (long long blk = blockIdx.x * (long long)(blockDim.x / 32) + threadIdx.x / 32; blk < total;
         blk += (long long)gridDim.x * (blockDim.x / 32)) {
        const uint8_t *src = W + blk * 210;
        uint8_t *dst = A + blk * Q6A_BYTES;
        for (int i = threadIdx.x & 31; i < Q6A_BYTES; i += 32)
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
    return (size_t)N * nblk * Q6A_BYTES + (size_t)N * nblk8 * 2;
}

// ------------------------------------------------------------- launchers

template <typename K>
static int set_smem(K kernel, size_t bytes)
{
    return cuda_check(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes),
                      "cudaFuncSetAttribute");
}

int frag_nt(int M) { return M <= 8 ? 1 : 2; }

int launch_prep(int fmt, int K, int M, const PrepSrc &src, const FragBuf &fb, cudaStream_t s, bool pdl,
                unsigned long long *trace)
{
    const int nt = frag_nt(M);
    PrepArgs a{src, K, M, fb, trace};
    void (*kern)(PrepArgs);
    if (fmt == 4)
        kern = nt == 1 ? k_prep<4, 1> : k_prep<4, 2>;
    else
        kern = nt == 1 ? k_prep<6, 1> : k_prep<6, 2>;
    const dim3 grid((K / 256 + 3) / 4, 8 * nt);
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
        return encode_tmap_2d(&m->w, W, 1, (uint64_t)nblk * 144, (uint64_t)N, (uint64_t)nblk * 144, 144,
                              Cfg<4>::TILE);
    int rc = encode_tmap_2d(&m->w, W, 1, (uint64_t)nblk * Q6A_BYTES, (uint64_t)N, (uint64_t)nblk * Q6A_BYTES,
                            Q6A_BYTES, Cfg<6>::TILE);
    if (rc)
        return rc;
    const int nblk8 = (nblk + 7) & ~7;
    const uint8_t *D = (const uint8_t *)W + (size_t)N * nblk * Q6A_BYTES;
    return encode_tmap_2d(&m->d, D, 2, (uint64_t)nblk8, (uint64_t)N, (uint64_t)nblk8 * 2, 8, Cfg<6>::TILE);
}

int launch_gemm(int fmt, const WeightMapsBlob &maps_blob, int N, int K, int M, const FragBuf &fb, float *Y, int ldy,
                cudaStream_t s, bool pdl, unsigned long long *trace)
{
    const int nt = frag_nt(M);
    const WeightMaps &maps = reinterpret_cast<const WeightMaps &>(maps_blob);
    GemmArgs a;
    a.N = N;
    a.nblk = K / 256;
    a.M = M;
    a.ldy = ldy;
    const int tile = fmt == 4 ? Cfg<4>::TILE : Cfg<6>::TILE;
    a.units = ((N + tile - 1) / tile) * a.nblk;
    a.rec = fb.rec;
    a.Y = Y;
    a.trace = trace;
    void (*kern)(const WeightMaps, GemmArgs);
    size_t smem;
    int threads = fmt == 4 ? Cfg<4>::THREADS : Cfg<6>::THREADS;
    if (fmt == 4 && QAD_Q4_SELF_REFILL) {
        kern = nt == 1 ? k_qgemm_sr<1> : k_qgemm_sr<2>;
        smem = nt == 1 ? gemm_sr_smem_bytes<1>() : gemm_sr_smem_bytes<2>();
        threads = sr::THREADS;
    } else if (fmt == 4) {
        kern = nt == 1 ? k_qgemm<4, 1> : k_qgemm<4, 2>;
        smem = nt == 1 ? gemm_smem_bytes<4, 1>() : gemm_smem_bytes<4, 2>();
    } else {
        kern = nt == 1 ? k_qgemm<6, 1> : k_qgemm<6, 2>;
        smem = nt == 1 ? gemm_smem_bytes<6, 1>() : gemm_smem_bytes<6, 2>();
    }
    static bool done[64][4] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const int v = (fmt == 4 ? 0 : 2) + (nt - 1);
    if (dev < 0 || dev >= 64 || !done[dev][v]) {
        int rc = set_smem(kern, smem);
        if (rc)
            return rc;
        if (dev >= 0 && dev < 64)
            done[dev][v] = true;
    }
    const int grid = num_sms();
    cudaError_t e = pdl ? launch_pdl(kern, dim3(grid), dim3(threads), smem, s, maps, a)
                        : (kern<<<grid, threads, smem, s>>>(maps, a), cudaGetLastError());
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

static constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)1 << 20;  // 1 MiB: K <= 30720 at 16 rows
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// The array's host-side name is not a device address: resolve it once per
// device (with that device current) and reuse the address.
static void *noalloc_scratch_address(int *rc)
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
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) {
            *rc = qad::cuda_check(e, "qad_q4k_gemm_noalloc: cudaGetSymbolAddress");
            return nullptr;
        }
        addr[dev] = p;
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
    void *scratch = noalloc_scratch_address(&rc);
    if (!scratch)
        return rc;
    return gemm_entry(4, W, N, K, X, M, Y, accumulate, scratch, NOALLOC_SCRATCH_BYTES, stream);
}
