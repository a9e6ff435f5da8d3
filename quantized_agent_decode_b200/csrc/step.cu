// step.cu -- one batched decode-and-verify step through the whole synthetic
// decoder stack, the model handle, CUDA-graph capture and the host-buffer
// entry point.
//
// [OpenJet page] = rebasdaily.com 2026-10-29, "OpenJet ... multi-agent
// serving", section 只搬一次权重: per step all active agents' rows (next
// token + two drafts each) form one batch, the weights stream once for the
// whole batch and each agent reads its own KV cache; the drafts are checked in
// the same forward pass. The page runs this as one persistent megakernel on an
// RTX 3090; here the step is a chain of sm_100a kernels linked by
// programmatic dependent launch (each GEMM starts streaming its weights while
// its producer drains) and replayed as one CUDA graph.
//
// Per layer, nine launches (rounding points as in the layer definition of qad.h):
//   prep(rmsnorm h)          -> fp16 fragments; zeroes the qkv buffer
//   q4k_gemm(Wqkv)           -> qkv fp32 (atomic partial sums)
//   decode_attn (fused)      -> per-split partials; Q, k, v rounded to bf16 from
//                               qkv, k and v appended at each row's position
//   prep(merge splits -> O)  -> O bf16 -> fragments
//   q4k_gemm(Wo)             -> h += ...
//   prep(rmsnorm h)          -> fragments; zeroes the gate|up buffer
//   q4k_gemm(Wgu)            -> gate|up fp32
//   prep(silu(gate) * up)    -> fragments (Q6_K order)
//   q6k_gemm(Wdown)          -> h += ...
#include <vector>

#include "attn.cuh"
#include "dense.cuh"
#include "gemm.cuh"

struct qad_step_graph {
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
};

// Kernel classes timed by the optional per-launch event profiler.
enum ProfKind { PK_INIT = 0, PK_PREP, PK_GEMM_QKV, PK_ATTN, PK_GEMM_O, PK_GEMM_GU, PK_GEMM_DOWN, PK_COUNT };

struct qad_model {
    qad_model_desc d;
    // per-launch event profiler (eager steps only)
    bool prof = false;
    std::vector<cudaEvent_t> prof_ev;
    std::vector<int> prof_kind;
    double prof_ms[PK_COUNT] = {};
    long long prof_n[PK_COUNT] = {};
    size_t prof_used = 0;
    bool prof_pending = false;
    std::vector<const void *> wqkv, wo, wgu, wdown;
    std::vector<qad::WeightMapsBlob> mqkv, mo, mgu, mdown;  // TMA descriptors, built once
    std::vector<uint16_t *> kc, vc;
    void *dbg = nullptr;
    size_t dbg_bytes = 0;
    unsigned long long *trace = nullptr;  // 3 words per launch (see trace_start)
    int trace_n = 0;
    // graph cache of the host-buffer entry point
    qad_step_graph *hg = nullptr;
    int hg_M = -1, hg_agents = -1, hg_rows = -1;
    void *hg_ws = nullptr;
    cudaStream_t hg_stream = nullptr;
};

namespace qad {

static inline size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

struct StepLayout {
    size_t qkv, gu, frag, part, x_in, ars_in, lens_in, h_out, total;
    AttnPlan plan;
};

// Largest attention-partials footprint over the launch shapes a step of M
// rows can take (n_agents <= max_agents, rows per agent <= M).
static size_t max_part_bytes(const qad_model_desc &d, int M)
{
    size_t best = 0;
    for (int na = 1; na <= d.max_agents; ++na)
        for (int rows = 1; rows <= M; ++rows) {
            size_t b = attn_plan(na, d.n_qh, d.n_kvh, d.kv_cap, rows).part_bytes;
            if (b > best)
                best = b;
        }
    return best;
}

static StepLayout step_layout(const qad_model_desc &d, int M)
{
    StepLayout L;
    const int nq = d.n_qh * d.head_dim, nqkv = (d.n_qh + 2 * d.n_kvh) * d.head_dim;
    const int nt = 2;  // the larger fragment layout serves every backend and row count
    size_t off = 0;
    L.qkv = off;
    off += a256((size_t)M * nqkv * 4);
    L.gu = off;
    off += a256((size_t)M * 2 * d.inter * 4);
    L.frag = off;
    size_t fb = frag_bytes(d.hidden, nt);
    if (frag_bytes(nq, nt) > fb)
        fb = frag_bytes(nq, nt);
    if (frag_bytes(d.inter, nt) > fb)
        fb = frag_bytes(d.inter, nt);
    off += a256(fb);
    L.part = off;
    off += a256(max_part_bytes(d, M));
    L.x_in = off;
    off += a256((size_t)M * d.hidden * 2);
    L.ars_in = off;
    off += a256((size_t)(d.max_agents + 1) * 4);
    L.lens_in = off;
    off += a256((size_t)d.max_agents * 4);
    L.h_out = off;
    off += a256((size_t)M * d.hidden * 4);
    L.total = off;
    return L;
}

// Debug intermediates of one layer (teacher-forced parity checks).
struct DbgLayout {
    size_t x1, qkv, attn, hmid, x2, gu, act, hout, per_layer;
};
static DbgLayout dbg_layout(const qad_model_desc &d, int M)
{
    DbgLayout L;
    const int nq = d.n_qh * d.head_dim, nqkv = (d.n_qh + 2 * d.n_kvh) * d.head_dim;
    size_t off = 0;
    L.x1 = off;
    off += a256((size_t)M * d.hidden * 2);
    L.qkv = off;
    off += a256((size_t)M * nqkv * 4);
    L.attn = off;
    off += a256((size_t)M * nq * 2);
    L.hmid = off;
    off += a256((size_t)M * d.hidden * 4);
    L.x2 = off;
    off += a256((size_t)M * d.hidden * 2);
    L.gu = off;
    off += a256((size_t)M * 2 * d.inter * 4);
    L.act = off;
    off += a256((size_t)M * d.inter * 2);
    L.hout = off;
    off += a256((size_t)M * d.hidden * 4);
    L.per_layer = off;
    return L;
}

// h[r][k] = X[r][k] (bf16 -> fp32): the residual stream starts at the input rows.
__global__ void k_init_h(const uint16_t *__restrict__ X, float *__restrict__ h, int n, unsigned long long *trace)
{
    trace_start(trace);
    pdl_trigger();
    pdl_wait();
    trace_ready(trace);
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        h[i] = bf16_to_f(X[i]);
    trace_end(trace);
}

// Profiler: events around each launch (serialises the chain; eager steps only).
struct Prof {
    qad_model *m;
    cudaStream_t s;
    size_t next = 0;
    int begin(int kind)
    {
        if (!m->prof)
            return QAD_OK;
        if (next + 2 > m->prof_ev.size()) {
            for (int i = 0; i < 64; ++i) {
                cudaEvent_t e;
                int rc = cuda_check(cudaEventCreate(&e), "profiler event");
                if (rc)
                    return rc;
                m->prof_ev.push_back(e);
            }
        }
        if (m->prof_kind.size() < m->prof_ev.size() / 2)
            m->prof_kind.resize(m->prof_ev.size() / 2);
        m->prof_kind[next / 2] = kind;
        return cuda_check(cudaEventRecord(m->prof_ev[next++], s), "profiler record");
    }
    int end()
    {
        if (!m->prof)
            return QAD_OK;
        return cuda_check(cudaEventRecord(m->prof_ev[next++], s), "profiler record");
    }
};

static int copy_d2d(void *dst, const void *src, size_t n, cudaStream_t s)
{
    return cuda_check(cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToDevice, s), "debug copy");
}

static int run_step(qad_model *m, const uint16_t *X, int M, const int *ars, int n_agents, int max_rows,
                    const int *lens, float *h, char *ws, cudaStream_t s)
{
    const qad_model_desc &d = m->d;
    const int H = d.hidden, I = d.inter, hd = d.head_dim;
    const int nq = d.n_qh * hd, nkv = d.n_kvh * hd, nqkv = nq + 2 * nkv;
    const StepLayout L = step_layout(d, M);
    const int nt = frag_nt(M);
    float *qkv = (float *)(ws + L.qkv), *gu = (float *)(ws + L.gu);
    float *part = (float *)(ws + L.part);
    const AttnPlan plan = attn_plan(n_agents, d.n_qh, d.n_kvh, d.kv_cap, max_rows);
    const float scale = 1.0f / sqrtf((float)hd);
    const DbgLayout DL = dbg_layout(d, M);
    int rc;

    Prof P{m, s};
    if (m->prof && !m->prof_ev.empty() && m->prof_pending) {
        m->prof_pending = false;  // a previous profiled step was never read: drop it
    }
#define QAD_PROF(kind, launch_expr)                     \
    do {                                                \
        if ((rc = P.begin(kind)))                       \
            return rc;                                  \
        if ((rc = (launch_expr)))                       \
            return rc;                                  \
        if ((rc = P.end()))                             \
            return rc;                                  \
    } while (0)
    int slot = 0;
    auto tr = [&]() -> unsigned long long * {  // this launch's trace record, if tracing
        const int k = slot++;
        return m->trace && k < m->trace_n ? m->trace + 3 * (size_t)k : nullptr;
    };
    QAD_PROF(PK_INIT, (k_init_h<<<(M * H + 255) / 256, 256, 0, s>>>(X, h, M * H, tr()),
                       cuda_check(cudaGetLastError(), "init launch")));
    for (int l = 0; l < d.n_layers; ++l) {
        char *dbg = m->dbg ? (char *)m->dbg + (size_t)l * DL.per_layer : nullptr;
        PrepSrc src = {};
        // x1 = bf16(rmsnorm(h)) -> qkv
        FragBuf fb = frag_carve(ws + L.frag, H, nt);
        src.kind = PREP_RMSNORM;
        src.xf = h;
        src.ldx = H;
        src.eps = d.rms_eps;
        src.zero = qkv;
        src.zero_n = (long long)M * nqkv;
        src.dbg = dbg ? (uint16_t *)(dbg + DL.x1) : nullptr;
        src.ld_dbg = H;
        QAD_PROF(PK_PREP, launch_prep(4, H, M, src, fb, s, true, tr()));
        QAD_PROF(PK_GEMM_QKV, launch_gemm(4, m->mqkv[l], nqkv, H, M, fb, qkv, nqkv, s, true, tr()));
        if (dbg && (rc = copy_d2d(dbg + DL.qkv, qkv, (size_t)M * nqkv * 4, s)))
            return rc;
        // attention over each agent's cache; k, v of the new rows appended
        if (d.kv_format == QAD_KV_Q8_0) {
            const size_t so = kv_q8_scale_offset(d.max_agents, d.n_kvh, d.kv_cap);
            int8_t *Kq = (int8_t *)m->kc[l], *Vq = (int8_t *)m->vc[l];
            uint16_t *Kd = (uint16_t *)((char *)m->kc[l] + so), *Vd = (uint16_t *)((char *)m->vc[l] + so);
            QAD_PROF(PK_ATTN, launch_attn_q8_fused(plan, qkv, nqkv, Kq, Kd, Vq, Vd, lens, ars, n_agents, d.kv_cap,
                                                   d.n_qh, d.n_kvh, scale, part, s, true, tr()));
        } else {
            QAD_PROF(PK_ATTN, launch_attn_fused(plan, qkv, nqkv, m->kc[l], m->vc[l], lens, ars, n_agents, d.kv_cap,
                                                d.n_qh, d.n_kvh, scale, part, s, true, tr()));
        }
        // O = merged splits (bf16); h += O Wo^T
        fb = frag_carve(ws + L.frag, nq, nt);
        src = PrepSrc{};
        src.kind = PREP_ATTN;
        src.att = attn_part_view(plan, part, ars, lens, d.kv_cap, d.n_qh, d.n_kvh);
        src.n_agents = n_agents;
        src.dbg = dbg ? (uint16_t *)(dbg + DL.attn) : nullptr;
        src.ld_dbg = nq;
        QAD_PROF(PK_PREP, launch_prep(4, nq, M, src, fb, s, true, tr()));
        QAD_PROF(PK_GEMM_O, launch_gemm(4, m->mo[l], H, nq, M, fb, h, H, s, true, tr()));
        if (dbg && (rc = copy_d2d(dbg + DL.hmid, h, (size_t)M * H * 4, s)))
            return rc;
        // x2 = bf16(rmsnorm(h)) -> gate | up
        fb = frag_carve(ws + L.frag, H, nt);
        src = PrepSrc{};
        src.kind = PREP_RMSNORM;
        src.xf = h;
        src.ldx = H;
        src.eps = d.rms_eps;
        src.zero = gu;
        src.zero_n = (long long)M * 2 * I;
        src.dbg = dbg ? (uint16_t *)(dbg + DL.x2) : nullptr;
        src.ld_dbg = H;
        QAD_PROF(PK_PREP, launch_prep(4, H, M, src, fb, s, true, tr()));
        QAD_PROF(PK_GEMM_GU, launch_gemm(4, m->mgu[l], 2 * I, H, M, fb, gu, 2 * I, s, true, tr()));
        if (dbg && (rc = copy_d2d(dbg + DL.gu, gu, (size_t)M * 2 * I * 4, s)))
            return rc;
        // h += bf16(silu(gate) * up) Wdown^T
        fb = frag_carve(ws + L.frag, I, nt);
        src = PrepSrc{};
        src.kind = PREP_SILU;
        src.xf = gu;
        src.ldx = 2 * I;
        src.dbg = dbg ? (uint16_t *)(dbg + DL.act) : nullptr;
        src.ld_dbg = I;
        QAD_PROF(PK_PREP, launch_prep(6, I, M, src, fb, s, true, tr()));
        QAD_PROF(PK_GEMM_DOWN, launch_gemm(6, m->mdown[l], H, I, M, fb, h, H, s, true, tr()));
        if (dbg && (rc = copy_d2d(dbg + DL.hout, h, (size_t)M * H * 4, s)))
            return rc;
    }
#undef QAD_PROF
    if (m->prof) {
        m->prof_used = P.next;
        m->prof_pending = true;
    }
    return QAD_OK;
}

// ------------------------------------------------------------- mixed step: decode rows + one prompt chunk
//
// [OpenJet page], section 真正重要的是少互相堵车: a long prompt must not stall the
// other agents. A mixed step carries the decode batch (M rows, as above) and C
// prompt rows of one more agent, all R = M + C rows through the dense (tcgen05)
// GEMMs; the decode rows attend with the split-KV kernel, the chunk with the
// causal prefill kernel. Per layer: rmsnorm -> qkv -> attention (decode rows
// append their k, v; the chunk's k, v are appended first) -> o -> residual +
// rmsnorm -> gate|up -> silu*up -> down -> residual.

// h += Y (when Y is given), then X = bf16(h / sqrt(mean(h^2) + eps)); one CTA per row.
__global__ void __launch_bounds__(256) k_rows_rmsnorm(float *__restrict__ h, const float *__restrict__ Y,
                                                      uint16_t *__restrict__ X, int H, float eps)
{
    __shared__ float red[8];
    const int r = blockIdx.x, tid = threadIdx.x;
    float *hr = h + (size_t)r * H;
    float ss = 0.f;
    for (int i = 4 * tid; i < H; i += 1024) {
        float4 v = *reinterpret_cast<float4 *>(hr + i);
        if (Y) {
            const float4 y = *reinterpret_cast<const float4 *>(Y + (size_t)r * H + i);
            v.x += y.x, v.y += y.y, v.z += y.z, v.w += y.w;
            *reinterpret_cast<float4 *>(hr + i) = v;
        }
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((tid & 31) == 0)
        red[tid >> 5] = ss;
    __syncthreads();
    ss = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w)
        ss += red[w];
    const float inv = 1.f / sqrtf(ss / (float)H + eps);
    for (int i = 4 * tid; i < H; i += 1024) {
        const float4 v = *reinterpret_cast<const float4 *>(hr + i);
        *reinterpret_cast<uint2 *>(X + (size_t)r * H + i) =
            make_uint2(pack_bf162(v.x * inv, v.y * inv), pack_bf162(v.z * inv, v.w * inv));
    }
}

// act = bf16(silu(gate) * up) from gate|up fp32 [R][2I]; one CTA per row.
__global__ void __launch_bounds__(256) k_rows_silu(const float *__restrict__ gu, uint16_t *__restrict__ act, int I)
{
    const int r = blockIdx.x;
    const float *g = gu + (size_t)r * 2 * I, *u = g + I;
    for (int i = 2 * threadIdx.x; i < I; i += 512) {
        const float2 gv = *reinterpret_cast<const float2 *>(g + i), uv = *reinterpret_cast<const float2 *>(u + i);
        *reinterpret_cast<uint32_t *>(act + (size_t)r * I + i) = pack_bf162(silu_mul(gv.x, uv.x), silu_mul(gv.y, uv.y));
    }
}

// h += Y over n floats.
__global__ void k_rows_add(float *__restrict__ h, const float *__restrict__ Y, long long n)
{
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n / 4; i += (long long)gridDim.x * blockDim.x) {
        float4 v = reinterpret_cast<float4 *>(h)[i];
        const float4 y = reinterpret_cast<const float4 *>(Y)[i];
        v.x += y.x, v.y += y.y, v.z += y.z, v.w += y.w;
        reinterpret_cast<float4 *>(h)[i] = v;
    }
}

// Chunk row j (projection row M + j): Q = bf16(q) into Qc [C][nq]; k, v as bf16
// into the agent's caches (Kc, Vc point at its [n_kvh][cap][128] slice) at pos0 + j.
__global__ void __launch_bounds__(256) k_chunk_qkv(const float *__restrict__ qkv, int ldqkv, int M, int nq, int n_kvh,
                                                   uint16_t *__restrict__ Qc, uint16_t *__restrict__ Kc,
                                                   uint16_t *__restrict__ Vc, int cap, int pos0)
{
    const int j = blockIdx.x, nkv = n_kvh * 128;
    const float *row = qkv + (size_t)(M + j) * ldqkv;
    for (int i = 2 * threadIdx.x; i < nq; i += 512)
        *reinterpret_cast<uint32_t *>(Qc + (size_t)j * nq + i) = pack_bf162(row[i], row[i + 1]);
    for (int i = 2 * threadIdx.x; i < nkv; i += 512) {
        const int g = i >> 7, dd = i & 127;
        const size_t dst = ((size_t)g * cap + pos0 + j) * 128 + dd;
        *reinterpret_cast<uint32_t *>(Kc + dst) = pack_bf162(row[nq + i], row[nq + i + 1]);
        *reinterpret_cast<uint32_t *>(Vc + dst) = pack_bf162(row[nq + nkv + i], row[nq + nkv + i + 1]);
    }
}

struct MixedLayout {
    size_t x, qkv, y, qc, part, dense, total;
};

static MixedLayout mixed_layout(const qad_model_desc &d, int M, int C)
{
    MixedLayout L;
    const int R = M + C, nq = d.n_qh * d.head_dim, nqkv = (d.n_qh + 2 * d.n_kvh) * d.head_dim;
    const int xw = d.hidden > nq ? (d.hidden > d.inter ? d.hidden : d.inter) : (nq > d.inter ? nq : d.inter);
    const int yw = d.hidden > 2 * d.inter ? d.hidden : 2 * d.inter;
    size_t off = 0;
    L.x = off;  // bf16 activations: x1, attention output, x2, act (each dead after its GEMM's prep)
    off += a256((size_t)R * xw * 2);
    L.qkv = off;
    off += a256((size_t)R * nqkv * 4);
    L.y = off;  // fp32 GEMM outputs: o, gate|up, down
    off += a256((size_t)R * yw * 4);
    L.qc = off;
    off += a256((size_t)(C > 0 ? C : 1) * nq * 2);
    L.part = off;
    off += a256(M > 0 ? max_part_bytes(d, M) : 0);
    L.dense = off;
    size_t db = dense_ws_bytes(d.hidden, R);
    if (dense_ws_bytes(nq, R) > db)
        db = dense_ws_bytes(nq, R);
    if (dense_ws_bytes(d.inter, R) > db)
        db = dense_ws_bytes(d.inter, R);
    off += a256(db);
    L.total = off;
    return L;
}

static int run_mixed(qad_model *m, const uint16_t *X, int M, const int *ars, int n_agents, int max_rows,
                     const int *lens, int ca, int clen, int C, float *h, char *ws, cudaStream_t s)
{
    const qad_model_desc &d = m->d;
    const int H = d.hidden, I = d.inter, hd = d.head_dim, R = M + C;
    const int nq = d.n_qh * hd, nkv = d.n_kvh * hd, nqkv = nq + 2 * nkv;
    const MixedLayout L = mixed_layout(d, M, C);
    uint16_t *xb = (uint16_t *)(ws + L.x), *Qc = (uint16_t *)(ws + L.qc);
    float *qkv = (float *)(ws + L.qkv), *y = (float *)(ws + L.y), *part = (float *)(ws + L.part);
    void *dws = ws + L.dense;
    const float scale = 1.0f / sqrtf((float)hd);
    const DbgLayout DL = dbg_layout(d, R);
    int rc;
    auto ok = [](const char *what) { return cuda_check(cudaGetLastError(), what); };
    k_init_h<<<(R * H + 255) / 256, 256, 0, s>>>(X, h, R * H, nullptr);
    if ((rc = ok("init launch")))
        return rc;
    for (int l = 0; l < d.n_layers; ++l) {
        char *dbg = m->dbg ? (char *)m->dbg + (size_t)l * DL.per_layer : nullptr;
        k_rows_rmsnorm<<<R, 256, 0, s>>>(h, nullptr, xb, H, d.rms_eps);
        if ((rc = ok("rmsnorm launch")))
            return rc;
        if (dbg && (rc = copy_d2d(dbg + DL.x1, xb, (size_t)R * H * 2, s)))
            return rc;
        if ((rc = launch_dense(4, m->wqkv[l], nqkv, H, xb, R, qkv, dws, s)))
            return rc;
        if (dbg && (rc = copy_d2d(dbg + DL.qkv, qkv, (size_t)R * nqkv * 4, s)))
            return rc;
        if (M > 0) {  // decode rows: split-KV attention (appends their k, v), splits merged into O rows 0..M-1
            const AttnPlan plan = attn_plan(n_agents, d.n_qh, d.n_kvh, d.kv_cap, max_rows);
            if ((rc = launch_attn_fused(plan, qkv, nqkv, m->kc[l], m->vc[l], lens, ars, n_agents, d.kv_cap, d.n_qh,
                                        d.n_kvh, scale, part, s, false)))
                return rc;
            if ((rc = launch_attn_combine(plan, part, lens, ars, n_agents, d.kv_cap, d.n_qh, d.n_kvh, xb, s, false)))
                return rc;
        }
        if (C > 0) {  // the chunk: append its k, v, then causal attention into O rows M..R-1
            const size_t slice = (size_t)ca * d.n_kvh * d.kv_cap * hd;
            k_chunk_qkv<<<C, 256, 0, s>>>(qkv, nqkv, M, nq, d.n_kvh, Qc, m->kc[l] + slice, m->vc[l] + slice, d.kv_cap,
                                          clen);
            if ((rc = ok("chunk qkv launch")))
                return rc;
            if ((rc = launch_prefill_attn(Qc, m->kc[l] + slice, m->vc[l] + slice, clen, C, d.kv_cap, d.n_qh, d.n_kvh,
                                          scale, xb + (size_t)M * nq, s)))
                return rc;
        }
        if (dbg && (rc = copy_d2d(dbg + DL.attn, xb, (size_t)R * nq * 2, s)))
            return rc;
        if ((rc = launch_dense(4, m->wo[l], H, nq, xb, R, y, dws, s)))
            return rc;
        k_rows_rmsnorm<<<R, 256, 0, s>>>(h, y, xb, H, d.rms_eps);  // h += o; x2
        if ((rc = ok("rmsnorm launch")))
            return rc;
        if (dbg && (rc = copy_d2d(dbg + DL.hmid, h, (size_t)R * H * 4, s)))
            return rc;
        if (dbg && (rc = copy_d2d(dbg + DL.x2, xb, (size_t)R * H * 2, s)))
            return rc;
        if ((rc = launch_dense(4, m->wgu[l], 2 * I, H, xb, R, y, dws, s)))
            return rc;
        if (dbg && (rc = copy_d2d(dbg + DL.gu, y, (size_t)R * 2 * I * 4, s)))
            return rc;
        k_rows_silu<<<R, 256, 0, s>>>(y, xb, I);
        if ((rc = ok("silu launch")))
            return rc;
        if (dbg && (rc = copy_d2d(dbg + DL.act, xb, (size_t)R * I * 2, s)))
            return rc;
        if ((rc = launch_dense(6, m->wdown[l], H, I, xb, R, y, dws, s)))
            return rc;
        k_rows_add<<<(R * H / 4 + 255) / 256, 256, 0, s>>>(h, y, (long long)R * H);
        if ((rc = ok("residual launch")))
            return rc;
        if (dbg && (rc = copy_d2d(dbg + DL.hout, h, (size_t)R * H * 4, s)))
            return rc;
    }
    return QAD_OK;
}

static int check_step_args(const qad_model *m, const void *X, int M, const void *ars, int n_agents, int max_rows,
                           const void *lens, const void *H_out, const void *ws, size_t ws_bytes)
{
    if (!m || !X || !ars || !lens || !H_out || !ws || M <= 0 || n_agents <= 0 || max_rows <= 0)
        return fail(QAD_ERR_INVALID, "decode_step: null pointer or non-positive size");
    if (M > QAD_MAX_ROWS || n_agents > m->d.max_agents || max_rows > M)
        return fail(QAD_ERR_UNSUPPORTED, "decode_step: need M <= 16, n_agents <= %d, max_rows_per_agent <= M",
                    m->d.max_agents);
    if (max_rows * (m->d.n_qh / m->d.n_kvh) > 96)
        return fail(QAD_ERR_UNSUPPORTED, "decode_step: rows per agent x group exceeds 96");
    if ((uintptr_t)ws & 255)
        return fail(QAD_ERR_INVALID, "decode_step: workspace must be 256-byte aligned");
    if ((uintptr_t)H_out & 15)
        return fail(QAD_ERR_INVALID, "decode_step: H_out must be 16-byte aligned");
    if (ws_bytes < step_layout(m->d, M).total)
        return fail(QAD_ERR_WORKSPACE, "decode_step: workspace %zu < %zu bytes", ws_bytes, step_layout(m->d, M).total);
    return QAD_OK;
}

}  // namespace qad

extern "C" int qad_model_create(const qad_model_desc *desc, qad_model **out)
{
    if (!desc || !out)
        return qad::fail(QAD_ERR_INVALID, "qad_model_create: null argument");
    const qad_model_desc &d = *desc;
    if (d.n_layers <= 0 || d.hidden <= 0 || d.inter <= 0 || d.n_qh <= 0 || d.n_kvh <= 0 || d.max_agents <= 0 ||
        d.kv_cap <= 0 || !(d.rms_eps >= 0.f) || !d.w_qkv || !d.w_o || !d.w_gu || !d.w_down || !d.k_cache ||
        !d.v_cache)
        return qad::fail(QAD_ERR_INVALID, "qad_model_create: invalid descriptor");
    if (d.kv_format != QAD_KV_BF16 && d.kv_format != QAD_KV_Q8_0)
        return qad::fail(QAD_ERR_UNSUPPORTED, "qad_model_create: kv_format %d (need QAD_KV_BF16 or QAD_KV_Q8_0)",
                         d.kv_format);
    if (d.head_dim != 128 || d.n_qh % d.n_kvh || d.hidden % 256 || d.inter % 256 || (d.n_qh * d.head_dim) % 256 ||
        d.hidden > 65536 || d.inter > 65536)
        return qad::fail(QAD_ERR_UNSUPPORTED,
                         "qad_model_create: need head_dim 128, n_qh %% n_kvh == 0, hidden/inter/n_qh*hd multiples "
                         "of 256 and <= 65536");
    qad_model *m = new qad_model();
    m->d = d;
    for (int l = 0; l < d.n_layers; ++l) {
        if (!d.w_qkv[l] || !d.w_o[l] || !d.w_gu[l] || !d.w_down[l] || !d.k_cache[l] || !d.v_cache[l] ||
            (((uintptr_t)d.w_qkv[l] | (uintptr_t)d.w_o[l] | (uintptr_t)d.w_gu[l] | (uintptr_t)d.w_down[l] |
              (uintptr_t)d.k_cache[l] | (uintptr_t)d.v_cache[l]) & 15)) {
            delete m;
            return qad::fail(QAD_ERR_INVALID, "qad_model_create: null or misaligned pointer in layer %d", l);
        }
        qad::WeightMapsBlob mb[4];
        const int nqkv = (d.n_qh + 2 * d.n_kvh) * d.head_dim, nq = d.n_qh * d.head_dim;
        int rc = qad::make_weight_maps(4, d.w_qkv[l], nqkv, d.hidden, &mb[0]);
        if (!rc)
            rc = qad::make_weight_maps(4, d.w_o[l], d.hidden, nq, &mb[1]);
        if (!rc)
            rc = qad::make_weight_maps(4, d.w_gu[l], 2 * d.inter, d.hidden, &mb[2]);
        if (!rc)
            rc = qad::make_weight_maps(6, d.w_down[l], d.hidden, d.inter, &mb[3]);
        if (rc) {
            delete m;
            return rc;
        }
        m->mqkv.push_back(mb[0]);
        m->mo.push_back(mb[1]);
        m->mgu.push_back(mb[2]);
        m->mdown.push_back(mb[3]);
        m->wqkv.push_back(d.w_qkv[l]);
        m->wo.push_back(d.w_o[l]);
        m->wgu.push_back(d.w_gu[l]);
        m->wdown.push_back(d.w_down[l]);
        m->kc.push_back(d.k_cache[l]);
        m->vc.push_back(d.v_cache[l]);
    }
    m->d.w_qkv = m->wqkv.data();
    m->d.w_o = m->wo.data();
    m->d.w_gu = m->wgu.data();
    m->d.w_down = m->wdown.data();
    m->d.k_cache = m->kc.data();
    m->d.v_cache = m->vc.data();
    *out = m;
    return QAD_OK;
}

extern "C" void qad_model_destroy(qad_model *m)
{
    if (!m)
        return;
    qad_step_graph_destroy(m->hg);
    for (cudaEvent_t e : m->prof_ev)
        cudaEventDestroy(e);
    delete m;
}

extern "C" size_t qad_decode_step_ws_bytes(const qad_model *m, int M)
{
    if (!m || M <= 0 || M > QAD_MAX_ROWS)
        return 0;
    return qad::step_layout(m->d, M).total;
}

extern "C" size_t qad_decode_step_debug_bytes(const qad_model *m, int M)
{
    if (!m || M <= 0 || M > QAD_MAX_ROWS)
        return 0;
    return qad::dbg_layout(m->d, M).per_layer * m->d.n_layers;
}

extern "C" int qad_model_set_debug(qad_model *m, void *dbg, size_t bytes)
{
    if (!m)
        return qad::fail(QAD_ERR_INVALID, "qad_model_set_debug: null model");
    if ((uintptr_t)dbg & 255)
        return qad::fail(QAD_ERR_INVALID, "qad_model_set_debug: buffer must be 256-byte aligned");
    m->dbg = dbg;
    m->dbg_bytes = bytes;
    return QAD_OK;
}

extern "C" int qad_model_set_trace(qad_model *m, unsigned long long *buf, int n_records)
{
    if (!m || n_records < 0 || (buf && n_records == 0))
        return qad::fail(QAD_ERR_INVALID, "qad_model_set_trace: null model or bad record count");
    if ((uintptr_t)buf & 7)
        return qad::fail(QAD_ERR_INVALID, "qad_model_set_trace: buffer must be 8-byte aligned");
    m->trace = buf;
    m->trace_n = buf ? n_records : 0;
    return QAD_OK;
}

extern "C" int qad_decode_step(qad_model *m, const uint16_t *X, int M, const int *agent_row_start, int n_agents,
                               int max_rows_per_agent, const int *lens, float *H_out, void *ws, size_t ws_bytes,
                               void *stream)
{
    int rc = qad::check_step_args(m, X, M, agent_row_start, n_agents, max_rows_per_agent, lens, H_out, ws, ws_bytes);
    if (rc)
        return rc;
    if (m->dbg && m->dbg_bytes < qad_decode_step_debug_bytes(m, M))
        return qad::fail(QAD_ERR_WORKSPACE, "decode_step: debug buffer too small");
    return qad::run_step(m, X, M, agent_row_start, n_agents, max_rows_per_agent, lens, H_out, (char *)ws,
                         (cudaStream_t)stream);
}

extern "C" size_t qad_mixed_step_ws_bytes(const qad_model *m, int M, int C)
{
    if (!m || M < 0 || C < 0 || M + C <= 0 || M > QAD_MAX_ROWS)
        return 0;
    return qad::mixed_layout(m->d, M, C).total;
}

extern "C" size_t qad_mixed_step_debug_bytes(const qad_model *m, int M, int C)
{
    if (!m || M < 0 || C < 0 || M + C <= 0 || M > QAD_MAX_ROWS)
        return 0;
    return qad::dbg_layout(m->d, M + C).per_layer * m->d.n_layers;
}

extern "C" int qad_mixed_step(qad_model *m, const uint16_t *X, int M, const int *agent_row_start, int n_agents,
                              int max_rows_per_agent, const int *lens, int chunk_agent, int chunk_len, int C,
                              float *H_out, void *ws, size_t ws_bytes, void *stream)
{
    if (!m || !X || !H_out || !ws || M < 0 || C < 0 || M + C <= 0)
        return qad::fail(QAD_ERR_INVALID, "qad_mixed_step: null pointer or empty step");
    if (M > 0) {
        int rc = qad::check_step_args(m, X, M, agent_row_start, n_agents, max_rows_per_agent, lens, H_out, ws,
                                      ws_bytes);
        if (rc)
            return rc;
    }
    if (m->d.kv_format != QAD_KV_BF16)
        return qad::fail(QAD_ERR_UNSUPPORTED, "qad_mixed_step: the prompt chunk needs bf16 KV caches");
    if (C > 0 && (chunk_agent < 0 || chunk_agent >= m->d.max_agents || chunk_len < 0 ||
                  (long long)chunk_len + C > m->d.kv_cap))
        return qad::fail(QAD_ERR_INVALID, "qad_mixed_step: chunk agent %d or positions %d..%lld outside the cache",
                         chunk_agent, chunk_len, (long long)chunk_len + C - 1);
    if ((uintptr_t)ws & 255 || (uintptr_t)H_out & 15 || (uintptr_t)X & 15)
        return qad::fail(QAD_ERR_INVALID, "qad_mixed_step: ws 256-byte, X and H_out 16-byte aligned");
    if (ws_bytes < qad::mixed_layout(m->d, M, C).total)
        return qad::fail(QAD_ERR_WORKSPACE, "qad_mixed_step: workspace %zu < %zu bytes", ws_bytes,
                         qad::mixed_layout(m->d, M, C).total);
    if (m->dbg && m->dbg_bytes < qad_mixed_step_debug_bytes(m, M, C))
        return qad::fail(QAD_ERR_WORKSPACE, "qad_mixed_step: debug buffer too small");
    return qad::run_mixed(m, X, M, agent_row_start, n_agents, max_rows_per_agent, lens, chunk_agent, chunk_len, C,
                          H_out, (char *)ws, (cudaStream_t)stream);
}

extern "C" int qad_decode_step_launches(const qad_model *m)
{
    if (!m)
        return 0;
    return 1 + 9 * m->d.n_layers;
}

extern "C" int qad_step_graph_create(qad_model *m, const uint16_t *X, int M, const int *agent_row_start, int n_agents,
                                     int max_rows_per_agent, const int *lens, float *H_out, void *ws, size_t ws_bytes,
                                     void *stream, qad_step_graph **out)
{
    if (!out)
        return qad::fail(QAD_ERR_INVALID, "qad_step_graph_create: null output");
    int rc = qad::check_step_args(m, X, M, agent_row_start, n_agents, max_rows_per_agent, lens, H_out, ws, ws_bytes);
    if (rc)
        return rc;
    if (m->dbg || m->prof)
        return qad::fail(QAD_ERR_UNSUPPORTED,
                         "qad_step_graph_create: a model with a debug buffer or the profiler on is not captured");
    cudaStream_t s = (cudaStream_t)stream;
    if (!s)
        return qad::fail(QAD_ERR_INVALID, "qad_step_graph_create: needs a non-default stream");
    if ((rc = qad::cuda_check(cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal), "begin capture")))
        return rc;
    rc = qad::run_step(m, X, M, agent_row_start, n_agents, max_rows_per_agent, lens, H_out, (char *)ws, s);
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamEndCapture(s, &graph);
    if (rc) {
        if (graph)
            cudaGraphDestroy(graph);
        return rc;
    }
    if ((rc = qad::cuda_check(e, "end capture")))
        return rc;
    qad_step_graph *g = new qad_step_graph();
    g->graph = graph;
    if ((rc = qad::cuda_check(cudaGraphInstantiate(&g->exec, graph, 0), "graph instantiate"))) {
        cudaGraphDestroy(graph);
        delete g;
        return rc;
    }
    *out = g;
    return QAD_OK;
}

extern "C" int qad_step_graph_launch(qad_step_graph *g, void *stream)
{
    if (!g || !g->exec)
        return qad::fail(QAD_ERR_INVALID, "qad_step_graph_launch: null graph");
    return qad::cuda_check(cudaGraphLaunch(g->exec, (cudaStream_t)stream), "graph launch");
}

extern "C" void qad_step_graph_destroy(qad_step_graph *g)
{
    if (!g)
        return;
    if (g->exec)
        cudaGraphExecDestroy(g->exec);
    if (g->graph)
        cudaGraphDestroy(g->graph);
    delete g;
}

extern "C" int qad_decode_step_host(qad_model *m, const uint16_t *X_host, int M, const int *agent_row_start_host,
                                    int n_agents, int max_rows_per_agent, const int *lens_host, float *H_out_host,
                                    void *ws, size_t ws_bytes, void *stream)
{
    if (!X_host || !agent_row_start_host || !lens_host || !H_out_host)
        return qad::fail(QAD_ERR_INVALID, "qad_decode_step_host: null host pointer");
    int rc = qad::check_step_args(m, X_host, M, agent_row_start_host, n_agents, max_rows_per_agent, lens_host,
                                  H_out_host, ws, ws_bytes);
    if (rc)
        return rc;
    for (int a = 0; a < n_agents; ++a)
        if (agent_row_start_host[a] > agent_row_start_host[a + 1] || lens_host[a] < 0 ||
            lens_host[a] + (agent_row_start_host[a + 1] - agent_row_start_host[a]) > m->d.kv_cap)
            return qad::fail(QAD_ERR_INVALID, "qad_decode_step_host: agent %d rows/len out of range", a);
    if (agent_row_start_host[0] != 0 || agent_row_start_host[n_agents] != M)
        return qad::fail(QAD_ERR_INVALID, "qad_decode_step_host: agent_row_start must span 0..M");
    cudaStream_t s = (cudaStream_t)stream;
    const qad::StepLayout L = qad::step_layout(m->d, M);
    char *w = (char *)ws;
    uint16_t *X = (uint16_t *)(w + L.x_in);
    int *ars = (int *)(w + L.ars_in), *lens = (int *)(w + L.lens_in);
    float *H = (float *)(w + L.h_out);
    if ((rc = qad::cuda_check(cudaMemcpyAsync(X, X_host, (size_t)M * m->d.hidden * 2, cudaMemcpyHostToDevice, s),
                              "H2D X")) ||
        (rc = qad::cuda_check(cudaMemcpyAsync(ars, agent_row_start_host, (size_t)(n_agents + 1) * 4,
                                              cudaMemcpyHostToDevice, s),
                              "H2D agent_row_start")) ||
        (rc = qad::cuda_check(cudaMemcpyAsync(lens, lens_host, (size_t)n_agents * 4, cudaMemcpyHostToDevice, s),
                              "H2D lens")))
        return rc;
    if (s && !m->dbg && !m->prof) {
        if (!m->hg || m->hg_M != M || m->hg_agents != n_agents || m->hg_rows != max_rows_per_agent || m->hg_ws != ws ||
            m->hg_stream != s) {
            qad_step_graph_destroy(m->hg);
            m->hg = nullptr;
            if ((rc = qad_step_graph_create(m, X, M, ars, n_agents, max_rows_per_agent, lens, H, ws, ws_bytes, stream,
                                            &m->hg)))
                return rc;
            m->hg_M = M;
            m->hg_agents = n_agents;
            m->hg_rows = max_rows_per_agent;
            m->hg_ws = ws;
            m->hg_stream = s;
        }
        if ((rc = qad_step_graph_launch(m->hg, stream)))
            return rc;
    } else if ((rc = qad::run_step(m, X, M, ars, n_agents, max_rows_per_agent, lens, H, w, s))) {
        return rc;
    }
    if ((rc = qad::cuda_check(cudaMemcpyAsync(H_out_host, H, (size_t)M * m->d.hidden * 4, cudaMemcpyDeviceToHost, s),
                              "D2H H")))
        return rc;
    return qad::cuda_check(cudaStreamSynchronize(s), "step sync");
}

extern "C" int qad_model_set_profile(qad_model *m, int enable)
{
    if (!m)
        return qad::fail(QAD_ERR_INVALID, "qad_model_set_profile: null model");
    m->prof = enable != 0;
    for (int k = 0; k < PK_COUNT; ++k) {
        m->prof_ms[k] = 0;
        m->prof_n[k] = 0;
    }
    m->prof_pending = false;
    return QAD_OK;
}

extern "C" int qad_model_profile_read(qad_model *m, double *ms, long long *count, int n_kinds)
{
    if (!m || !ms || !count || n_kinds < PK_COUNT)
        return qad::fail(QAD_ERR_INVALID, "qad_model_profile_read: invalid arguments");
    if (m->prof_pending) {
        int rc = qad::cuda_check(cudaEventSynchronize(m->prof_ev[m->prof_used - 1]), "profiler sync");
        if (rc)
            return rc;
        for (size_t i = 0; i + 1 < m->prof_used; i += 2) {
            float t = 0.f;
            rc = qad::cuda_check(cudaEventElapsedTime(&t, m->prof_ev[i], m->prof_ev[i + 1]), "profiler elapsed");
            if (rc)
                return rc;
            m->prof_ms[m->prof_kind[i / 2]] += t;
            m->prof_n[m->prof_kind[i / 2]] += 1;
        }
        m->prof_pending = false;
    }
    for (int k = 0; k < PK_COUNT; ++k) {
        ms[k] = m->prof_ms[k];
        count[k] = m->prof_n[k];
    }
    return PK_COUNT;
}
