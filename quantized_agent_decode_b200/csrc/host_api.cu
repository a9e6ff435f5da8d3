// host_api.cu -- error state, device queries and the host-only row packer.
#include <cuda.h>

#include <cstring>
#include <mutex>

#include "common.cuh"

namespace qad {

static thread_local char g_err[512] = "";

void set_error(const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}

int fail(int code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return code;
}

int cuda_check(cudaError_t e, const char *what)
{
    if (e == cudaSuccess)
        return QAD_OK;
    return fail(QAD_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn();

int encode_tmap_kmajor_bf16(void *map, const void *base, uint64_t rows, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return fail(QAD_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    // [rows][128] bf16 viewed as (8 values, row, 16-value chunk): a box lands as
    // [chunk][row][8 values], the K-major no-swizzle core-matrix layout
    const cuuint64_t dims[3] = {8, rows, 16};
    const cuuint64_t strides[2] = {256, 16};
    const cuuint32_t box[3] = {8, box_rows, 16};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(reinterpret_cast<CUtensorMap *>(map), CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void *>(base),
                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(QAD_ERR_CUDA, "cuTensorMapEncodeTiled (3-D chunk view) failed (%d): rows %llu box %u", (int)r,
                    (unsigned long long)rows, box_rows);
    return QAD_OK;
}

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

int encode_tmap_2d(void *map, const void *base, int elem_bytes, uint64_t cols, uint64_t rows, uint64_t row_stride_bytes,
                   uint32_t box_cols, uint32_t box_rows)
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    if (!fn)
        return fail(QAD_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(reinterpret_cast<CUtensorMap *>(map),
                    elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                    const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(QAD_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d): cols %llu rows %llu stride %llu box %u x %u",
                    (int)r, (unsigned long long)cols, (unsigned long long)rows, (unsigned long long)row_stride_bytes,
                    box_cols, box_rows);
    return QAD_OK;
}

}  // namespace qad

extern "C" const char *qad_last_error(void) { return qad::g_err; }

extern "C" int qad_version(void) { return 100; }

// Row packer ([OpenJet page], section 只搬一次权重): stack each active agent's
// next-token and draft rows agent-major into one batch. Pure host code.
extern "C" int qad_pack_rows(const qad_agent_rows *agents, int n_agents, int hidden, int max_rows,
                             uint16_t *X, int *row_agent, int *row_pos, int *agent_row_start)
{
    if (n_agents < 0 || hidden <= 0 || max_rows < 0 || (n_agents > 0 && !agents) || !agent_row_start)
        return qad::fail(QAD_ERR_INVALID, "qad_pack_rows: invalid arguments");
    int total = 0;
    for (int a = 0; a < n_agents; ++a) {
        if (agents[a].n_rows < 0 || agents[a].len < 0)
            return qad::fail(QAD_ERR_INVALID, "qad_pack_rows: agent %d has n_rows %d len %d", a,
                             agents[a].n_rows, agents[a].len);
        if (agents[a].n_rows > 0 && !agents[a].rows)
            return qad::fail(QAD_ERR_INVALID, "qad_pack_rows: agent %d rows is null", a);
        total += agents[a].n_rows;
    }
    if (total > max_rows)
        return qad::fail(QAD_ERR_UNSUPPORTED, "qad_pack_rows: %d rows exceed capacity %d", total, max_rows);
    if (total > 0 && (!X || !row_agent || !row_pos))
        return qad::fail(QAD_ERR_INVALID, "qad_pack_rows: null output");
    int r = 0;
    for (int a = 0; a < n_agents; ++a) {
        agent_row_start[a] = r;
        for (int j = 0; j < agents[a].n_rows; ++j, ++r) {
            std::memcpy(X + (size_t)r * hidden, agents[a].rows + (size_t)j * hidden, sizeof(uint16_t) * hidden);
            row_agent[r] = a;
            row_pos[r] = agents[a].len + j;
        }
    }
    agent_row_start[n_agents] = r;
    return r;
}
