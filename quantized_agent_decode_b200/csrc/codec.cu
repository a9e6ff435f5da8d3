// codec.cu -- Q4_K / Q6_K-like block unpack kernels (diagnostics and the
// bit-exact codec parity tests). The GEMM kernels decode blocks in registers
// with the same field layout; these kernels expose the decoded fields.
//
// Q4_K super-block (the Q4_K_M weights of the OpenJet multi-agent page,
// intro; layout per the GGUF Q4_K convention): [0:2] d, [2:4] dmin (fp16),
// [4:16] twelve bytes holding eight 6-bit scales and eight 6-bit mins,
// [16:144] 128 bytes of 4-bit quants (byte 32p+l: low nibble = weight 64p+l,
// high nibble = weight 64p+32+l).
// Q6_K-like block: [0:128] low 4 bits, [128:192] high 2 bits, [192:208] int8
// scales of the 16 sub-blocks of 16, [208:210] d (fp16).
#include "common.cuh"

namespace qad {

// One warp per block; lane l handles quant bytes l, l+32, l+64, l+96.
__global__ void k_q4k_unpack(const uint8_t *__restrict__ W, long long nb, uint8_t *q, uint8_t *sc, uint8_t *m,
                             uint16_t *d, uint16_t *dmin)
{
    long long blk = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    int lane = threadIdx.x & 31;
    if (blk >= nb)
        return;
    const uint8_t *b = W + blk * 144;
    for (int p = 0; p < 4; ++p) {
        uint8_t v = b[16 + 32 * p + lane];
        q[blk * 256 + 64 * p + lane] = v & 15;
        q[blk * 256 + 64 * p + 32 + lane] = v >> 4;
    }
    if (lane < 8) {
        const uint8_t *s = b + 4;
        int j = lane;
        uint8_t scv, mv;
        if (j < 4) {
            scv = s[j] & 63;
            mv = s[j + 4] & 63;
        } else {
            scv = (uint8_t)((s[j + 4] & 15) | ((s[j - 4] >> 6) << 4));
            mv = (uint8_t)((s[j + 4] >> 4) | ((s[j] >> 6) << 4));
        }
        sc[blk * 8 + j] = scv;
        m[blk * 8 + j] = mv;
    }
    if (lane == 0) {
        d[blk] = (uint16_t)(b[0] | b[1] << 8);
        dmin[blk] = (uint16_t)(b[2] | b[3] << 8);
    }
}

__global__ void k_q6k_unpack(const uint8_t *__restrict__ W, long long nb, uint8_t *q, int8_t *sc, uint16_t *d)
{
    long long blk = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    int l = threadIdx.x & 31;
    if (blk >= nb)
        return;
    const uint8_t *b = W + blk * 210;
    for (int h = 0; h < 2; ++h) {
        const uint8_t *L = b + 64 * h, *H = b + 128 + 32 * h;
        uint8_t hv = H[l];
        uint8_t *qq = q + blk * 256 + 128 * h;
        qq[l] = (uint8_t)((L[l] & 15) | ((hv & 3) << 4));
        qq[l + 32] = (uint8_t)((L[l + 32] & 15) | (((hv >> 2) & 3) << 4));
        qq[l + 64] = (uint8_t)((L[l] >> 4) | (((hv >> 4) & 3) << 4));
        qq[l + 96] = (uint8_t)((L[l + 32] >> 4) | (((hv >> 6) & 3) << 4));
    }
    if (l < 16)
        sc[blk * 16 + l] = (int8_t)b[192 + l];
    if (l == 0)
        d[blk] = (uint16_t)(b[208] | b[209] << 8);
}

}  // namespace qad

extern "C" int qad_q4k_unpack(const void *W, long long n_blocks, uint8_t *q, uint8_t *sc, uint8_t *m, uint16_t *d,
                              uint16_t *dmin, void *stream)
{
    if (n_blocks < 0 || (n_blocks > 0 && (!W || !q || !sc || !m || !d || !dmin)))
        return qad::fail(QAD_ERR_INVALID, "qad_q4k_unpack: invalid arguments");
    if (n_blocks == 0)
        return QAD_OK;
    long long grid = (n_blocks + 7) / 8;
    if (grid > 0x7fffffffLL)
        return qad::fail(QAD_ERR_UNSUPPORTED, "qad_q4k_unpack: too many blocks");
    qad::k_q4k_unpack<<<(unsigned)grid, 256, 0, (cudaStream_t)stream>>>((const uint8_t *)W, n_blocks, q, sc, m, d,
                                                                         dmin);
    return qad::cuda_check(cudaGetLastError(), "qad_q4k_unpack launch");
}

extern "C" int qad_q6k_unpack(const void *W, long long n_blocks, uint8_t *q, int8_t *sc, uint16_t *d, void *stream)
{
    if (n_blocks < 0 || (n_blocks > 0 && (!W || !q || !sc || !d)))
        return qad::fail(QAD_ERR_INVALID, "qad_q6k_unpack: invalid arguments");
    if (n_blocks == 0)
        return QAD_OK;
    long long grid = (n_blocks + 7) / 8;
    if (grid > 0x7fffffffLL)
        return qad::fail(QAD_ERR_UNSUPPORTED, "qad_q6k_unpack: too many blocks");
    qad::k_q6k_unpack<<<(unsigned)grid, 256, 0, (cudaStream_t)stream>>>((const uint8_t *)W, n_blocks, q, sc, d);
    return qad::cuda_check(cudaGetLastError(), "qad_q6k_unpack launch");
}
