// gemm.cuh -- skinny quantized GEMM (M <= 16) launch interface shared by the
// standalone C-ABI entry points and the decode-step driver.
#pragma once
#include "attn.cuh"

namespace qad {

enum PrepKind { PREP_BF16 = 0, PREP_RMSNORM = 1, PREP_SILU = 2, PREP_ATTN = 3 };

// Activation operand of one GEMM input of K columns: one record per 256-wide
// block b, record size rec_bytes(fmt, nt):
//   X  [s 16][g 8][c 4][nt][2 words]  fp16 B fragments of x * 2^e(r,b)
//   S  [g 8][c 4][nt][2 words]        Q4_K sub-block sums (Q4_K only)
//   RS [16] float                     2^-e(r,b) per row (0 for rows >= M)
struct FragBuf {
    uint8_t *rec;
};

constexpr int rec_bytes(int fmt, int nt) { return 4096 * nt + (fmt == 4 ? 256 * nt : 0) + 64; }
size_t frag_bytes(int K, int nt);  // room for either format
int frag_nt(int M);                // fragment layout used for M rows
FragBuf frag_carve(void *ws, int K, int nt);

struct PrepSrc {
    int kind;            // PrepKind
    const uint16_t *xb;  // PREP_BF16: bf16 [M][ldx]
    const float *xf;     // PREP_RMSNORM: fp32 h [M][ldx]; PREP_SILU: fp32 [M][ldx] gate | up
    int ldx;
    float eps;
    AttnPartView att;    // PREP_ATTN: attention partials to merge (row r, column head*128 + d)
    int n_agents;        // PREP_ATTN
    float *zero;         // optional buffer zeroed by the prep (the next GEMM's output)
    long long zero_n;
    uint16_t *dbg;       // optional bf16 copy of the rows actually fed to the GEMM
    int ld_dbg;
};

// Tensor maps (TMA descriptors) of one quantized matrix, opaque outside gemm.cu.
struct alignas(64) WeightMapsBlob {
    unsigned char bytes[256];
};

// fmt: 4 = Q4_K (GGUF blocks), 6 = Q6_K-like in the packed layout of qad_q6k_pack.
int make_weight_maps(int fmt, const void *W, int N, int K, WeightMapsBlob *out);
// The prep runs one 256-thread CTA per (row < 8*nt, group of 4 blocks); the
// GEMM runs one CTA per SM.
// trace: optional 3-word launch record (see trace_start in common.cuh), or nullptr.
int launch_prep(int fmt, int K, int M, const PrepSrc &src, const FragBuf &fb, cudaStream_t s, bool pdl,
                unsigned long long *trace = nullptr);
int launch_gemm(int fmt, const WeightMapsBlob &maps, int N, int K, int M, const FragBuf &fb, float *Y, int ldy,
                cudaStream_t s, bool pdl, unsigned long long *trace = nullptr);
size_t q6k_packed_bytes(long long N, int K);
int launch_q6k_pack(const void *W, int N, int K, void *P, cudaStream_t s);

}  // namespace qad
