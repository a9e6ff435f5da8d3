// gemm.cuh -- skinny quantized GEMM (M <= 16) launch interface shared by the
// standalone C-ABI entry points and the decode-step driver.
#pragma once
#include "attn.cuh"

namespace qad {

enum PrepKind { PREP_BF16 = 0, PREP_RMSNORM = 1, PREP_SILU = 2, PREP_ATTN = 3 };

// Activation operand of one GEMM input of K columns: one record of REC_BYTES per
// 256-wide block b, 16 activation rows (rows >= M zero), in the tensor core's
// K-major no-swizzle layout (core matrices of 8 rows x 8 fp16):
//   X  [k chunk 32][row 16][8 fp16]  fp16 of x * 2^e(r,b); MMA position 4t + {0,1,2,3}
//                                    holds block column 4t + {0,2,1,3}
//   S  [2][row 16][8 fp16]           Q4_K sub-block sums of those fp16 values split
//                                    into a high part (first 8) and a low part
//   RS [16] float                    2^-e(r,b) per row (0 for rows >= M)
struct FragBuf {
    uint8_t *rec;
};

constexpr int REC_BYTES = 8192 + 512 + 64;
constexpr int REC_S_OFF = 8192;
constexpr int REC_RS_OFF = 8704;
size_t frag_bytes(int K, int nt = 2);  // records of a K-column input (either format)
int frag_nt(int M);                    // kept for callers: the record always has 16 rows
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
// The prep runs one 256-thread CTA per (row < 16, group of 4 blocks); the GEMM
// runs one CTA per SM.
// trace: optional 3-word launch record (see trace_start in common.cuh), or nullptr.
int launch_prep(int fmt, int K, int M, const PrepSrc &src, const FragBuf &fb, cudaStream_t s, bool pdl,
                unsigned long long *trace = nullptr);
int launch_gemm(int fmt, const WeightMapsBlob &maps, int N, int K, int M, const FragBuf &fb, float *Y, int ldy,
                cudaStream_t s, bool pdl, unsigned long long *trace = nullptr);
size_t q6k_packed_bytes(long long N, int K);
int launch_q6k_pack(const void *W, int N, int K, void *P, cudaStream_t s);

}  // namespace qad
