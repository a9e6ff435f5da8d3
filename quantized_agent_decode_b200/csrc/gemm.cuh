// gemm.cuh -- skinny quantized GEMM (M <= 16) launch interface shared by the
// standalone C-ABI entry points and the decode-step driver.
#pragma once
#include "common.cuh"

namespace qad {

enum PrepKind { PREP_BF16 = 0, PREP_RMSNORM = 1, PREP_SILU = 2 };

// Activation-fragment workspace for one GEMM input of K columns.
struct FragBuf {
    uint32_t *xp;  // x fragments
    uint32_t *sp;  // sub-block sums (Q4_K only)
    float *rs;     // per-row output scale (16 floats)
};

size_t frag_bytes(int K, int nt);
int frag_nt(int M);  // fragment layout used for M rows by the active GEMM backend
FragBuf frag_carve(void *ws, int K, int nt);

struct PrepSrc {
    int kind;            // PrepKind
    const uint16_t *xb;  // PREP_BF16: bf16 [M][ldx]
    const float *xf;     // PREP_RMSNORM: fp32 h [M][ldx]; PREP_SILU: fp32 [M][ldx] gate | up
    int ldx;
    float eps;
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
// Launch the prep (8 or 16 CTAs) then the GEMM (one CTA per SM).
int launch_prep(int fmt, int K, int M, const PrepSrc &src, const FragBuf &fb, cudaStream_t s, bool pdl);
int launch_gemm(int fmt, const WeightMapsBlob &maps, int N, int K, int M, const FragBuf &fb, float *Y, int ldy,
                cudaStream_t s, bool pdl);
size_t q6k_packed_bytes(long long N, int K);
int launch_q6k_pack(const void *W, int N, int K, void *P, cudaStream_t s);

}  // namespace qad
