// attn.cuh -- split-KV grouped-query decode attention launch interface.
#pragma once
#include "common.cuh"

namespace qad {

// Partial results of one (agent, kv-head, row group of 24 query vectors, key
// split): unnormalised O [24][128] fp32, then the running max m[24] (log2
// domain) and the sum l[24]. Record index
// ((agent * n_kvh + kv_head) * n_rg + rg) * max_splits + split.
constexpr int ATT_QG = 24;
constexpr int ATT_PART_FLOATS = ATT_QG * 128 + 2 * ATT_QG;

// What a consumer needs to merge the splits of one query vector.
struct AttnPartView {
    const float *part;
    const int *ars, *lens;
    int n_kvh, G, n_rg, max_splits, CH, kv_cap, n_qh;
};

struct AttnPlan {
    int G;           // q-heads per kv-head
    int n_rg;        // groups of 24 query vectors per (agent, kv-head)
    int CH;          // keys per split (multiple of 64)
    int max_splits;  // splits covering kv_cap keys
    int stages;      // per-warp cp.async ring depth of the kernel variant
    size_t part_bytes;
};

AttnPlan attn_plan(int n_agents, int n_qh, int n_kvh, int kv_cap, int max_rows_per_agent);
// Standalone form: Q bf16, caches already holding the new rows, O bf16 (combine included).
int launch_attn(const AttnPlan &pl, const uint16_t *Q, const uint16_t *Kc, const uint16_t *Vc, const int *lens,
                const int *ars, int n_agents, int kv_cap, int n_qh, int n_kvh, float scale, uint16_t *O, float *part,
                cudaStream_t s, bool pdl);
// Fused form used by the decode step: Q and the new rows' k, v are read from the
// fp32 q|k|v projection [M][ldqkv]; the split holding each new position also
// writes that row's k, v (bf16) into the caches. Writes only the partials
// (the o-projection prep merges them).
int launch_attn_fused(const AttnPlan &pl, const float *qkv, int ldqkv, uint16_t *Kc, uint16_t *Vc, const int *lens,
                      const int *ars, int n_agents, int kv_cap, int n_qh, int n_kvh, float scale, float *part,
                      cudaStream_t s, bool pdl, unsigned long long *trace = nullptr);
// Combine the splits of a standalone launch into bf16 O [M][n_qh][128].
int launch_attn_combine(const AttnPlan &pl, const float *part, const int *lens, const int *ars, int n_agents,
                        int kv_cap, int n_qh, int n_kvh, uint16_t *O, cudaStream_t s, bool pdl);
// q8_0 cache: int8 codes [A][n_kvh][kv_cap][128] and fp16 scales [A][n_kvh][kv_cap][4]
// (one per 32 values) for K and for V. Same plan and partial records as the bf16 form.
int launch_attn_q8_fused(const AttnPlan &pl, const float *qkv, int ldqkv, int8_t *Kq, uint16_t *Kd, int8_t *Vq,
                         uint16_t *Vd, const int *lens, const int *ars, int n_agents, int kv_cap, int n_qh, int n_kvh,
                         float scale, float *part, cudaStream_t s, bool pdl, unsigned long long *trace = nullptr);
int launch_attn_q8(const AttnPlan &pl, const uint16_t *Q, const int8_t *Kq, const uint16_t *Kd, const int8_t *Vq,
                   const uint16_t *Vd, const int *lens, const int *ars, int n_agents, int kv_cap, int n_qh, int n_kvh,
                   float scale, uint16_t *O, float *part, cudaStream_t s, bool pdl);
int prefill_set_stall(int at);  // test hook behind qad_debug_stall (kernel 2)
// Causal attention of a C-row prompt chunk of one agent (bf16 caches of that agent).
int launch_prefill_attn(const uint16_t *Q, const uint16_t *Kc, const uint16_t *Vc, int len, int C, int kv_cap, int n_qh,
                        int n_kvh, float scale, uint16_t *O, cudaStream_t s);
// Byte offset of the scale plane inside one q8_0 cache allocation.
size_t kv_q8_scale_offset(int n_agents, int n_kvh, int kv_cap);
AttnPartView attn_part_view(const AttnPlan &pl, const float *part, const int *ars, const int *lens, int kv_cap,
                            int n_qh, int n_kvh);

}  // namespace qad
