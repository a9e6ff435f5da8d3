// attn.cuh -- split-KV grouped-query decode attention launch interface.
#pragma once
#include "common.cuh"

namespace qad {

struct AttnPlan {
    int G;           // q-heads per kv-head
    int n_rg;        // groups of 24 query vectors per (agent, kv-head)
    int CH;          // keys per split (multiple of 64)
    int max_splits;  // splits covering kv_cap keys
    size_t part_bytes;
};

AttnPlan attn_plan(int n_agents, int n_qh, int n_kvh, int kv_cap, int max_rows_per_agent);
int launch_attn(const AttnPlan &pl, const uint16_t *Q, const uint16_t *Kc, const uint16_t *Vc, const int *lens,
                const int *ars, int n_agents, int kv_cap, int n_qh, int n_kvh, float scale, uint16_t *O, float *part,
                cudaStream_t s, bool pdl);

}  // namespace qad
