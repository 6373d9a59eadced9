// Argument block of the expert mat-vec kernel (gemv.cu).
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kGvMaxSlots = 8192;  // the mat-vec path handles n_tokens*k up to this

struct GemvSide {
    const uint8_t* W0;  // prepared weights (single, or gate)
    const uint8_t* W1;  // up (dual) or null
    WLayout L;
    const void* x;      // activations: rows of L.n_in elements
    int x_type;         // MOE_BF16 / MOE_F16 / MOE_F32
    int x_per_slot;     // routed x row: 1 -> slot t*k+s, 0 -> token t
    float* out;         // single: out[slot][n] (routed) or out[t][n] (shared)
    __nv_bfloat16* h;   // dual: h[slot][n] (routed) or h[t][n] (shared)
    int rows;           // rows per work item: 16, 32 or 64
    int items;          // work items per expert: n_out_pad / rows
    int n_stages;       // weight k-steps resident at once (one activation window)
    int kw;             // activation window (columns)
};

struct GemvArgs {
    GemvSide routed, shared;
    int has_shared;
    int dual;
    const int32_t* ids;  // [n_tokens][k]
    int n_tokens, k, n_experts;
    int max_distinct;    // min(n_tokens*k, n_experts): routed items = max_distinct * routed.items
    int pdl_secondary;   // launched as a programmatic dependent: wait before reading activations
    int* hdr;
    // launch plan (filled by launch_gemv)
    int nt_cap;          // tokens per pass
    int nbuf;            // 2: double-buffered whole weight slices; 1: windowed
    uint32_t buf_bytes, x_bytes, red_bytes, bm_words;
    int max_stages;
};

moe_status launch_gemv(const GemvArgs& a, cudaStream_t stream);
// Fill rows / items / n_stages / kw of a side for its shape and activation type.
void gemv_plan_side(GemvSide& s, int dual);

}  // namespace moe
