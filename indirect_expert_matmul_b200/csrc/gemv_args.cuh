// Argument block of the expert mat-vec kernel (gemv.cu).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace moe {

constexpr int kGvMaxSlots = 1024;   // the mat-vec path handles n_tokens*k up to this
constexpr int kGvNT = 8;            // tokens per pass over a weight stage

struct GemvSide {
    const uint8_t* W0;  // prepared weights (single, or gate)
    const uint8_t* W1;  // up (dual) or null
    WLayout L;
    const void* x;      // activations: rows of L.n_in elements
    int x_type;         // MOE_BF16 / MOE_F16 / MOE_F32
    int x_per_slot;     // routed x row: 1 -> slot t*k+s, 0 -> token t
    float* out;         // single: out[slot][n] (routed) or out[t][n] (shared)
    __nv_bfloat16* h;   // dual: h[slot][n] (routed) or h[t][n] (shared)
    // launch plan (filled by launch_gemv)
    int rsub;           // rows per work item: 32, 64 or 128
    int subs;           // work items per expert (row sub-tiles, counting empty ones of a tail tile)
    int kps;            // k-steps per ring stage
    // tensor maps of W0 / W1 over [tile][k-step][line][inner bytes] (filled by
    // launch_gemv when every row tile is full): one copy fetches a stage's
    // k-steps of a sub-tile; tma = 0: one bulk copy per k-step instead
    CUtensorMap tm[2];
    int tma;
};

struct GemvArgs {
    GemvSide routed, shared;
    int has_shared;
    int dual;
    int wtype;           // MOE_Q8_0 / MOE_MXFP4 (both sides)
    const int32_t* ids;  // [n_tokens][k]
    int n_tokens, k, n_experts;
    int max_distinct;    // min(n_tokens*k, n_experts)
    int pdl_wait;        // may start before the previous kernel of the stream ends: wait first
    int pdl_trigger;     // has a programmatic dependent: let it start once ids are valid
    int pdl_secondary;   // programmatic dependent: consumers wait before reading activations
    int finalize;        // the last CTA to finish copies the status to status_out and clears the header
    int* status_out;     // finalize: receives the status word (may be null)
    int* hdr;
    long long wait_limit;  // cycles a bounded wait may take (0: the default, ~2 s)
    int stall_cta, stall_stage;  // test-only: this CTA's producer skips this ring stage (-1: none)
    int ns;              // ring stages (filled by launch_gemv)
};

moe_status launch_gemv(const GemvArgs& a, cudaStream_t stream);
// Default plan of a side (128-row items); launch_gemv chooses the final plan.
void gemv_plan_side(GemvSide& s, int dual);

}  // namespace moe
