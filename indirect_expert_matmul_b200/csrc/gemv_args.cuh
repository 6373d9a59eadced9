// Argument block of the expert mat-vec kernel (gemv.cu).
#pragma once
#include "common.cuh"

namespace moe {

struct GemvSide {
    const uint8_t* W0;  // prepared weights (single, or gate)
    const uint8_t* W1;  // up (dual) or null
    WLayout L;
    const void* x;      // activations: rows of L.n_in elements
    int x_type;         // MOE_BF16 / MOE_F16 / MOE_F32
    float* out;         // single: out[row][n], row = ids_dst[p] (routed) or t (shared)
    __nv_bfloat16* h;   // dual: h[p][n] (routed) or h[t][n] (shared)
    int row_groups;     // ceil(n_out_pad / 16)
};

struct GemvArgs {
    GemvSide routed, shared;
    int has_shared;
    int dual;
    int src_from_table;  // routed x row: 1 -> ids_src1[p], 0 -> p
    int n_tokens;
    int max_active;
    const int32_t* bounds;
    const int32_t* active;
    const int32_t* ids_src1;
    const int32_t* ids_dst;
    const int* hdr;
};

moe_status launch_gemv(const GemvArgs& a, cudaStream_t stream);

}  // namespace moe
