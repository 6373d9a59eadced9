// Host-side argument blocks of the grouped tensor-core GEMM (gemm.cu).
#pragma once
#include "common.cuh"

namespace moe {

struct GemmMulMatId {
    int wtype;        // MOE_Q8_0 / MOE_MXFP4
    const uint8_t* W;
    int E, n_out, n_in;
    const void* x;
    int x_type;
    int64_t x_rows;   // rows of x: n_tokens (broadcast) or n_tokens*k (per_slot)
    void* xt;         // workspace: gathered x, tile-major and swizzled (rows_pad rows), fp16
    float* xs;        // workspace: per tiled row, the power of two that undoes its scaling
    int64_t rows_pad;
    const int32_t* pad_start;
    int64_t S;
    float* dst;
    const int32_t* bounds;
    const int32_t* ntile_prefix;
    const int32_t* ids_src1;
    const int32_t* ids_dst;
    const int32_t* slot_prow;  // tiled row of each slot t*k+s
    int k;
    int* hdr;
};

struct GemmFfn {
    int wtype;        // MOE_Q8_0 / MOE_MXFP4
    const uint8_t *Wg, *Wu, *Wd;
    int E, n_embd, n_ff;
    const uint8_t *Sg, *Su, *Sd;
    int n_ff_shared;
    const void* x;
    int x_type;
    void* xt;         // gathered x (routed), tile-major and swizzled, fp16
    void* xt_sh;      // x in token order for the shared expert, fp16
    float* xs;        // per tiled row of xt / xt_sh: the power of two that undoes its scaling
    float* xs_sh;
    int64_t rows_pad, rows_pad_sh;
    const int32_t* pad_start;
    int64_t T, S;
    float* dst;
    float* dst_shared;
    __nv_bfloat16* h;     // tile-major swizzled hidden activations (GEMM path)
    __nv_bfloat16* h_sh;
    const int32_t* bounds;
    const int32_t* ntile_prefix;
    const int32_t* ids_src1;
    const int32_t* ids_dst;
    const int32_t* slot_prow;  // tiled row of each slot t*k+s
    int k;
    int* hdr;
};

moe_status launch_gemm_mul_mat_id(const GemmMulMatId& g, cudaStream_t stream);
moe_status launch_gemm_ffn(const GemmFfn& g, cudaStream_t stream);

}  // namespace moe
