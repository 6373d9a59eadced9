// extern "C" entry points of include/moe.h: argument checks on the host,
// workspace carving, and dispatch to the kernels.  No entry point allocates
// memory or synchronises (except moe_get_status, which is documented to).
#include <atomic>

#include "common.cuh"

namespace moe {
moe_status launch_row_ids(const int32_t* ids, int64_t S, int k, int E, int mode, int32_t* ids_src1,
                          int32_t* ids_dst, int32_t* bounds, int32_t* active, int32_t* ntile_prefix,
                          int32_t* pad_start, int32_t* slot_prow, int bn, int* hdr, int32_t* rid_scratch,
                          cudaStream_t stream, int* launches = nullptr);
moe_status launch_prepare(int wtype, const void* src, int E, int n_out, int n_in, void* dst, cudaStream_t stream);
}  // namespace moe

#include "gemv_args.cuh"
#include "gemm_api.cuh"

using namespace moe;

// (the mat-vec path measured faster than the GEMM path up to 24 tokens on the
// 2048 -> 512 -> 2048 decode shape, and past 32 on the 7168 -> 2048 one)
static std::atomic<int> g_gemv_threshold{24};
static std::atomic<int> g_path{0};

static bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

static moe_status check_sizes(int64_t n_tokens, int k, int n_experts) {
    if (n_tokens < 0 || k < 1 || n_experts < 1) return MOE_ERR_INVALID;
    if (n_tokens >= kMaxTokens || k >= kMaxK || k > n_experts) return MOE_ERR_RANGE;
    if (n_tokens * (int64_t)k >= ((int64_t)1 << 31)) return MOE_ERR_RANGE;
    if (n_experts > kMaxExperts) return MOE_ERR_RANGE;
    return MOE_OK;
}

static bool use_gemv(int64_t n_tokens, int64_t S) {
    if (S > kGvMaxSlots) return false;  // beyond the mat-vec kernel's slot scan
    int p = g_path.load();
    if (p == 1) return true;
    if (p == 2) return false;
    return n_tokens <= g_gemv_threshold.load();
}

extern "C" {

const char* moe_status_string(int s) {
    switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID: return "MOE_ERR_INVALID";
    case MOE_ERR_RANGE: return "MOE_ERR_RANGE";
    case MOE_ERR_BAD_ID: return "MOE_ERR_BAD_ID";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    default: return "unknown moe_status";
    }
}

size_t moe_workspace_size(int64_t n_tokens, int k, int n_experts, int n_in, int n_hidden, int n_hidden_shared,
                          moe_dtype x_type) {
    if (n_tokens < 0 || k < 0 || n_experts < 0 || n_in < 0 || n_hidden < 0 || n_hidden_shared < 0) return 0;
    return WsLayout(n_tokens, k, n_experts, n_in, n_hidden, n_hidden_shared, x_type).total;
}

moe_status moe_workspace_init(void* workspace, moe_stream stream) {
    if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID;
    return cudaMemsetAsync(workspace, 0, 256, (cudaStream_t)stream) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_get_status(void* workspace, moe_stream stream) {
    if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
    int st = 0;
    if (cudaMemcpy(&st, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (st != 0 && cudaMemset(workspace, 0, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    return (moe_status)st;
}

static bool valid_wtype(int w) { return w == MOE_Q8_0 || w == MOE_MXFP4; }

size_t moe_weights_prepared_size_w(moe_wtype w_type, int n_experts, int n_out, int n_in) {
    if (!valid_wtype(w_type) || n_experts <= 0 || n_out <= 0 || n_in <= 0) return 0;
    return (size_t)(n_experts * WLayout(n_out, n_in, w_type).expert_bytes);
}

size_t moe_weights_prepared_size(int n_experts, int n_out, int n_in) {
    return moe_weights_prepared_size_w(MOE_Q8_0, n_experts, n_out, n_in);
}

moe_status moe_weights_prepare_w(moe_wtype w_type, const void* blocks, int n_experts, int n_out, int n_in,
                                 void* prepared, moe_stream stream) {
    if (!valid_wtype(w_type)) return MOE_ERR_INVALID;
    if (!blocks || !prepared || n_experts <= 0 || n_out <= 0 || n_in <= 0) return MOE_ERR_INVALID;
    if (n_in % 32 || !aligned(prepared, 16) || (w_type == MOE_Q8_0 && !aligned(blocks, 2))) return MOE_ERR_INVALID;
    if (n_experts > kMaxExperts) return MOE_ERR_RANGE;
    return launch_prepare(w_type, blocks, n_experts, n_out, n_in, prepared, (cudaStream_t)stream);
}

moe_status moe_weights_prepare(const void* q8_0_blocks, int n_experts, int n_out, int n_in, void* prepared,
                               moe_stream stream) {
    return moe_weights_prepare_w(MOE_Q8_0, q8_0_blocks, n_experts, n_out, n_in, prepared, stream);
}

moe_status moe_row_ids(const int32_t* ids, int64_t n_tokens, int k, int n_experts, moe_mode mode,
                       int32_t* ids_src1, int32_t* ids_dst, int32_t* expert_bounds, void* workspace,
                       moe_stream stream) {
    moe_status st = check_sizes(n_tokens, k, n_experts);
    if (st) return st;
    if (mode != MOE_BROADCAST && mode != MOE_PER_SLOT) return MOE_ERR_INVALID;
    if (!expert_bounds || !workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID;
    if (n_tokens > 0 && (!ids || !ids_src1 || !ids_dst)) return MOE_ERR_INVALID;
    WsLayout W(n_tokens, k, n_experts, 0, 0, 0, MOE_BF16);
    char* ws = (char*)workspace;
    prof_begin((cudaStream_t)stream);
    int n_rid = 1;  // launches of the row-id pass
    st = launch_row_ids(ids, n_tokens * k, k, n_experts, mode, ids_src1, ids_dst, expert_bounds,
                        (int32_t*)(ws + W.active), (int32_t*)(ws + W.tiles), (int32_t*)(ws + W.pad),
                        (int32_t*)(ws + W.sprow), kGemmBN, (int*)(ws + W.hdr),
                        n_experts <= kRidMaxE ? (int32_t*)(ws + W.rid) : nullptr, (cudaStream_t)stream, &n_rid);
    prof_mark((cudaStream_t)stream, "row_ids", n_rid);
    return st;
}

moe_status moe_mul_mat_id(const void* W_prepared, int n_experts, int n_out, int n_in, const void* x,
                          moe_dtype x_type, const int32_t* ids, int64_t n_tokens, int k, moe_mode mode,
                          float* dst, void* workspace, moe_stream stream) {
    return moe_mul_mat_id_w(MOE_Q8_0, W_prepared, n_experts, n_out, n_in, x, x_type, ids, n_tokens, k, mode, dst,
                            workspace, stream);
}

moe_status moe_mul_mat_id_w(moe_wtype w_type, const void* W_prepared, int n_experts, int n_out, int n_in,
                            const void* x, moe_dtype x_type, const int32_t* ids, int64_t n_tokens, int k,
                            moe_mode mode, float* dst, void* workspace, moe_stream stream) {
    if (!valid_wtype(w_type)) return MOE_ERR_INVALID;
    moe_status st = check_sizes(n_tokens, k, n_experts);
    if (st) return st;
    if (mode != MOE_BROADCAST && mode != MOE_PER_SLOT) return MOE_ERR_INVALID;
    if (x_type != MOE_BF16 && x_type != MOE_F16 && x_type != MOE_F32) return MOE_ERR_INVALID;
    if (n_out <= 0 || n_in <= 0 || n_in % 32) return MOE_ERR_INVALID;
    if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID;
    if (n_tokens == 0) return MOE_OK;
    if (!W_prepared || !x || !ids || !dst || !aligned(W_prepared, 256)) return MOE_ERR_INVALID;
    if (!aligned(x, 16) || !aligned(dst, 16)) return MOE_ERR_INVALID;
    cudaStream_t s = (cudaStream_t)stream;
    WsLayout W(n_tokens, k, n_experts, n_in, 0, 0, x_type);
    char* ws = (char*)workspace;
    int* hdr = (int*)(ws + W.hdr);
    int32_t *src1 = (int32_t*)(ws + W.src1), *dstr = (int32_t*)(ws + W.dst);
    int32_t *bounds = (int32_t*)(ws + W.bounds), *active = (int32_t*)(ws + W.active);
    int32_t* tiles = (int32_t*)(ws + W.tiles);
    const int64_t S = n_tokens * k;
    prof_begin(s);
    if (use_gemv(n_tokens, S)) {
        GemvArgs a = {};
        a.routed.W0 = (const uint8_t*)W_prepared;
        a.routed.L = WLayout(n_out, n_in, w_type);
        a.routed.x = x;
        a.routed.x_type = x_type;
        a.routed.x_per_slot = mode == MOE_PER_SLOT;
        a.routed.out = dst;
        gemv_plan_side(a.routed, 0);
        a.dual = 0;
        a.wtype = w_type;
        a.ids = ids;
        a.n_tokens = (int)n_tokens;
        a.k = k;
        a.n_experts = n_experts;
        a.max_distinct = (int)(S < n_experts ? S : n_experts);
        a.hdr = hdr;
        a.pdl_wait = 1;
        st = launch_gemv(a, s);
        prof_mark(s, "gemv");
        return st;
    }
    int n_rid = 1;  // launches of the row-id pass
    st = launch_row_ids(ids, S, k, n_experts, mode, src1, dstr, bounds, active, tiles, (int32_t*)(ws + W.pad),
                        (int32_t*)(ws + W.sprow), kGemmBN, hdr,
                        n_experts <= kRidMaxE ? (int32_t*)(ws + W.rid) : nullptr, s, &n_rid);
    if (st) return st;
    prof_mark(s, "row_ids", n_rid);
    GemmMulMatId g = {};
    g.wtype = w_type;
    g.W = (const uint8_t*)W_prepared;
    g.E = n_experts;
    g.n_out = n_out;
    g.n_in = n_in;
    g.x = x;
    g.x_type = x_type;
    g.x_rows = mode == MOE_BROADCAST ? n_tokens : S;
    g.xt = ws + W.xt;
    g.xs = (float*)(ws + W.xs);
    g.rows_pad = W.rows_pad;
    g.pad_start = (const int32_t*)(ws + W.pad);
    g.S = S;
    g.dst = dst;
    g.bounds = bounds;
    g.ntile_prefix = tiles;
    g.ids_src1 = src1;
    g.ids_dst = dstr;
    g.slot_prow = (const int32_t*)(ws + W.sprow);
    g.k = k;
    g.hdr = hdr;
    return launch_gemm_mul_mat_id(g, s);
}

moe_status moe_ffn(const void* Wg, const void* Wu, const void* Wd, int n_experts, int n_embd, int n_ff,
                   const void* Sg, const void* Su, const void* Sd, int n_ff_shared, const void* x, moe_dtype x_type,
                   const int32_t* ids, int64_t n_tokens, int k, float* dst, float* dst_shared, void* workspace,
                   moe_stream stream) {
    return moe_ffn_w(MOE_Q8_0, Wg, Wu, Wd, n_experts, n_embd, n_ff, Sg, Su, Sd, n_ff_shared, x, x_type, ids, n_tokens,
                     k, dst, dst_shared, workspace, stream);
}

moe_status moe_ffn_w(moe_wtype w_type, const void* Wg, const void* Wu, const void* Wd, int n_experts, int n_embd,
                     int n_ff, const void* Sg, const void* Su, const void* Sd, int n_ff_shared, const void* x,
                     moe_dtype x_type, const int32_t* ids, int64_t n_tokens, int k, float* dst, float* dst_shared,
                     void* workspace, moe_stream stream) {
    if (!valid_wtype(w_type)) return MOE_ERR_INVALID;
    moe_status st = check_sizes(n_tokens, k, n_experts);
    if (st) return st;
    if (x_type != MOE_BF16 && x_type != MOE_F16 && x_type != MOE_F32) return MOE_ERR_INVALID;
    if (n_embd <= 0 || n_ff <= 0 || n_embd % 32 || n_ff % 32 || n_ff_shared < 0 || n_ff_shared % 32)
        return MOE_ERR_INVALID;
    const bool has_shared = n_ff_shared > 0;
    if (has_shared && (!Sg || !Su || !Sd || !dst_shared)) return MOE_ERR_INVALID;
    if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID;
    if (n_tokens == 0) return MOE_OK;
    if (!Wg || !Wu || !Wd || !x || !ids || !dst) return MOE_ERR_INVALID;
    if (!aligned(Wg, 256) || !aligned(Wu, 256) || !aligned(Wd, 256) || !aligned(x, 16) || !aligned(dst, 16))
        return MOE_ERR_INVALID;
    if (has_shared && (!aligned(Sg, 256) || !aligned(Su, 256) || !aligned(Sd, 256) || !aligned(dst_shared, 16)))
        return MOE_ERR_INVALID;
    cudaStream_t s = (cudaStream_t)stream;
    WsLayout W(n_tokens, k, n_experts, n_embd, n_ff, n_ff_shared, x_type);
    char* ws = (char*)workspace;
    int* hdr = (int*)(ws + W.hdr);
    int32_t *src1 = (int32_t*)(ws + W.src1), *dstr = (int32_t*)(ws + W.dst);
    int32_t *bounds = (int32_t*)(ws + W.bounds), *active = (int32_t*)(ws + W.active);
    int32_t* tiles = (int32_t*)(ws + W.tiles);
    __nv_bfloat16* h = (__nv_bfloat16*)(ws + W.h);
    __nv_bfloat16* h_sh = (__nv_bfloat16*)(ws + W.h_sh);
    const int64_t S = n_tokens * k;
    prof_begin(s);
    if (use_gemv(n_tokens, S)) {
        GemvArgs a = {};
        a.has_shared = has_shared;
        a.ids = ids;
        a.n_tokens = (int)n_tokens;
        a.k = k;
        a.n_experts = n_experts;
        a.max_distinct = (int)(S < n_experts ? S : n_experts);
        a.hdr = hdr;
        // gate/up -> h[t][s] (SwiGLU), shared -> h_sh[t]
        a.dual = 1;
        a.wtype = w_type;
        a.routed.W0 = (const uint8_t*)Wg;
        a.routed.W1 = (const uint8_t*)Wu;
        a.routed.L = WLayout(n_ff, n_embd, w_type);
        a.routed.x = x;
        a.routed.x_type = x_type;
        a.routed.h = h;
        gemv_plan_side(a.routed, 1);
        a.pdl_wait = 1;     // may start during the previous kernel's tail; reads nothing before its wait
        a.pdl_trigger = 1;  // the down launch below may start once ids are valid
        if (has_shared) {
            a.shared.W0 = (const uint8_t*)Sg;
            a.shared.W1 = (const uint8_t*)Su;
            a.shared.L = WLayout(n_ff_shared, n_embd, w_type);
            a.shared.x = x;
            a.shared.x_type = x_type;
            a.shared.h = h_sh;
            gemv_plan_side(a.shared, 1);
        }
        st = launch_gemv(a, s);
        if (st) return st;
        prof_mark(s, "gemv_gate_up");
        // down -> dst[t][s], dst_shared[t]; a programmatic dependent of gate/up: its
        // producer streams the down weights while gate/up runs
        GemvArgs b = {};
        b.has_shared = has_shared;
        b.ids = ids;
        b.n_tokens = (int)n_tokens;
        b.k = k;
        b.n_experts = n_experts;
        b.max_distinct = a.max_distinct;
        b.hdr = hdr;
        b.dual = 0;
        b.wtype = w_type;
        b.pdl_secondary = 1;
        b.routed.W0 = (const uint8_t*)Wd;
        b.routed.L = WLayout(n_embd, n_ff, w_type);
        b.routed.x = h;
        b.routed.x_type = MOE_BF16;
        b.routed.x_per_slot = 1;
        b.routed.out = dst;
        gemv_plan_side(b.routed, 0);
        if (has_shared) {
            b.shared.W0 = (const uint8_t*)Sd;
            b.shared.L = WLayout(n_embd, n_ff_shared, w_type);
            b.shared.x = h_sh;
            b.shared.x_type = MOE_BF16;
            b.shared.out = dst_shared;
            gemv_plan_side(b.shared, 0);
        }
        st = launch_gemv(b, s);
        prof_mark(s, "gemv_down");
        return st;
    }
    int n_rid = 1;  // launches of the row-id pass
    st = launch_row_ids(ids, S, k, n_experts, MOE_BROADCAST, src1, dstr, bounds, active, tiles,
                        (int32_t*)(ws + W.pad), (int32_t*)(ws + W.sprow), kGemmBN, hdr,
                        n_experts <= kRidMaxE ? (int32_t*)(ws + W.rid) : nullptr, s, &n_rid);
    if (st) return st;
    prof_mark(s, "row_ids", n_rid);
    GemmFfn g = {};
    g.wtype = w_type;
    g.Wg = (const uint8_t*)Wg;
    g.Wu = (const uint8_t*)Wu;
    g.Wd = (const uint8_t*)Wd;
    g.E = n_experts;
    g.n_embd = n_embd;
    g.n_ff = n_ff;
    g.Sg = (const uint8_t*)Sg;
    g.Su = (const uint8_t*)Su;
    g.Sd = (const uint8_t*)Sd;
    g.n_ff_shared = n_ff_shared;
    g.x = x;
    g.x_type = x_type;
    g.xt = ws + W.xt;
    g.xt_sh = ws + W.xt_sh;
    g.xs = (float*)(ws + W.xs);
    g.xs_sh = (float*)(ws + W.xs_sh);
    g.rows_pad = W.rows_pad;
    g.rows_pad_sh = W.rows_pad_sh;
    g.pad_start = (const int32_t*)(ws + W.pad);
    g.T = n_tokens;
    g.S = S;
    g.dst = dst;
    g.dst_shared = dst_shared;
    g.h = h;
    g.h_sh = h_sh;
    g.bounds = bounds;
    g.ntile_prefix = tiles;
    g.ids_src1 = src1;
    g.ids_dst = dstr;
    g.slot_prow = (const int32_t*)(ws + W.sprow);
    g.k = k;
    g.hdr = hdr;
    return launch_gemm_ffn(g, s);
}

void moe_set_gemv_threshold(int n_tokens) { g_gemv_threshold.store(n_tokens < 0 ? 0 : n_tokens); }
int moe_get_gemv_threshold(void) { return g_gemv_threshold.load(); }
void moe_set_path(int path) { g_path.store(path); }

}  // extern "C"
