// moe_ffn_decode_noalloc: the decode-size SwiGLU expert FFN on the mat-vec
// path with its scratch in a static device array instead of a caller
// workspace.  It exists for callers that cannot pass scratch memory (a graph
// executor that plans every buffer per tensor ahead of time and runs each
// operation with only its inputs and outputs); nothing here allocates or
// frees memory.  The kernels and their arguments are those of moe_ffn's
// mat-vec branch; only where the status header and the hidden activations
// live differs.
#include <atomic>

#include "common.cuh"
#include "gemv_args.cuh"

namespace moe {

constexpr int64_t kNaMaxSlots = 64;      // n_tokens * k
constexpr int kNaMaxFF = 2048;           // n_ff and n_ff_shared
constexpr size_t kNaHdrBytes = 256;
constexpr size_t kNaHBytes = (size_t)kNaMaxSlots * kNaMaxFF * 2;  // bf16 h[slot][n_ff]
constexpr size_t kNaBytes = kNaHdrBytes + 2 * kNaHBytes;         // + h_sh[token][n_ff_shared]
constexpr int kNaMaxDevices = 64;

// The scratch: [status header | routed h | shared h].  One per device (a
// __device__ variable exists once in every device context that loads the
// library).
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNaBytes];

static std::atomic<unsigned char*> g_noalloc_addr[kNaMaxDevices];

// Address of this device's scratch, looked up once per device with that
// device current.
static moe_status noalloc_scratch(unsigned char** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kNaMaxDevices) return MOE_ERR_UNSUPPORTED;
    unsigned char* p = g_noalloc_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        void* sym = nullptr;
        if (cudaGetSymbolAddress(&sym, g_noalloc_scratch) != cudaSuccess || !sym) return MOE_ERR_CUDA;
        p = (unsigned char*)sym;
        g_noalloc_addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

static bool na_aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

extern "C" moe_status moe_ffn_decode_noalloc(const void* Wg, const void* Wu, const void* Wd, int n_experts,
                                              int n_embd, int n_ff, const void* Sg, const void* Su, const void* Sd,
                                              int n_ff_shared, const void* x, moe_dtype x_type, const int32_t* ids,
                                              int64_t n_tokens, int k, float* dst, float* dst_shared, int* status_out,
                                              moe_stream stream) {
    // host checks, before any CUDA call
    if (n_tokens < 0 || k < 1 || n_experts < 1) return MOE_ERR_INVALID;
    // the library-wide limits first, so that n_tokens * k below cannot overflow
    if (n_tokens >= kMaxTokens || k >= kMaxK) return MOE_ERR_RANGE;
    if (k > n_experts || n_experts > kMaxExperts) return MOE_ERR_RANGE;
    if (n_tokens * (int64_t)k > kNaMaxSlots || n_ff > kNaMaxFF || n_ff_shared > kNaMaxFF) return MOE_ERR_RANGE;
    if (x_type != MOE_BF16 && x_type != MOE_F16 && x_type != MOE_F32) return MOE_ERR_INVALID;
    if (n_embd <= 0 || n_ff <= 0 || n_embd % 32 || n_ff % 32 || n_ff_shared < 0 || n_ff_shared % 32)
        return MOE_ERR_INVALID;
    const bool has_shared = n_ff_shared > 0;
    if (has_shared && (!Sg || !Su || !Sd || !dst_shared)) return MOE_ERR_INVALID;
    if (status_out && !na_aligned(status_out, 4)) return MOE_ERR_INVALID;
    if (n_tokens > 0) {
        if (!Wg || !Wu || !Wd || !x || !ids || !dst) return MOE_ERR_INVALID;
        if (!na_aligned(Wg, 256) || !na_aligned(Wu, 256) || !na_aligned(Wd, 256) || !na_aligned(x, 16) ||
            !na_aligned(dst, 16))
            return MOE_ERR_INVALID;
        if (has_shared && (!na_aligned(Sg, 256) || !na_aligned(Su, 256) || !na_aligned(Sd, 256) ||
                           !na_aligned(dst_shared, 16)))
            return MOE_ERR_INVALID;
    }

    unsigned char* scratch = nullptr;
    moe_status st = noalloc_scratch(&scratch);
    if (st) return st;
    cudaStream_t s = (cudaStream_t)stream;
    int* hdr = (int*)scratch;
    __nv_bfloat16* h = (__nv_bfloat16*)(scratch + kNaHdrBytes);
    __nv_bfloat16* h_sh = (__nv_bfloat16*)(scratch + kNaHdrBytes + kNaHBytes);
    // The header is zero when the library loads and every call leaves it zero:
    // the down launch's last CTA copies the status to status_out and clears
    // it.  So a call is two launches, gate/up a programmatic dependent of
    // whatever ran before it on the stream.
    if (n_tokens == 0) {
        if (status_out && cudaMemsetAsync(status_out, 0, sizeof(int), s) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    {
        const int64_t S = n_tokens * k;
        GemvArgs a = {};
        a.has_shared = has_shared;
        a.ids = ids;
        a.n_tokens = (int)n_tokens;
        a.k = k;
        a.n_experts = n_experts;
        a.max_distinct = (int)(S < n_experts ? S : n_experts);
        a.hdr = hdr;
        a.dual = 1;  // gate/up -> h[t][s] (SwiGLU), shared -> h_sh[t]
        a.routed.W0 = (const uint8_t*)Wg;
        a.routed.W1 = (const uint8_t*)Wu;
        a.routed.L = WLayout(n_ff, n_embd);
        a.routed.x = x;
        a.routed.x_type = x_type;
        a.routed.h = h;
        gemv_plan_side(a.routed, 1);
        a.pdl_wait = 1;     // may start during the previous kernel's tail; reads nothing before its wait
        a.pdl_trigger = 1;  // the down launch may start once ids are valid
        if (has_shared) {
            a.shared.W0 = (const uint8_t*)Sg;
            a.shared.W1 = (const uint8_t*)Su;
            a.shared.L = WLayout(n_ff_shared, n_embd);
            a.shared.x = x;
            a.shared.x_type = x_type;
            a.shared.h = h_sh;
            gemv_plan_side(a.shared, 1);
        }
        st = launch_gemv(a, s);
        if (st) return st;
        GemvArgs b = {};  // down -> dst[t][s], dst_shared[t]
        b.has_shared = has_shared;
        b.ids = ids;
        b.n_tokens = (int)n_tokens;
        b.k = k;
        b.n_experts = n_experts;
        b.max_distinct = a.max_distinct;
        b.hdr = hdr;
        b.dual = 0;
        b.pdl_secondary = 1;
        b.finalize = 1;
        b.status_out = status_out;
        b.routed.W0 = (const uint8_t*)Wd;
        b.routed.L = WLayout(n_embd, n_ff);
        b.routed.x = h;
        b.routed.x_type = MOE_BF16;
        b.routed.x_per_slot = 1;
        b.routed.out = dst;
        gemv_plan_side(b.routed, 0);
        if (has_shared) {
            b.shared.W0 = (const uint8_t*)Sd;
            b.shared.L = WLayout(n_embd, n_ff_shared);
            b.shared.x = h_sh;
            b.shared.x_type = MOE_BF16;
            b.shared.out = dst_shared;
            gemv_plan_side(b.shared, 0);
        }
        st = launch_gemv(b, s);
        if (st) {
            // gate/up may have written the header: leave it zero for the next call
            cudaMemsetAsync(hdr, 0, kNaHdrBytes, s);
            return st;
        }
    }
    return MOE_OK;
}
