// Router: the step before the indirect matmul in a MoE layer ("Optimalizace
// MoE modelů na slabém GPU: spuštění GPT-OSS-120B s 6 GB VRAM až 30 t/s",
// section "Architektura Mixture of Experts": a gating network picks k of the
// experts for every token).  For token t:
//
//   key[e]  = logits[t][e] + bias[e]     (one float addition)
//   ids[t]  = the k largest keys, descending, equal keys in ascending e
//   p[e]    = softmax over all experts of logits[t]
//   w[t][i] = p[ids[t][i]]  (divided by the sum over the k when normalising,
//             evaluated as the softmax over the k chosen logits)
//
// One warp per token.  The keys and logits of a token live in registers
// (ceil(n_experts / 32) per lane, rounded up to a power of two; n_experts <= 1024); each of the k rounds is a per-lane pairwise
// tree over the lane's candidates followed by a butterfly argmax, both
// comparing (key descending, expert ascending) - a total order, so every lane
// agrees on the same winner and the choice is a pure function of the float keys.  The softmax sums run in a fixed order
// (per lane ascending, then a fixed butterfly): bit-identical reruns.
#include <math.h>

#include "common.cuh"

namespace moe {

namespace {

constexpr int kRouteWarps = 8;
constexpr int kRouteMaxPerLane = 32;  // n_experts <= 1024

// (key, expert, logit) of a candidate; a beats b: larger key, or equal key and smaller expert
__device__ __forceinline__ bool beats(float ka, int ea, float kb, int eb) {
    return ka > kb || (ka == kb && ea < eb);
}

// NPL: expert slots per lane (n_experts <= 32 * NPL), a compile-time count so
// that the per-lane arrays stay in registers and no lane scans empty slots.
template <int NPL>
__global__ void __launch_bounds__(kRouteWarps * 32)
route_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int64_t n_tokens, int n_experts,
             int k, int normalize, int32_t* __restrict__ ids, float* __restrict__ weights) {
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
    if (t >= n_tokens) return;
    const float* lt = logits + t * n_experts;
    float l[NPL], key[NPL];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
        const int e = j * 32 + lane;
        l[j] = e < n_experts ? __ldg(lt + e) : -INFINITY;
        key[j] = e < n_experts ? (bias ? __fadd_rn(l[j], __ldg(bias + e)) : l[j]) : -INFINITY;
        mx = fmaxf(mx, l[j]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float z = 0.f;  // softmax denominator over all experts (unnormalised weights only)
    if (!normalize) {
#pragma unroll
        for (int j = 0; j < NPL; ++j)
            if (j * 32 + lane < n_experts) z = __fadd_rn(z, expf(__fsub_rn(l[j], mx)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z = __fadd_rn(z, __shfl_xor_sync(0xffffffffu, z, o));
    }

    uint32_t taken = 0u;  // bit j: expert j*32 + lane chosen
    float mine = -INFINITY;  // lane i (k <= 32): the logit chosen in round i
    int32_t* it = ids + t * k;
    float* wt = weights + t * k;
    for (int i = 0; i < k; ++i) {
        // this lane's best untaken candidate: a pairwise tree over its 32 slots
        // (the order is total, so any association picks the same winner)
        float ck[NPL], cl[NPL];
        int ce[NPL];
#pragma unroll
        for (int j = 0; j < NPL; ++j) {
            const int e = j * 32 + lane;
            const bool live = e < n_experts && !(taken >> j & 1u);
            ck[j] = live ? key[j] : -INFINITY;
            ce[j] = live ? e : 0x7fffffff;
            cl[j] = l[j];
        }
#pragma unroll
        for (int w = NPL / 2; w > 0; w >>= 1)
#pragma unroll
            for (int j = 0; j < w; ++j)
                if (beats(ck[j + w], ce[j + w], ck[j], ce[j])) {
                    ck[j] = ck[j + w];
                    ce[j] = ce[j + w];
                    cl[j] = cl[j + w];
                }
        float bk = ck[0], bl = cl[0];
        int be = ce[0];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const float ol = __shfl_xor_sync(0xffffffffu, bl, o);
            if (beats(ok, oe, bk, be)) {
                bk = ok;
                be = oe;
                bl = ol;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == (i & 31)) mine = bl;
        if (lane == 0) {
            it[i] = be;
            // unnormalised: the probability itself; normalised, k > 32: the chosen
            // logit, turned into its weight below
            wt[i] = normalize ? bl : __fdiv_rn(expf(__fsub_rn(bl, mx)), z);
        }
    }
    if (!normalize) return;
    // Renormalised weights p_i / sum_chosen p_j are the softmax over the chosen
    // logits alone; taken relative to the largest chosen logit, the sum is at
    // least 1, so it cannot underflow to zero however far the chosen logits sit
    // below the row's maximum.
    if (k <= 32) {
        // one chosen logit per lane; the sums run in a fixed butterfly order
        float mc = mine;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
        const float e = lane < k ? expf(__fsub_rn(mine, mc)) : 0.f;
        float sel = e;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sel = __fadd_rn(sel, __shfl_xor_sync(0xffffffffu, sel, o));
        if (lane < k) wt[lane] = __fdiv_rn(e, sel);
        return;
    }
    __syncwarp();
    if (lane == 0) {  // k > 32: lane 0, in choice order
        float mc = -INFINITY;
        for (int i = 0; i < k; ++i) mc = fmaxf(mc, wt[i]);
        float sel = 0.f;
        for (int i = 0; i < k; ++i) {
            const float e = expf(__fsub_rn(wt[i], mc));
            wt[i] = e;
            sel = __fadd_rn(sel, e);
        }
        for (int i = 0; i < k; ++i) wt[i] = __fdiv_rn(wt[i], sel);
    }
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_route(const float* logits, const float* bias, int64_t n_tokens, int n_experts, int k,
                                int normalize, int32_t* ids, float* weights, moe_stream stream) {
    if (n_tokens < 0 || n_experts < 1 || k < 1 || k > n_experts) return MOE_ERR_INVALID;
    if (n_tokens >= kMaxTokens || n_experts > kRouteMaxPerLane * 32 || k >= kMaxK) return MOE_ERR_RANGE;
    if (n_tokens == 0) return MOE_OK;
    if (!logits || !ids || !weights) return MOE_ERR_INVALID;
    if (((uintptr_t)logits | (uintptr_t)bias | (uintptr_t)ids | (uintptr_t)weights) & 3u) return MOE_ERR_INVALID;
    const unsigned blocks = (unsigned)((n_tokens + kRouteWarps - 1) / kRouteWarps);
    cudaStream_t s = (cudaStream_t)stream;
    const dim3 block(kRouteWarps * 32);
    if (n_experts <= 32) route_kernel<1><<<blocks, block, 0, s>>>(logits, bias, n_tokens, n_experts, k, normalize, ids, weights);
    else if (n_experts <= 64) route_kernel<2><<<blocks, block, 0, s>>>(logits, bias, n_tokens, n_experts, k, normalize, ids, weights);
    else if (n_experts <= 128) route_kernel<4><<<blocks, block, 0, s>>>(logits, bias, n_tokens, n_experts, k, normalize, ids, weights);
    else if (n_experts <= 256) route_kernel<8><<<blocks, block, 0, s>>>(logits, bias, n_tokens, n_experts, k, normalize, ids, weights);
    else if (n_experts <= 512) route_kernel<16><<<blocks, block, 0, s>>>(logits, bias, n_tokens, n_experts, k, normalize, ids, weights);
    else route_kernel<32><<<blocks, block, 0, s>>>(logits, bias, n_tokens, n_experts, k, normalize, ids, weights);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
