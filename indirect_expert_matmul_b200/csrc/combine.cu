// Weighted combine of each token's expert outputs - the step that follows the
// indirect matmul in a MoE layer ("Optimalizace MoE modelů na slabém GPU:
// spuštění GPT-OSS-120B s 6 GB VRAM až 30 t/s", section "Architektura Mixture
// of Experts": a router picks k experts per token in every layer; the layer's
// output is their outputs weighted by the router), plus the always-on shared
// expert of "llama.cpp 發布 b11370，CUDA 後端將共享專家融合進 MMVQ":
//
//   y[t][j] = sum_s r[t][s] * dst[t][s][j]  (+ dst_shared[t][j])
//
// The slots are taken in ascending s with one fused multiply-add each, then
// the shared term is added once: every output is a fixed sequence of float
// roundings, bit-identical from run to run and independent of the launch shape.
//
// The kernel is a pure stream over dst (k reads per output element) and
// bound by HBM: 16-byte loads that bypass L1 retention, one thread per four
// consecutive outputs of a token row, 256-thread units of one token row
// handed out grid-stride over a grid sized to the SM count.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kCombineThreads = 256;

template <bool VEC, bool SHARED>
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const float* __restrict__ dst, const float* __restrict__ r, const float* __restrict__ sh,
               int64_t n_tokens, int k, int64_t n, float* __restrict__ y) {
    const int64_t nv = VEC ? n / 4 : n;  // vectors (or elements) per token row
    const int64_t units_per_row = (nv + kCombineThreads - 1) / kCombineThreads;
    const int64_t units = n_tokens * units_per_row;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int64_t t = u / units_per_row;
        const int64_t j = (u - t * units_per_row) * kCombineThreads + threadIdx.x;
        if (j >= nv) continue;
        const float* rt = r + t * k;
        const float* dt = dst + t * (int64_t)k * n;
        if (VEC) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int s = 0; s < k; ++s) {
                const float w = __ldg(rt + s);
                const float4 v = __ldcs(reinterpret_cast<const float4*>(dt + (int64_t)s * n) + j);
                acc.x = __fmaf_rn(w, v.x, acc.x);
                acc.y = __fmaf_rn(w, v.y, acc.y);
                acc.z = __fmaf_rn(w, v.z, acc.z);
                acc.w = __fmaf_rn(w, v.w, acc.w);
            }
            if (SHARED) {
                const float4 b = __ldcs(reinterpret_cast<const float4*>(sh + t * n) + j);
                acc.x = __fadd_rn(acc.x, b.x);
                acc.y = __fadd_rn(acc.y, b.y);
                acc.z = __fadd_rn(acc.z, b.z);
                acc.w = __fadd_rn(acc.w, b.w);
            }
            __stcs(reinterpret_cast<float4*>(y + t * n) + j, acc);
        } else {
            float acc = 0.f;
            for (int s = 0; s < k; ++s) acc = __fmaf_rn(__ldg(rt + s), __ldcs(dt + (int64_t)s * n + j), acc);
            if (SHARED) acc = __fadd_rn(acc, __ldcs(sh + t * n + j));
            __stcs(y + t * n + j, acc);
        }
    }
}

int sm_count_combine() {
    static int dev_cached = -1, n = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != dev_cached) {
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        dev_cached = dev;
    }
    return n > 0 ? n : 148;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_combine(const float* dst, const float* weights, const float* dst_shared, int64_t n_tokens,
                                  int k, int64_t n, float* y, moe_stream stream) {
    if (n_tokens < 0 || k < 1 || n < 1) return MOE_ERR_INVALID;
    if (n_tokens >= kMaxTokens || k >= kMaxK || n >= ((int64_t)1 << 31)) return MOE_ERR_RANGE;
    if (n_tokens == 0) return MOE_OK;
    if (!dst || !weights || !y) return MOE_ERR_INVALID;
    const uintptr_t a4 = (uintptr_t)dst | (uintptr_t)weights | (uintptr_t)y | (uintptr_t)dst_shared;
    if (a4 & 3u) return MOE_ERR_INVALID;
    const bool vec = n % 4 == 0 && aligned16(dst) && aligned16(y) && (!dst_shared || aligned16(dst_shared));
    const int64_t nv = vec ? n / 4 : n;
    const int64_t units = n_tokens * ((nv + kCombineThreads - 1) / kCombineThreads);
    const int64_t cap = (int64_t)sm_count_combine() * (2048 / kCombineThreads);  // one full wave of resident blocks
    const unsigned grid = (unsigned)(units < cap ? units : cap);
    cudaStream_t s = (cudaStream_t)stream;
    if (vec) {
        if (dst_shared)
            combine_kernel<true, true><<<grid, kCombineThreads, 0, s>>>(dst, weights, dst_shared, n_tokens, k, n, y);
        else
            combine_kernel<true, false><<<grid, kCombineThreads, 0, s>>>(dst, weights, nullptr, n_tokens, k, n, y);
    } else {
        if (dst_shared)
            combine_kernel<false, true><<<grid, kCombineThreads, 0, s>>>(dst, weights, dst_shared, n_tokens, k, n, y);
        else
            combine_kernel<false, false><<<grid, kCombineThreads, 0, s>>>(dst, weights, nullptr, n_tokens, k, n, y);
    }
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
