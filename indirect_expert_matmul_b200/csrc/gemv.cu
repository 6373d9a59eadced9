// Weight-streaming expert mat-vec for small token counts (decode), with the
// shared expert handled as one more work item of the same launch - the
// fusion of llama.cpp PR #29184 ("CUDA: fuse shared experts into MMVQ",
// release b11370) restated for this library.
//
// Work item = (expert with >= 1 slot, group of 16 output rows), or (shared
// expert, group of 16 rows).  Each item streams its rows' repacked Q8_0
// blocks exactly once per group of up to 8 tokens with 128-bit loads,
// dequantises in registers (exact fp32 q*d) and accumulates fp32 dot products
// against the staged activations of the expert's tokens.  Partial sums are
// combined by a fixed shuffle tree and a fixed-order shared-memory sum: the
// result does not depend on timing.
//
// Modes: single matrix (mul_mat_id, or the down projection that scatters to
// dst by ids_dst), or dual gate/up with a SwiGLU epilogue writing bf16 h in
// expert-sorted order.
#include "common.cuh"
#include "gemv_args.cuh"

namespace moe {

constexpr int kGvThreads = 256;
constexpr int kGvNT = 8;     // tokens per pass
constexpr int kGvRows = 16;  // rows per work item (2 per thread)
constexpr int kGvKW = 2048;  // activation window staged in shared memory

__device__ __forceinline__ float load_x(const void* x, int type, int64_t i) {
    if (type == MOE_BF16) return __bfloat162float(((const __nv_bfloat16*)x)[i]);
    if (type == MOE_F16) return __half2float(((const __half*)x)[i]);
    return ((const float*)x)[i];
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16 weights of one 16-byte chunk: w[l] = q_l * d, exact.
__device__ __forceinline__ void dequant16(uint4 q, float d, float w[16]) {
    const float nd = -32896.0f * d;
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int b = 0; b < 4; ++b) w[i * 4 + b] = fmaf(magic_byte(words[i], b), d, nd);
}

template <int DUAL>
__global__ void __launch_bounds__(kGvThreads)
gemv_kernel(GemvArgs a) {
    extern __shared__ float xs[];  // [kGvNT][kw]
    __shared__ float red[2][8][kGvRows][kGvNT];
    __shared__ int rows_sh[kGvNT];

    if (read_status(a.hdr + kHdrStatus) != 0) return;
    const int tid = threadIdx.x;
    const int c = tid & 3, rs = (tid >> 2) & 7, ktp = tid >> 5;

    // which work item
    int bid = blockIdx.x;
    const bool is_shared = bid >= a.max_active * a.routed.row_groups;
    const GemvSide& sd = is_shared ? a.shared : a.routed;
    int e = 0, rg, p0, p1;
    if (!is_shared) {
        int j = bid / a.routed.row_groups;
        rg = bid % a.routed.row_groups;
        if (j >= a.hdr[kHdrActive]) return;
        e = a.active[j];
        p0 = a.bounds[e];
        p1 = a.bounds[e + 1];
    } else {
        rg = bid - a.max_active * a.routed.row_groups;
        p0 = 0;
        p1 = a.n_tokens;
    }
    const WLayout L = sd.L;
    const int mt = rg / (kTileM / kGvRows);
    const int r_base = (rg % (kTileM / kGvRows)) * kGvRows;
    const int rows = L.rows(mt);
    if (r_base >= rows) return;
    const int kw = min(kGvKW, L.kt_count * kTileK);

    for (int g0 = p0; g0 < p1; g0 += kGvNT) {
        const int nt = min(kGvNT, p1 - g0);
        if (tid < nt) {
            int p = g0 + tid;
            rows_sh[tid] = is_shared ? p : (a.src_from_table ? a.ids_src1[p] : p);
        }
        float acc[2][2][kGvNT];
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int m = 0; m < 2; ++m)
#pragma unroll
                for (int i = 0; i < kGvNT; ++i) acc[s][m][i] = 0.f;

        for (int w0 = 0; w0 < L.kt_count * kTileK; w0 += kw) {
            __syncthreads();  // previous window / rows_sh
            for (int idx = tid; idx < nt * kw; idx += kGvThreads) {
                int i = idx / kw, kk = idx - i * kw, col = w0 + kk;
                xs[idx] = col < L.n_in ? load_x(sd.x, sd.x_type, (int64_t)rows_sh[i] * L.n_in + col) : 0.f;
            }
            __syncthreads();
            const int kt_end = min(L.kt_count, (w0 + kw) / kTileK);
#pragma unroll 2
            for (int kt = w0 / kTileK + ktp; kt < kt_end; kt += 8) {
                float wv[2][2][16];
                #pragma unroll
                for (int s = 0; s <= DUAL; ++s) {
                    const uint8_t* blk = (s ? sd.W1 : sd.W0) + L.block(e, mt, kt);
#pragma unroll
                    for (int m = 0; m < 2; ++m) {
                        int r = r_base + rs + 8 * m;
                        uint4 q = ldg_nc_v4(blk + (size_t)r * kTileK + c * 16);
                        float d = __half2float(*(const __half*)(blk + (size_t)rows * kTileK + r * 4 + (c >> 1) * 2));
                        dequant16(q, d, wv[s][m]);
                    }
                }
                const float* xk = xs + (kt * kTileK - w0) + c * 16;
#pragma unroll
                for (int i = 0; i < kGvNT; ++i) {
                    if (i < nt) {
                        float xv[16];
#pragma unroll
                        for (int l = 0; l < 16; l += 4) {
                            float4 v = *(const float4*)(xk + i * kw + l);
                            xv[l] = v.x; xv[l + 1] = v.y; xv[l + 2] = v.z; xv[l + 3] = v.w;
                        }
#pragma unroll
                        for (int s = 0; s <= DUAL; ++s)
#pragma unroll
                            for (int m = 0; m < 2; ++m) {
                                float t = 0.f;
#pragma unroll
                                for (int l = 0; l < 16; ++l) t = fmaf(wv[s][m][l], xv[l], t);
                                acc[s][m][i] += t;
                            }
                    }
                }
            }
        }
        // reduce over the 4 chunk lanes (fixed butterfly), then over the 8 k phases
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int m = 0; m < 2; ++m)
#pragma unroll
                for (int i = 0; i < kGvNT; ++i) {
                    float v = acc[s][m][i];
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    acc[s][m][i] = v;
                }
        if (c == 0) {
#pragma unroll
            for (int s = 0; s <= DUAL; ++s)
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int i = 0; i < kGvNT; ++i) red[s][ktp][rs + 8 * m][i] = acc[s][m][i];
        }
        __syncthreads();
        if (tid < kGvRows * kGvNT) {
            const int row = tid / kGvNT, i = tid % kGvNT;
            const int n = mt * kTileM + r_base + row;
            if (i < nt && n < L.n_out) {
                float v0 = 0.f, v1 = 0.f;
                for (int k8 = 0; k8 < 8; ++k8) v0 += red[0][k8][row][i];
                const int p = g0 + i;
                if (DUAL) {
                    for (int k8 = 0; k8 < 8; ++k8) v1 += red[1][k8][row][i];
                    float hval = v0 / (1.0f + expf(-v0)) * v1;  // silu(gate) * up
                    sd.h[(int64_t)p * L.n_out + n] = __float2bfloat16_rn(hval);
                } else {
                    int64_t orow = is_shared ? p : a.ids_dst[p];
                    sd.out[orow * L.n_out + n] = v0;
                }
            }
        }
    }
}

moe_status launch_gemv(const GemvArgs& a, cudaStream_t stream) {
    int64_t grid = (int64_t)a.max_active * a.routed.row_groups + (a.has_shared ? a.shared.row_groups : 0);
    if (grid == 0) return MOE_OK;
    int kt_max = a.routed.L.kt_count;
    if (a.has_shared && a.shared.L.kt_count > kt_max) kt_max = a.shared.L.kt_count;
    int kw = kt_max * kTileK < kGvKW ? kt_max * kTileK : kGvKW;
    size_t smem = (size_t)kGvNT * kw * sizeof(float);
    static int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        const int max_smem = (int)(kGvNT * kGvKW * sizeof(float));
        if (cudaFuncSetAttribute(gemv_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem) !=
                cudaSuccess)
            return MOE_ERR_CUDA;
        attr_dev = dev;
    }
    // each side derives its window from its own K; smem covers the larger one
    if (a.dual)
        gemv_kernel<1><<<(unsigned)grid, kGvThreads, smem, stream>>>(a);
    else
        gemv_kernel<0><<<(unsigned)grid, kGvThreads, smem, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
