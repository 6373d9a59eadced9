// Weight-streaming expert mat-vec for small token counts (decode), with the
// shared expert handled as more work items of the same launch - the fusion of
// llama.cpp PR #29184 ("CUDA: fuse shared experts into MMVQ", release b11370)
// restated for this library.
//
// Work item = (j-th distinct routed expert, slice of 16/32/64 output rows), or
// (shared expert, slice).  A CTA finds its expert from ids itself (a bitmap of
// used experts, the j-th set bit), so the decode path needs no row-id launch.
// It then issues 1-D bulk copies for its whole weight slice (all k-steps of one
// activation window) into shared memory at once - the largest number of bytes
// in flight per SM - and stages the activations of its tokens while they
// land.  Dequantisation is exact (fp32 q*d); dot products accumulate in fp32,
// partial sums are combined by a fixed shuffle tree and a fixed-order sum, so
// the result does not depend on timing.
//
// Modes: single matrix (mul_mat_id rows, or the down projection writing
// dst[t][s]), or dual gate/up with a SwiGLU epilogue writing bf16 h[t][s].
// The down launch is a programmatic dependent of the gate/up launch: its CTAs
// start while gate/up runs, issue their weight copies, and only then wait for
// gate/up to finish before reading h.
#include "common.cuh"
#include "gemv_args.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kGvThreads = 256;
constexpr int kGvNT = 8;                 // tokens per pass
constexpr int kGvWeightBudget = 72 * 1024;
constexpr long long kGvWaitLimit = 1ll << 32;

struct GvSmem {
    uint32_t w_off, x_off, red_off, bm_off, bar_off, misc_off, total;
};

__host__ __device__ inline GvSmem gv_smem(const GemvSide& s, int dual, int n_experts) {
    const int nmat = dual + 1;
    const int xb = s.x_type == MOE_F32 ? 4 : 2;
    const int P = kGvThreads / (s.rows * 4);
    GvSmem m;
    uint32_t o = 0;
    m.w_off = o; o += (uint32_t)s.n_stages * nmat * s.rows * kRowBytes;
    m.x_off = o; o += (uint32_t)kGvNT * s.kw * xb;
    m.red_off = o; o += (uint32_t)P * s.rows * kGvNT * nmat * 4;
    m.bm_off = o; o += (uint32_t)((n_experts + 31) / 32 + 1) * 4;
    o = (o + 15) & ~15u;
    m.bar_off = o; o += (uint32_t)s.n_stages * 8;
    m.misc_off = o; o += 64 * 4;
    m.total = o;
    return m;
}

__device__ __forceinline__ float ld_x16(uint32_t bits16, int x_type) {
    return x_type == MOE_BF16 ? __uint_as_float(bits16 << 16) : __half2float(__ushort_as_half((unsigned short)bits16));
}

__device__ __forceinline__ bool gv_wait(uint64_t* bar, uint32_t parity, int* status) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!ptx::mbar_try_wait_sleep(bar, parity, 20000)) {
        if (clock64() - t0 > kGvWaitLimit) {
            set_status(status, MOE_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Exclusive block prefix sum (256 threads) of v; *total receives the sum.
__device__ __forceinline__ int gv_scan(int v, int* scratch, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int w = 0; w < kGvThreads / 32; ++w) {
            int t = scratch[w];
            scratch[w] = run;
            run += t;
        }
        *total = run;
    }
    __syncthreads();
    int r = scratch[warp] + incl - v;
    __syncthreads();
    return r;
}

template <int DUAL, int XB>
__global__ void __launch_bounds__(kGvThreads)
gemv_kernel(const GemvArgs a) {
    extern __shared__ __align__(16) uint8_t sm[];
    constexpr int NMAT = DUAL + 1;
    int* status = a.hdr + kHdrStatus;
    if (!a.pdl_secondary) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (read_status(status) != 0) return;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int routed_items = a.max_distinct * a.routed.items;
    const bool is_shared = (int)blockIdx.x >= routed_items;
    const GemvSide& sd = is_shared ? a.shared : a.routed;
    const WLayout L = sd.L;
    const int R = sd.rows;
    const int item = is_shared ? (int)blockIdx.x - routed_items : (int)blockIdx.x % sd.items;
    const int j = is_shared ? 0 : (int)blockIdx.x / sd.items;
    const int mt = item * R / kTileM, r0 = item * R % kTileM;
    const int rows_mt = L.rows(mt);
    const GvSmem lay = gv_smem(sd, DUAL, a.n_experts);
    uint8_t* sw = sm + lay.w_off;
    uint8_t* sx = sm + lay.x_off;
    float* red = (float*)(sm + lay.red_off);
    uint32_t* bm = (uint32_t*)(sm + lay.bm_off);
    uint64_t* bars = (uint64_t*)(sm + lay.bar_off);
    int* misc = (int*)(sm + lay.misc_off);  // [0..7] scan scratch, [8] total, [9] expert, [16..23] rows
    const int S = a.n_tokens * a.k;

    // ---- which expert, and how many of its slots
    int e = 0, n_sl = a.n_tokens;
    if (!is_shared) {
        const int nwords = (a.n_experts + 31) / 32;
        for (int w = tid; w < nwords; w += kGvThreads) bm[w] = 0u;
        __syncthreads();
        for (int i = tid; i < S; i += kGvThreads) {
            const int v = __ldg(a.ids + i);
            if (v >= 0 && v < a.n_experts) atomicOr(&bm[v >> 5], 1u << (v & 31));
            else set_status(status, MOE_ERR_BAD_ID);
        }
        __syncthreads();
        const int wpt = (nwords + kGvThreads - 1) / kGvThreads;
        const int w0 = min(nwords, tid * wpt), w1 = min(nwords, w0 + wpt);
        int local = 0;
        for (int w = w0; w < w1; ++w) local += __popc(bm[w]);
        const int before = gv_scan(local, misc, &misc[8]);
        if (j >= before && j < before + local) {
            int need = j - before;
            for (int w = w0; w < w1; ++w) {
                const int cw = __popc(bm[w]);
                if (need < cw) {
                    uint32_t bits = bm[w];
                    for (int q = 0; q < need; ++q) bits &= bits - 1;
                    misc[9] = w * 32 + __ffs(bits) - 1;
                    break;
                }
                need -= cw;
            }
        }
        __syncthreads();
        if (j >= misc[8]) return;  // fewer distinct experts than this item's index
        e = misc[9];
        int cnt = 0;
        for (int i = tid; i < S; i += kGvThreads) cnt += (__ldg(a.ids + i) == e);
        cnt = __reduce_add_sync(0xffffffffu, cnt);
        __syncthreads();
        if (lane == 0) misc[warp] = cnt;
        __syncthreads();
        n_sl = 0;
        for (int w = 0; w < kGvThreads / 32; ++w) n_sl += misc[w];
        __syncthreads();
    }

    // ---- weight stream: one window of k-steps at a time, all copies issued at once
    const int KT = L.kt_count;
    const int NW = sd.kw / kTileK;
    const bool resident = KT <= NW;
    const uint32_t piece_q = (uint32_t)R * kTileK, piece_d = (uint32_t)R * 4;
    const uint32_t stage_bytes = (uint32_t)NMAT * (piece_q + piece_d);
    if (tid == 0) {
        for (int s = 0; s < sd.n_stages; ++s) ptx::mbar_init(&bars[s], 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    // stage s completes one phase per arm; windows may arm different numbers of
    // stages, so each stage keeps its own parity bit
    uint32_t next_par = 0, wait_par = 0;
    auto issue = [&](int kt0, int kt1) {
        if (tid == 0) {
            for (int kt = kt0; kt < kt1; ++kt) {
                const int s = kt - kt0;
                uint8_t* dst = sw + (size_t)s * stage_bytes;
                ptx::mbar_arrive_expect_tx(&bars[s], stage_bytes);
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    const uint8_t* blk = (m ? sd.W1 : sd.W0) + L.block(e, mt, kt);
                    ptx::bulk_g2s(dst + m * (piece_q + piece_d), blk + (size_t)r0 * kTileK, piece_q, &bars[s]);
                    ptx::bulk_g2s(dst + m * (piece_q + piece_d) + piece_q, blk + (size_t)rows_mt * kTileK + r0 * 4,
                                  piece_d, &bars[s]);
                }
            }
        }
        const uint32_t armed = (kt1 - kt0) >= 32 ? 0xffffffffu : ((1u << (kt1 - kt0)) - 1u);
        wait_par = next_par;
        next_par ^= armed;
    };
    if (resident) issue(0, KT);
    if (a.pdl_secondary) asm volatile("griddepcontrol.wait;" ::: "memory");

    const int c = tid & 3, r = (tid >> 2) % R, ph = tid / (R * 4);
    const int P = kGvThreads / (R * 4);
    int* rows_sh = misc + 16;
    bool ok = true;
    for (int g0 = 0; g0 < n_sl && ok; g0 += kGvNT) {
        const int nt = min(kGvNT, n_sl - g0);
        // slots (routed: ascending t*k+s) or tokens (shared) of this group
        if (is_shared) {
            if (tid < nt) rows_sh[tid] = g0 + tid;
        } else {
            int base = 0;
            for (int i0 = 0; i0 < S; i0 += kGvThreads) {
                const int i = i0 + tid;
                const bool hit = i < S && __ldg(a.ids + i) == e;
                const unsigned bal = __ballot_sync(0xffffffffu, hit);
                if (lane == 0) misc[warp] = __popc(bal);
                __syncthreads();
                int before = base;
                for (int w = 0; w < warp; ++w) before += misc[w];
                const int rank = before + __popc(bal & ((1u << lane) - 1u));
                if (hit && rank >= g0 && rank < g0 + nt) rows_sh[rank - g0] = i;
                int tot = 0;
                for (int w = 0; w < kGvThreads / 32; ++w) tot += misc[w];
                base += tot;
                __syncthreads();
            }
        }
        float acc[NMAT][kGvNT];
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int i = 0; i < kGvNT; ++i) acc[m][i] = 0.f;

        for (int kt0 = 0; kt0 < KT && ok; kt0 += NW) {
            const int kt1 = min(KT, kt0 + NW);
            __syncthreads();  // previous window's stages and activations are free
            if (!resident) issue(kt0, kt1);
            // stage the activation window [kt0*64, kt1*64) of the group's rows
            const int cols = (kt1 - kt0) * kTileK;
            if (XB == 2) {
                const uint16_t* xg = (const uint16_t*)sd.x;
                for (int idx = tid; idx < nt * cols / 8; idx += kGvThreads) {
                    const int i = idx / (cols / 8), c8 = (idx % (cols / 8)) * 8, col = kt0 * kTileK + c8;
                    const int row = is_shared ? rows_sh[i] : (sd.x_per_slot ? rows_sh[i] : rows_sh[i] / a.k);
                    uint4 v = make_uint4(0, 0, 0, 0);
                    if (col < L.n_in) v = __ldg((const uint4*)(xg + (size_t)row * L.n_in + col));
                    *(uint4*)(sx + ((size_t)i * sd.kw + c8) * 2) = v;
                }
            } else {
                const float* xg = (const float*)sd.x;
                for (int idx = tid; idx < nt * cols / 4; idx += kGvThreads) {
                    const int i = idx / (cols / 4), c4 = (idx % (cols / 4)) * 4, col = kt0 * kTileK + c4;
                    const int row = is_shared ? rows_sh[i] : (sd.x_per_slot ? rows_sh[i] : rows_sh[i] / a.k);
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (col < L.n_in) v = __ldg((const float4*)(xg + (size_t)row * L.n_in + col));
                    *(float4*)(sx + ((size_t)i * sd.kw + c4) * 4) = v;
                }
            }
            __syncthreads();
            for (int kt = kt0 + ph; kt < kt1; kt += P) {
                const int s = kt - kt0;
                if (!gv_wait(&bars[s], (wait_par >> s) & 1u, status)) { ok = false; break; }
                const uint8_t* st = sw + (size_t)s * stage_bytes;
                float w[NMAT][16];
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    const uint8_t* pm = st + m * (piece_q + piece_d);
                    const uint4 q = *(const uint4*)(pm + r * kTileK + c * 16);
                    const float d = __half2float(*(const __half*)(pm + piece_q + r * 4 + (c >> 1) * 2));
                    const float nd = -32896.0f * d;
                    const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int b = 0; b < 16; ++b) w[m][b] = fmaf(magic_byte(qw[b >> 2], b & 3), d, nd);
                }
                const int xc = s * kTileK + c * 16;
#pragma unroll
                for (int i = 0; i < kGvNT; ++i) {
                    if (i < nt) {
                        float xv[16];
                        if (XB == 2) {
                            const uint4 u0 = *(const uint4*)(sx + ((size_t)i * sd.kw + xc) * 2);
                            const uint4 u1 = *(const uint4*)(sx + ((size_t)i * sd.kw + xc + 8) * 2);
                            const uint32_t uw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                            for (int b = 0; b < 8; ++b) {
                                xv[2 * b] = ld_x16(uw[b] & 0xffffu, sd.x_type);
                                xv[2 * b + 1] = ld_x16(uw[b] >> 16, sd.x_type);
                            }
                        } else {
#pragma unroll
                            for (int b = 0; b < 16; b += 4) {
                                const float4 v = *(const float4*)(sx + ((size_t)i * sd.kw + xc + b) * 4);
                                xv[b] = v.x; xv[b + 1] = v.y; xv[b + 2] = v.z; xv[b + 3] = v.w;
                            }
                        }
#pragma unroll
                        for (int m = 0; m < NMAT; ++m) {
                            float t = 0.f;
#pragma unroll
                            for (int b = 0; b < 16; ++b) t = fmaf(w[m][b], xv[b], t);
                            acc[m][i] += t;
                        }
                    }
                }
            }
        }
        // reduce: the 4 chunk lanes by a fixed butterfly, then the k phases in order
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int i = 0; i < kGvNT; ++i) {
                float v = acc[m][i];
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                acc[m][i] = v;
            }
        if (c == 0)
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int i = 0; i < kGvNT; ++i) red[((ph * R + r) * kGvNT + i) * NMAT + m] = acc[m][i];
        __syncthreads();
        for (int idx = tid; idx < R * kGvNT; idx += kGvThreads) {
            const int row = idx / kGvNT, i = idx % kGvNT;
            const int n = mt * kTileM + r0 + row;
            if (i < nt && n < L.n_out) {
                float v[NMAT];
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    v[m] = 0.f;
                    for (int q = 0; q < P; ++q) v[m] += red[((q * R + row) * kGvNT + i) * NMAT + m];
                }
                const int64_t orow = rows_sh[i];
                if (DUAL) {
                    const float g = v[0], u = v[NMAT - 1];
                    sd.h[orow * L.n_out + n] = __float2bfloat16_rn(g / (1.0f + expf(-g)) * u);
                } else {
                    sd.out[orow * L.n_out + n] = v[0];
                }
            }
        }
        __syncthreads();
    }
}

void gemv_plan_side(GemvSide& s, int dual) {
    const int nmat = dual + 1;
    const int xb = s.x_type == MOE_F32 ? 4 : 2;
    s.kw = xb == 2 ? 2048 : 1024;
    s.n_stages = s.L.kt_count < s.kw / kTileK ? s.L.kt_count : s.kw / kTileK;
    s.rows = 16;
    for (int R : {64, 32}) {
        if (s.L.n_out_pad % R == 0 && s.n_stages * nmat * R * kRowBytes <= kGvWeightBudget) {
            s.rows = R;
            break;
        }
    }
    s.items = s.L.n_out_pad / s.rows;
}

template <int DUAL, int XB>
static moe_status launch_t(const GemvArgs& a, size_t smem, unsigned grid, cudaStream_t stream) {
    static int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        if (cudaFuncSetAttribute(gemv_kernel<DUAL, XB>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        attr_dev = dev;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kGvThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl_secondary ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemv_kernel<DUAL, XB>, a) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status launch_gemv(const GemvArgs& a, cudaStream_t stream) {
    const int64_t grid = (int64_t)a.max_distinct * a.routed.items + (a.has_shared ? a.shared.items : 0);
    if (grid == 0) return MOE_OK;
    size_t smem = gv_smem(a.routed, a.dual, a.n_experts).total;
    if (a.has_shared) {
        size_t s2 = gv_smem(a.shared, a.dual, a.n_experts).total;
        if (s2 > smem) smem = s2;
    }
    const bool f32 = a.routed.x_type == MOE_F32 || (a.has_shared && a.shared.x_type == MOE_F32);
    if (f32 && a.has_shared && a.routed.x_type != a.shared.x_type) return MOE_ERR_UNSUPPORTED;
    if (a.dual)
        return f32 ? launch_t<1, 4>(a, smem, (unsigned)grid, stream) : launch_t<1, 2>(a, smem, (unsigned)grid, stream);
    return f32 ? launch_t<0, 4>(a, smem, (unsigned)grid, stream) : launch_t<0, 2>(a, smem, (unsigned)grid, stream);
}

}  // namespace moe
