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
constexpr int kGvNT = 8;                   // tokens per pass, at most
constexpr int kGvWeightBudget = 72 * 1024; // weight bytes of one work item (one buffer)
constexpr long long kGvWaitLimit = 1ll << 32;

struct GvLay {
    uint32_t buf0, buf1, x, red, bm, wp, bars, misc, total;
};

__host__ __device__ inline GvLay gv_lay(const GemvArgs& a) {
    GvLay m;
    uint32_t o = 0;
    m.buf0 = o; o += a.buf_bytes;
    m.buf1 = o; o += a.nbuf == 2 ? a.buf_bytes : 0u;
    m.x = o; o += a.x_bytes;
    m.red = o; o += a.red_bytes;
    m.bm = o; o += a.bm_words * 4u;
    m.wp = o; o += (a.bm_words + 1u) * 4u;
    o = (o + 15u) & ~15u;
    m.bars = o; o += 2u * a.max_stages * 8u;
    m.misc = o; o += 64u * 4u;
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

// One work item: a slice of `R` output rows of one expert's matrix (or two).
struct GvItem {
    const GemvSide* sd;
    int shared, e, mt, r0, rows_mt;
};

template <int DUAL, int XB>
__global__ void __launch_bounds__(kGvThreads)
gemv_kernel(const GemvArgs a) {
    extern __shared__ __align__(128) uint8_t sm[];
    constexpr int NMAT = DUAL + 1;
    int* status = a.hdr + kHdrStatus;
    if (!a.pdl_secondary) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (read_status(status) != 0) return;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const GvLay lay = gv_lay(a);
    uint8_t* sbuf[2] = {sm + lay.buf0, sm + lay.buf1};
    uint8_t* sx = sm + lay.x;
    float* red = (float*)(sm + lay.red);
    uint32_t* bm = (uint32_t*)(sm + lay.bm);
    int* wp = (int*)(sm + lay.wp);
    uint64_t* bars = (uint64_t*)(sm + lay.bars);
    int* misc = (int*)(sm + lay.misc);  // [0..7] reduce scratch, [16..23] rows of the token group
    int* rows_sh = misc + 16;
    const int S = a.n_tokens * a.k;
    const int nwords = (int)a.bm_words;

    // ---- the distinct routed experts, once per CTA: bitmap + per-word prefix
    for (int w = tid; w < nwords; w += kGvThreads) bm[w] = 0u;
    if (tid == 0)
        for (int s = 0; s < 2 * a.max_stages; ++s) ptx::mbar_init(&bars[s], 1);
    ptx::fence_mbar_init();
    __syncthreads();
    for (int i = tid; i < S; i += kGvThreads) {
        const int v = __ldg(a.ids + i);
        if (v >= 0 && v < a.n_experts) atomicOr(&bm[v >> 5], 1u << (v & 31));
        else set_status(status, MOE_ERR_BAD_ID);
    }
    __syncthreads();
    if (warp == 0) {  // exclusive prefix of popcounts, 32 words per step
        int run = 0;
        for (int w0 = 0; w0 < nwords; w0 += 32) {
            const int w = w0 + lane;
            const int c = w < nwords ? __popc(bm[w]) : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (w < nwords) wp[w] = run + incl - c;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) wp[nwords] = run;
    }
    __syncthreads();
    const int n_distinct = wp[nwords];
    const int routed_items = n_distinct * a.routed.items;
    const int n_items = routed_items + (a.has_shared ? a.shared.items : 0);

    auto item_of = [&](int it) {
        GvItem f;
        int slice;
        if (it < routed_items) {
            const int j = it / a.routed.items;
            slice = it - j * a.routed.items;
            int lo = 0, hi = nwords;  // wp[lo] <= j < wp[hi]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (wp[mid] <= j) lo = mid; else hi = mid;
            }
            uint32_t bits = bm[lo];
            for (int q = j - wp[lo]; q > 0; --q) bits &= bits - 1;
            f.e = lo * 32 + __ffs(bits) - 1;
            f.shared = 0;
            f.sd = &a.routed;
        } else {
            slice = it - routed_items;
            f.e = 0;
            f.shared = 1;
            f.sd = &a.shared;
        }
        const int r = slice * f.sd->rows;
        f.mt = r / kTileM;
        f.r0 = r % kTileM;
        f.rows_mt = f.sd->L.rows(f.mt);
        return f;
    };

    // stage s of buffer b completes one phase per arm; each keeps its own parity bit
    uint32_t next_par[2] = {0u, 0u}, wait_par[2] = {0u, 0u};
    auto issue = [&](const GvItem& f, int b, int kt0, int kt1) {
        const GemvSide& sd = *f.sd;
        const uint32_t pq = (uint32_t)sd.rows * kTileK, pd = (uint32_t)sd.rows * 4u;
        const uint32_t stage_bytes = (uint32_t)NMAT * (pq + pd);
        if (warp == 0) {
            for (int s = lane; s < kt1 - kt0; s += 32) {
                uint8_t* dst = sbuf[b] + (size_t)s * stage_bytes;
                uint64_t* bar = &bars[b * a.max_stages + s];
                ptx::mbar_arrive_expect_tx(bar, stage_bytes);
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    // the slice's rows of both 32-column halves, then their scales
                    const uint8_t* blk = (m ? sd.W1 : sd.W0) + sd.L.block(f.e, f.mt, kt0 + s);
                    uint8_t* o = dst + m * (pq + pd);
                    ptx::bulk_g2s(o, blk + (size_t)f.r0 * 32, pq / 2, bar);
                    ptx::bulk_g2s(o + pq / 2, blk + (size_t)f.rows_mt * 32 + (size_t)f.r0 * 32, pq / 2, bar);
                    ptx::bulk_g2s(o + pq, blk + (size_t)f.rows_mt * kTileK + f.r0 * 4, pd, bar);
                }
            }
        }
        const int ns = kt1 - kt0;
        const uint32_t armed = ns >= 32 ? 0xffffffffu : ((1u << ns) - 1u);
        wait_par[b] = next_par[b];
        next_par[b] ^= armed;
    };

    const bool resident = a.nbuf == 2;
    const int step = gridDim.x;
    int it = blockIdx.x;
    if (resident) {
        if (it < n_items) { const GvItem f = item_of(it); issue(f, 0, 0, f.sd->L.kt_count); }
        if (it + step < n_items) { const GvItem f = item_of(it + step); issue(f, 1, 0, f.sd->L.kt_count); }
    }
    if (a.pdl_secondary) asm volatile("griddepcontrol.wait;" ::: "memory");

    bool ok = true;
    for (int i = 0; it < n_items && ok; ++i, it += step) {
        const int b = resident ? (i & 1) : 0;
        const GvItem f = item_of(it);
        const GemvSide& sd = *f.sd;
        const WLayout L = sd.L;
        const int R = sd.rows, KT = L.kt_count, NW = sd.kw / kTileK;
        const uint32_t pq = (uint32_t)R * kTileK, pd = (uint32_t)R * 4u;
        const uint32_t stage_bytes = (uint32_t)NMAT * (pq + pd);
        const int c = tid & 3, r = (tid >> 2) % R, ph = tid / (R * 4);
        const int P = kGvThreads / (R * 4);
        const int ntc = a.nt_cap;

        // slots of this expert (routed) or tokens (shared)
        int n_sl = a.n_tokens;
        if (!f.shared) {
            int cnt = 0;
            for (int q = tid; q < S; q += kGvThreads) cnt += (__ldg(a.ids + q) == f.e);
            cnt = __reduce_add_sync(0xffffffffu, cnt);
            if (lane == 0) misc[warp] = cnt;
            __syncthreads();
            n_sl = 0;
            for (int w = 0; w < kGvThreads / 32; ++w) n_sl += misc[w];
            __syncthreads();
        }
        for (int g0 = 0; g0 < n_sl && ok; g0 += ntc) {
            const int nt = min(ntc, n_sl - g0);
            if (f.shared) {
                if (tid < nt) rows_sh[tid] = g0 + tid;
            } else {
                int base = 0;
                for (int q0 = 0; q0 < S; q0 += kGvThreads) {
                    const int q = q0 + tid;
                    const bool hit = q < S && __ldg(a.ids + q) == f.e;
                    const unsigned bal = __ballot_sync(0xffffffffu, hit);
                    if (lane == 0) misc[warp] = __popc(bal);
                    __syncthreads();
                    int before = base;
                    for (int w = 0; w < warp; ++w) before += misc[w];
                    const int rank = before + __popc(bal & ((1u << lane) - 1u));
                    if (hit && rank >= g0 && rank < g0 + nt) rows_sh[rank - g0] = q;
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
                for (int q = 0; q < kGvNT; ++q) acc[m][q] = 0.f;

            for (int kt0 = 0; kt0 < KT && ok; kt0 += NW) {
                const int kt1 = min(KT, kt0 + NW);
                __syncthreads();  // previous window's stages and activations are free
                if (!resident) issue(f, b, kt0, kt1);
                const int cols = (kt1 - kt0) * kTileK;
                if (XB == 2) {
                    const uint16_t* xg = (const uint16_t*)sd.x;
                    for (int idx = tid; idx < nt * cols / 8; idx += kGvThreads) {
                        const int q = idx / (cols / 8), c8 = (idx % (cols / 8)) * 8, col = kt0 * kTileK + c8;
                        const int row = f.shared ? rows_sh[q] : (sd.x_per_slot ? rows_sh[q] : rows_sh[q] / a.k);
                        uint4 v = make_uint4(0, 0, 0, 0);
                        if (col < L.n_in) v = __ldg((const uint4*)(xg + (size_t)row * L.n_in + col));
                        *(uint4*)(sx + ((size_t)q * sd.kw + c8) * 2) = v;
                    }
                } else {
                    const float* xg = (const float*)sd.x;
                    for (int idx = tid; idx < nt * cols / 4; idx += kGvThreads) {
                        const int q = idx / (cols / 4), c4 = (idx % (cols / 4)) * 4, col = kt0 * kTileK + c4;
                        const int row = f.shared ? rows_sh[q] : (sd.x_per_slot ? rows_sh[q] : rows_sh[q] / a.k);
                        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (col < L.n_in) v = __ldg((const float4*)(xg + (size_t)row * L.n_in + col));
                        *(float4*)(sx + ((size_t)q * sd.kw + c4) * 4) = v;
                    }
                }
                __syncthreads();
                for (int kt = kt0 + ph; kt < kt1; kt += P) {
                    const int s = kt - kt0;
                    if (!gv_wait(&bars[b * a.max_stages + s], (wait_par[b] >> s) & 1u, status)) { ok = false; break; }
                    const uint8_t* st = sbuf[b] + (size_t)s * stage_bytes;
                    float w[NMAT][16];
#pragma unroll
                    for (int m = 0; m < NMAT; ++m) {
                        const uint8_t* pm = st + m * (pq + pd);
                        const uint4 qv = *(const uint4*)(pm + (c >> 1) * (pq / 2) + r * 32 + (c & 1) * 16);
                        const float d = __half2float(*(const __half*)(pm + pq + r * 4 + (c >> 1) * 2));
                        const float nd = -32896.0f * d;
                        const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
                        for (int bb = 0; bb < 16; ++bb) w[m][bb] = fmaf(magic_byte(qw[bb >> 2], bb & 3), d, nd);
                    }
                    const int xc = s * kTileK + c * 16;
#pragma unroll
                    for (int q = 0; q < kGvNT; ++q) {
                        if (q < nt) {
                            float xv[16];
                            if (XB == 2) {
                                const uint4 u0 = *(const uint4*)(sx + ((size_t)q * sd.kw + xc) * 2);
                                const uint4 u1 = *(const uint4*)(sx + ((size_t)q * sd.kw + xc + 8) * 2);
                                const uint32_t uw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                                for (int bb = 0; bb < 8; ++bb) {
                                    xv[2 * bb] = ld_x16(uw[bb] & 0xffffu, sd.x_type);
                                    xv[2 * bb + 1] = ld_x16(uw[bb] >> 16, sd.x_type);
                                }
                            } else {
#pragma unroll
                                for (int bb = 0; bb < 16; bb += 4) {
                                    const float4 vv = *(const float4*)(sx + ((size_t)q * sd.kw + xc + bb) * 4);
                                    xv[bb] = vv.x; xv[bb + 1] = vv.y; xv[bb + 2] = vv.z; xv[bb + 3] = vv.w;
                                }
                            }
#pragma unroll
                            for (int m = 0; m < NMAT; ++m) {
                                float t = 0.f;
#pragma unroll
                                for (int bb = 0; bb < 16; ++bb) t = fmaf(w[m][bb], xv[bb], t);
                                acc[m][q] += t;
                            }
                        }
                    }
                }
                // every thread leaves a timed-out wait the same way (no divergent barriers)
                ok = __syncthreads_and(ok) != 0;
            }
            // reduce: the 4 chunk lanes by a fixed butterfly, then the k phases in order
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int q = 0; q < kGvNT; ++q) {
                    float v = acc[m][q];
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    acc[m][q] = v;
                }
            if (c == 0)
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
#pragma unroll
                    for (int q = 0; q < kGvNT; ++q)
                        if (q < ntc) red[((ph * R + r) * ntc + q) * NMAT + m] = acc[m][q];
            __syncthreads();
            for (int idx = tid; idx < R * ntc; idx += kGvThreads) {
                const int row = idx / ntc, q = idx % ntc;
                const int n = f.mt * kTileM + f.r0 + row;
                if (q < nt && n < L.n_out) {
                    float v[NMAT];
#pragma unroll
                    for (int m = 0; m < NMAT; ++m) {
                        v[m] = 0.f;
                        for (int p2 = 0; p2 < P; ++p2) v[m] += red[((p2 * R + row) * ntc + q) * NMAT + m];
                    }
                    const int64_t orow = rows_sh[q];
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
        __syncthreads();  // this item's buffer is free
        if (resident && it + 2 * step < n_items) {
            const GvItem nf = item_of(it + 2 * step);
            issue(nf, b, 0, nf.sd->L.kt_count);
        }
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
        if (cudaFuncSetAttribute(gemv_kernel<DUAL, XB>, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024) !=
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

static int gv_sm_count() {
    static int dev_cached = -1, n = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != dev_cached) {
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        dev_cached = dev;
    }
    return n > 0 ? n : 148;
}

moe_status launch_gemv(const GemvArgs& in, cudaStream_t stream) {
    GemvArgs a = in;
    const int64_t items_max = (int64_t)a.max_distinct * a.routed.items + (a.has_shared ? a.shared.items : 0);
    if (items_max == 0) return MOE_OK;
    const bool f32 = a.routed.x_type == MOE_F32 || (a.has_shared && a.shared.x_type == MOE_F32);
    if (f32 && a.has_shared && a.routed.x_type != a.shared.x_type) return MOE_ERR_UNSUPPORTED;
    const int nmat = a.dual + 1;
    const int xb = f32 ? 4 : 2;
    a.nt_cap = a.n_tokens < kGvNT ? (a.n_tokens > 0 ? a.n_tokens : 1) : kGvNT;
    const GemvSide* sides[2] = {&a.routed, a.has_shared ? &a.shared : nullptr};
    uint32_t buf = 0, red = 0;
    int kw = 0, max_stages = 0;
    bool resident = true;
    for (const GemvSide* s : sides) {
        if (!s) continue;
        const uint32_t b = (uint32_t)s->n_stages * nmat * s->rows * kRowBytes;
        const int P = kGvThreads / (s->rows * 4);
        const uint32_t rb = (uint32_t)P * s->rows * a.nt_cap * nmat * 4;
        if (b > buf) buf = b;
        if (rb > red) red = rb;
        if (s->kw > kw) kw = s->kw;
        if (s->n_stages > max_stages) max_stages = s->n_stages;
        if (s->L.kt_count > s->kw / kTileK) resident = false;
    }
    a.buf_bytes = buf;
    a.red_bytes = red;
    a.x_bytes = (uint32_t)a.nt_cap * kw * xb;
    a.bm_words = (uint32_t)((a.n_experts + 31) / 32);
    a.max_stages = max_stages;
    a.nbuf = resident ? 2 : 1;
    size_t smem = gv_lay(a).total;
    if (smem > 200 * 1024) {
        a.nbuf = 1;
        smem = gv_lay(a).total;
    }
    const int per_sm = (int)((228 * 1024) / (smem + 1024)) > 0 ? (int)((228 * 1024) / (smem + 1024)) : 1;
    int64_t grid = (int64_t)gv_sm_count() * per_sm;
    if (grid > items_max) grid = items_max;
    if (a.dual)
        return f32 ? launch_t<1, 4>(a, smem, (unsigned)grid, stream) : launch_t<1, 2>(a, smem, (unsigned)grid, stream);
    return f32 ? launch_t<0, 4>(a, smem, (unsigned)grid, stream) : launch_t<0, 2>(a, smem, (unsigned)grid, stream);
}

}  // namespace moe
