// A tensor-core GEMM for the backward pass's two contractions (16-bit operands, fp32
// accumulation and output):
//
//   C[z][m * c_sm + n * c_sn] = sum_{r < R} sum_{k < K} A_zr[m][k] * B_zr[n][k]
//
// Both operands are K-major 16-bit row-major arrays read by TMA (128-byte swizzle):
// A_zr's row m is row a_row0 + z * a_row_z + r * a_row_r + m of the A tensor map, B's
// likewise; K runs along the rows (the tensor maps' column extent ends the reduction,
// reading zeros past it).  One CTA per 128 x NT output tile and z: a TMA warp feeds a
// ring of stages, one thread issues tcgen05.mma (M = 128, N = NT, K = 16, both operands
// from shared memory) into a tensor-memory accumulator, four warps drain it (lanes =
// consecutive m, so with c_sm = 1 each warp store covers 128 contiguous bytes).
#include <string.h>

#include "common.cuh"
#include "sampler.cuh"
#include "sm100.cuh"

namespace dcn1d {

namespace {

constexpr int kGM = 128;                  // tile rows = TMEM lanes
constexpr int kGBK = 64;                  // reduction elements per stage (128 bytes)
constexpr int kGStages = 4;
constexpr int kGTma = 0, kGMma = 1;       // warps 2..5 drain
constexpr int kGThreads = 6 * 32;
constexpr uint64_t kGWaitNs = 2000000000ull;

struct GemmTcArgs {
    int M, N, K, R, NT;
    int tiles_m, tiles_n;
    int a_row0, a_row_z, a_row_r;
    int b_row0, b_row_z, b_row_r;
    float *C;
    int64_t c_sm, c_sn, c_sz;
    uint32_t a_bytes, b_bytes;            // one stage's A and B tiles
    unsigned int *status;
};

template <class E>
struct GElem;
template <>
struct GElem<__nv_bfloat16> {
    static __host__ __device__ constexpr uint32_t idesc(int M, int N) { return idesc_bf16_f32(M, N); }
};
template <>
struct GElem<__half> {
    static __host__ __device__ constexpr uint32_t idesc(int M, int N) { return idesc_f16_f32(M, N); }
};

template <class E>
__global__ void __launch_bounds__(kGThreads, 1)
    gemm_tc_kernel(const __grid_constant__ GemmTcArgs G, const __grid_constant__ CUtensorMap amap,
                   const __grid_constant__ CUtensorMap bmap) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int tile = blockIdx.x;
    const int tn = tile % G.tiles_n;
    const int tm = (tile / G.tiles_n) % G.tiles_m;
    const int z = tile / (G.tiles_n * G.tiles_m);
    const int m0 = tm * kGM, n0 = tn * G.NT;

    const uint32_t sraw = smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - sraw);
    const uint32_t a_s0 = sbase;
    const uint32_t b_s0 = sbase + kGStages * G.a_bytes;
    const uint32_t bar0 = b_s0 + kGStages * G.b_bytes;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (kGStages + s); };
    const uint32_t dfull = bar0 + 8u * (2 * kGStages);
    uint32_t *tmem_holder =
        reinterpret_cast<uint32_t *>(smem + (bar0 - sbase) + 8 * (2 * kGStages + 2));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(dfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kGMma) {
        tmem_alloc(smem_u32(tmem_holder), 256);
        tc_fence_before();
    }
    if (warp == kGTma && lane == 0) {
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&bmap);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const BoundedWait wait{abort_flag, kGWaitNs, G.status};
    const int nkb = (G.K + kGBK - 1) / kGBK;
    const int total = nkb * G.R;

    if (warp == kGTma) {
        if (lane == 0) {
            int it = 0;
            for (; it < total; ++it) {
                const int r = it / nkb, kb = it - r * nkb;
                const int s = it % kGStages;
                const uint32_t ph = (uint32_t)(it / kGStages) & 1u;
                if (!wait(empty(s), ph ^ 1u))
                    break;
                mbar_arrive_expect_tx(full(s), G.a_bytes + G.b_bytes);
                tma_load_2d(a_s0 + s * G.a_bytes, &amap, kb * kGBK,
                            G.a_row0 + z * G.a_row_z + r * G.a_row_r + m0, full(s));
                tma_load_2d(b_s0 + s * G.b_bytes, &bmap, kb * kGBK,
                            G.b_row0 + z * G.b_row_z + r * G.b_row_r + n0, full(s));
            }
            volatile int never = 0;
            const BoundedWait drain{&never, kGWaitNs, G.status};
            for (int j = (it > kGStages ? it - kGStages : 0); j < it; ++j)
                drain(full(j % kGStages), (uint32_t)(j / kGStages) & 1u);
        }
    } else if (warp == kGMma) {
        if (lane == 0) {
            const uint32_t idesc = GElem<E>::idesc(kGM, G.NT);
            for (int it = 0; it < total; ++it) {
                const int s = it % kGStages;
                if (!wait(full(s), (uint32_t)(it / kGStages) & 1u))
                    break;
                tc_fence_after();
                const uint32_t as = a_s0 + s * G.a_bytes, bs = b_s0 + s * G.b_bytes;
#pragma unroll
                for (int kk = 0; kk < kGBK / 16; ++kk)
                    mma_f16_ss(tmem, sw128_kmajor_desc(as + 32u * kk),
                               sw128_kmajor_desc(bs + 32u * kk), idesc,
                               (it > 0 || kk > 0) ? 1u : 0u);
                mma_commit(empty(s));
            }
            mma_commit(dfull);       // also the drain point: every MMA issued is complete
            volatile int never = 0;
            const BoundedWait drain{&never, kGWaitNs, G.status};
            drain(dfull, 0);
        }
    } else {
        // drain: warp w reads TMEM lanes 32 (w % 4) ..
        const int q = warp % 4;
        const int m = m0 + 32 * q + lane;
        if (__all_sync(0xffffffffu, wait(dfull, 0))) {
            tc_fence_after();
            float *Cz = G.C + (int64_t)z * G.c_sz;
            for (int c = 0; c < G.NT; c += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c, v);
                tmem_wait_ld();
                if (m < G.M) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int n = n0 + c + i;
                        if (n < G.N)
                            Cz[(int64_t)m * G.c_sm + (int64_t)n * G.c_sn] = __uint_as_float(v[i]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kGMma) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ---------------------------------------------------------------------------------
// The backward's column-gradient GEMM with the sampling gradient as its drain.
//
// Per (b, conv group g) and tile of 128 positions l x NT columns n = (c, k) of the
// group's reduction index: D[l][n] = sum_co grad_out[b, g*cout_g + co, l] * W[g*cout_g +
// co][n] (the gradient of the sampled column), exactly the GEMM above.  Instead of storing
// D, sixteen drain warps (four per lane quarter, taking the tile's channels round robin)
// form, per channel and tap, the sampled value v = (1-f) x[i0] + f x[i0+1] and with
// dv = D[l][n]:
//   grad_x[b, ci, i0] += m (1-f) dv,  grad_x[b, ci, i0+1] += m f dv   (in range only),
//   grad_offsets[b, og, l, k] += m (x[i0+1] - x[i0]) dv  (inside the clamp's range),
//   grad_mask[b, og, l, k] += v dv,
// and the sampled column m v in the 16-bit type for the weight gradient (cols16).  The
// column gradients never reach global memory.

constexpr int kSThreads = 18 * 32;   // TMA, MMA, 16 drain warps
constexpr int kSStages = 4;

struct GemmSampleArgs {
    int M, N, K, NT, tiles_m, tiles_n;   // M = L_out, N = Kg, K = cout_g
    int a_row_z;                          // A rows per batch (L_out)
    uint32_t a_bytes, b_bytes;
    unsigned int *status;
    const void *x, *off, *mask;           // the forward's inputs (element type E)
    void *cols16;                         // E [B][C_in * K][L_out] or NULL
    float *gx, *goff, *gmask;             // fp32 accumulators or NULL
    int C_in, L_in, L_out, stride, padding, dilation, offset_groups, cin_per_og, cin_g, g;
    int unconstrained;
};

template <class E, int KT, bool MASK>
__global__ void __launch_bounds__(kSThreads, 1)
    gemm_sample_kernel(const __grid_constant__ GemmSampleArgs G,
                       const __grid_constant__ CUtensorMap amap,
                       const __grid_constant__ CUtensorMap bmap) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int tile = blockIdx.x;
    const int tn = tile % G.tiles_n;
    const int tm = (tile / G.tiles_n) % G.tiles_m;
    const int b = tile / (G.tiles_n * G.tiles_m);
    const int m0 = tm * kGM, n0 = tn * G.NT;

    const uint32_t sraw = smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - sraw);
    const uint32_t a_s0 = sbase;
    const uint32_t b_s0 = sbase + kSStages * G.a_bytes;
    const uint32_t bar0 = b_s0 + kSStages * G.b_bytes;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (kSStages + s); };
    const uint32_t dfull = bar0 + 8u * (2 * kSStages);
    uint32_t *tmem_holder =
        reinterpret_cast<uint32_t *>(smem + (bar0 - sbase) + 8 * (2 * kSStages + 2));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSStages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(dfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kGMma) {
        tmem_alloc(smem_u32(tmem_holder), 256);
        tc_fence_before();
    }
    if (warp == kGTma && lane == 0) {
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&bmap);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const BoundedWait wait{abort_flag, kGWaitNs, G.status};
    const int nkb = (G.K + kGBK - 1) / kGBK;

    if (warp == kGTma) {
        if (lane == 0) {
            int it = 0;
            for (; it < nkb; ++it) {
                const int s = it % kSStages;
                const uint32_t ph = (uint32_t)(it / kSStages) & 1u;
                if (!wait(empty(s), ph ^ 1u))
                    break;
                mbar_arrive_expect_tx(full(s), G.a_bytes + G.b_bytes);
                tma_load_2d(a_s0 + s * G.a_bytes, &amap, it * kGBK, b * G.a_row_z + m0, full(s));
                tma_load_2d(b_s0 + s * G.b_bytes, &bmap, it * kGBK, n0, full(s));
            }
            volatile int never = 0;
            const BoundedWait drain{&never, kGWaitNs, G.status};
            for (int j = (it > kSStages ? it - kSStages : 0); j < it; ++j)
                drain(full(j % kSStages), (uint32_t)(j / kSStages) & 1u);
        }
    } else if (warp == kGMma) {
        if (lane == 0) {
            const uint32_t idesc = GElem<E>::idesc(kGM, G.NT);
            for (int it = 0; it < nkb; ++it) {
                const int s = it % kSStages;
                if (!wait(full(s), (uint32_t)(it / kSStages) & 1u))
                    break;
                tc_fence_after();
                const uint32_t as = a_s0 + s * G.a_bytes, bs = b_s0 + s * G.b_bytes;
#pragma unroll
                for (int kk = 0; kk < kGBK / 16; ++kk)
                    mma_f16_ss(tmem, sw128_kmajor_desc(as + 32u * kk),
                               sw128_kmajor_desc(bs + 32u * kk), idesc,
                               (it > 0 || kk > 0) ? 1u : 0u);
                mma_commit(empty(s));
            }
            mma_commit(dfull);       // also the drain point: every MMA issued is complete
            volatile int never = 0;
            const BoundedWait drain{&never, kGWaitNs, G.status};
            drain(dfull, 0);
        }
    } else {
        // ---------------------------------------------------------------- sampling drain
        const int q = warp % 4;              // TMEM lane quarter
        const int hq = (warp - 2) / 4;       // this warp's share of the tile's channels
        const int l = m0 + 32 * q + lane;
        const bool valid = l < G.L_out;
        const int start = l * G.stride - G.padding;
        const int span = G.dilation * (KT - 1);
        const uint32_t lanebase = tmem + ((uint32_t)(32 * q) << 16);
        const int n_end = min(n0 + G.NT, G.N);            // columns of this tile
        const int c_lo = n0 / KT, c_hi = (n_end - 1) / KT;  // channels they touch
        // (accumulating grad_x in a shared-memory window over the tile's receptive fields
        // measured slower than the global atomics: 876 against 549 us a launch)
        if (__all_sync(0xffffffffu, wait(dfull, 0))) {
            tc_fence_after();
            // the taps of this row in offset group og_cur, and their gradient sums
            int og_cur = -1;
            int i0[KT];
            float fr[KT], mk[KT], s_off[KT], s_mask[KT];
            bool gate[KT];
            auto flush = [&]() {
                if (og_cur < 0 || !valid)
                    return;
                const int64_t obase =
                    (((int64_t)b * G.offset_groups + og_cur) * G.L_out + l) * KT;
#pragma unroll
                for (int k = 0; k < KT; ++k) {
                    if (G.goff && gate[k])
                        atomicAdd(G.goff + obase + k, s_off[k]);
                    if (G.gmask)
                        atomicAdd(G.gmask + obase + k, s_mask[k]);
                }
            };
            for (int cr = c_lo + hq; cr <= c_hi; cr += 4) {
                __syncwarp();   // the tensor-memory loads below are warp-collective
                const int ci = G.g * G.cin_g + cr;
                const int og = ci / G.cin_per_og;
                if (og != og_cur) {
                    flush();
                    og_cur = og;
                    const int64_t obase =
                        (((int64_t)b * G.offset_groups + og) * G.L_out + (valid ? l : 0)) * KT;
#pragma unroll
                    for (int k = 0; k < KT; ++k) {
                        const float offv = ld_f32(static_cast<const E *>(G.off) + obase + k);
                        mk[k] = MASK ? ld_f32(static_cast<const E *>(G.mask) + obase + k) : 1.0f;
                        const float raw = __fadd_rn(__int2float_rn(start + k * G.dilation), offv);
                        gate[k] = G.unconstrained ||
                                  (raw >= __int2float_rn(start) &&
                                   raw <= __int2float_rn(start + span));
                        const Tap t = sample_tap(start, k, G.dilation, span, offv,
                                                 G.unconstrained != 0);
                        i0[k] = t.i0;
                        fr[k] = t.f;
                        s_off[k] = 0.0f;
                        s_mask[k] = 0.0f;
                    }
                }
                // this channel's neighbours first (their loads overlap the tensor-memory
                // loads), then its columns of the tile (a channel may straddle two tiles)
                const E *row = static_cast<const E *>(G.x) + ((int64_t)b * G.C_in + ci) * G.L_in;
                float x0[KT], x1[KT];
#pragma unroll
                for (int k = 0; k < KT; ++k) {
                    const int ia = i0[k];
                    x0[k] = (valid && ia >= 0 && ia < G.L_in) ? ld_f32(row + ia) : 0.0f;
                    x1[k] = (valid && ia >= -1 && ia < G.L_in - 1) ? ld_f32(row + ia + 1) : 0.0f;
                }
                float dv[KT];
#pragma unroll
                for (int k = 0; k < KT; ++k) {
                    const int n = cr * KT + k;
                    dv[k] = (n >= n0 && n < n_end)
                                ? __uint_as_float(tmem_ld1(lanebase + (uint32_t)(n - n0)))
                                : 0.0f;
                }
                tmem_wait_ld();
                if (valid) {
                    float *gxr = G.gx ? G.gx + ((int64_t)b * G.C_in + ci) * G.L_in : nullptr;
#pragma unroll
                    for (int k = 0; k < KT; ++k) {
                        const int n = cr * KT + k;
                        if (n < n0 || n >= n_end)
                            continue;
                        const int ia = i0[k];
                        const float f = fr[k], m = mk[k];
                        const float v = __fadd_rn(__fmul_rn(__fsub_rn(1.0f, f), x0[k]),
                                                  __fmul_rn(f, x1[k]));
                        if (G.cols16)
                            static_cast<E *>(G.cols16)[(((int64_t)b * G.C_in + ci) * KT + k) *
                                                           G.L_out + l] =
                                from_f32<E>(__fmul_rn(m, v));
                        const float d = dv[k];
                        if (gxr) {
                            if (ia >= 0 && ia < G.L_in)
                                atomicAdd(gxr + ia, __fmul_rn(__fmul_rn(m, __fsub_rn(1.0f, f)), d));
                            if (ia >= -1 && ia < G.L_in - 1)
                                atomicAdd(gxr + ia + 1, __fmul_rn(__fmul_rn(m, f), d));
                        }
                        s_off[k] = __fmaf_rn(__fmul_rn(m, __fsub_rn(x1[k], x0[k])), d, s_off[k]);
                        s_mask[k] = __fmaf_rn(v, d, s_mask[k]);
                    }
                }
            }
            flush();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kGMma) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ---------------------------------------------------------------------------------
// The same GEMM for fp32 operands, accurate to fp32 through three TF32 products: each
// operand v is split exactly into hi (v with its low 13 mantissa bits cleared; the tf32
// MMA reads an fp32 container that way) and lo = v - hi, and the MMA accumulates
// hi*hi + hi*lo + lo*hi.  TMA loads the fp32 tiles (32 elements = 128 bytes a row); while
// the MMA works, the four drain warps write each stage's lo tiles next to them.
//
// Rows: with `flat`, the M rows of A and C run over z as well (row m of the whole problem
// is row m of A; its output lands at C[(m / rpz) * c_sz + (m % rpz) * c_sm + n * c_sn]),
// so short per-z row counts still fill 128-row tiles.

constexpr int kXBK = 32;                 // fp32 reduction elements per stage
constexpr int kXStages = 2;
constexpr int kXThreads = 6 * 32;        // TMA, MMA, 4 lo-formers / drain

struct GemmX3Args {
    int M, N, K, R, NT;
    int tiles_m, tiles_n;
    int a_row0, a_row_z, a_row_r;
    int b_row0, b_row_z, b_row_r;
    int flat, rpz;                       // flat rows: rpz rows per z
    float *C;
    int64_t c_sm, c_sn, c_sz;
    uint32_t a_bytes, b_bytes;           // one stage's A and B tiles (each also has a lo tile)
    unsigned int *status;
};

__device__ __forceinline__ uint4 lds_v4x(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts_v4x(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint32_t tf32_lo(uint32_t v) {
    return __float_as_uint(__fsub_rn(__uint_as_float(v), __uint_as_float(v & 0xFFFFE000u)));
}

__global__ void __launch_bounds__(kXThreads, 1)
    gemm_x3_kernel(const __grid_constant__ GemmX3Args G, const __grid_constant__ CUtensorMap amap,
                   const __grid_constant__ CUtensorMap bmap) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int tile = blockIdx.x;
    const int tn = tile % G.tiles_n;
    const int tm = (tile / G.tiles_n) % G.tiles_m;
    const int z = tile / (G.tiles_n * G.tiles_m);
    const int m0 = tm * kGM, n0 = tn * G.NT;

    const uint32_t sraw = smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - sraw);
    // stage s: A hi, A lo, B hi, B lo
    const uint32_t stage_bytes = 2 * (G.a_bytes + G.b_bytes);
    auto a_hi = [&](int s) { return sbase + (uint32_t)s * stage_bytes; };
    auto a_lo = [&](int s) { return a_hi(s) + G.a_bytes; };
    auto b_hi = [&](int s) { return a_hi(s) + 2 * G.a_bytes; };
    auto b_lo = [&](int s) { return b_hi(s) + G.b_bytes; };
    const uint32_t bar0 = sbase + kXStages * stage_bytes;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (kXStages + s); };
    auto lo_ready = [&](int s) { return bar0 + 8u * (2 * kXStages + s); };
    const uint32_t dfull = bar0 + 8u * (3 * kXStages);
    uint32_t *tmem_holder =
        reinterpret_cast<uint32_t *>(smem + (bar0 - sbase) + 8 * (3 * kXStages + 2));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kXStages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
            mbar_init(lo_ready(s), 4);
        }
        mbar_init(dfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kGMma) {
        tmem_alloc(smem_u32(tmem_holder), 256);
        tc_fence_before();
    }
    if (warp == kGTma && lane == 0) {
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&bmap);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const BoundedWait wait{abort_flag, kGWaitNs, G.status};
    const int nkb = (G.K + kXBK - 1) / kXBK;
    const int total = nkb * G.R;
    // A's first row: flat rows index the whole problem, else z's block
    const int a_row_base = G.flat ? m0 : G.a_row0 + z * G.a_row_z + m0;

    if (warp == kGTma) {
        if (lane == 0) {
            int it = 0;
            for (; it < total; ++it) {
                const int r = it / nkb, kb = it - r * nkb;
                const int s = it % kXStages;
                const uint32_t ph = (uint32_t)(it / kXStages) & 1u;
                if (!wait(empty(s), ph ^ 1u))
                    break;
                mbar_arrive_expect_tx(full(s), G.a_bytes + G.b_bytes);
                tma_load_2d(a_hi(s), &amap, kb * kXBK, a_row_base + r * G.a_row_r, full(s));
                tma_load_2d(b_hi(s), &bmap, kb * kXBK,
                            G.b_row0 + z * G.b_row_z + r * G.b_row_r + n0, full(s));
            }
            volatile int never = 0;
            const BoundedWait drain{&never, kGWaitNs, G.status};
            for (int j = (it > kXStages ? it - kXStages : 0); j < it; ++j)
                drain(full(j % kXStages), (uint32_t)(j / kXStages) & 1u);
        }
    } else if (warp == kGMma) {
        if (lane == 0) {
            const uint32_t idesc = idesc_tf32_ss_f32(kGM, G.NT);
            for (int it = 0; it < total; ++it) {
                const int s = it % kXStages;
                const uint32_t ph = (uint32_t)(it / kXStages) & 1u;
                if (!wait(full(s), ph) || !wait(lo_ready(s), ph))
                    break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kXBK / 8; ++kk) {   // 8 tf32 = 32 bytes a step
                    const uint32_t o = 32u * kk;
                    const uint64_t ah = sw128_kmajor_desc(a_hi(s) + o);
                    const uint64_t al = sw128_kmajor_desc(a_lo(s) + o);
                    const uint64_t bh = sw128_kmajor_desc(b_hi(s) + o);
                    const uint64_t bl = sw128_kmajor_desc(b_lo(s) + o);
                    mma_tf32_ss(tmem, ah, bh, idesc, (it > 0 || kk > 0) ? 1u : 0u);
                    mma_tf32_ss(tmem, ah, bl, idesc, 1u);
                    mma_tf32_ss(tmem, al, bh, idesc, 1u);
                }
                mma_commit(empty(s));
            }
            mma_commit(dfull);
            volatile int never = 0;
            const BoundedWait drain{&never, kGWaitNs, G.status};
            drain(dfull, 0);
        }
    } else {
        // ---- lo parts of every stage (elementwise, so the swizzle does not matter), then
        // the drain: warp w reads TMEM lanes 32 (w % 4) ..
        const int dt = threadIdx.x - 64;                  // 0 .. 127
        bool ok = true;
        for (int it = 0; it < total && ok; ++it) {
            const int s = it % kXStages;
            ok = __all_sync(0xffffffffu, wait(full(s), (uint32_t)(it / kXStages) & 1u));
            if (ok) {
                for (uint32_t o = 16u * dt; o < G.a_bytes; o += 16u * 128u) {
                    uint4 v = lds_v4x(a_hi(s) + o);
                    v = make_uint4(tf32_lo(v.x), tf32_lo(v.y), tf32_lo(v.z), tf32_lo(v.w));
                    sts_v4x(a_lo(s) + o, v);
                }
                for (uint32_t o = 16u * dt; o < G.b_bytes; o += 16u * 128u) {
                    uint4 v = lds_v4x(b_hi(s) + o);
                    v = make_uint4(tf32_lo(v.x), tf32_lo(v.y), tf32_lo(v.z), tf32_lo(v.w));
                    sts_v4x(b_lo(s) + o, v);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(lo_ready(s));
            }
        }
        const int q = warp % 4;
        const int m = m0 + 32 * q + lane;
        if (ok && __all_sync(0xffffffffu, wait(dfull, 0))) {
            tc_fence_after();
            float *Crow = nullptr;
            if (m < G.M) {
                const int zz = G.flat ? m / G.rpz : z;
                const int mm = G.flat ? m - zz * G.rpz : m;
                Crow = G.C + (int64_t)zz * G.c_sz + (int64_t)mm * G.c_sm;
            }
            for (int c = 0; c < G.NT; c += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c, v);
                tmem_wait_ld();
                if (Crow) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int n = n0 + c + i;
                        if (n < G.N)
                            Crow[(int64_t)n * G.c_sn] = __uint_as_float(v[i]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kGMma) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace

// The A and B operands as 16-bit row-major [rows][cols] arrays (row strides in
// elements, multiples of 8), the reduction over their first `K` columns.
bool gemm_tc_supported(int dtype, const void *A, int64_t a_rows, int64_t a_ld, const void *B,
                       int64_t b_rows, int64_t b_ld) {
    if (dtype != DCN1D_BF16 && dtype != DCN1D_F16)
        return false;
    if ((reinterpret_cast<uintptr_t>(A) & 15) || (reinterpret_cast<uintptr_t>(B) & 15))
        return false;
    if (a_ld % 8 || b_ld % 8 || a_rows < 1 || b_rows < 1 || a_rows >= (1LL << 31) ||
        b_rows >= (1LL << 31))
        return false;
    return true;
}

cudaError_t launch_gemm_tc(int dtype, const void *A, int64_t a_rows, int64_t a_ld, int a_row0,
                           int a_row_z, int a_row_r, const void *B, int64_t b_rows, int64_t b_ld,
                           int b_row0, int b_row_z, int b_row_r, int M, int N, int K, int R,
                           int nz, float *C, int64_t c_sm, int64_t c_sn, int64_t c_sz,
                           cudaStream_t stream) {
    GemmTcArgs G;
    memset(&G, 0, sizeof(G));
    G.M = M;
    G.N = N;
    G.K = K;
    G.R = R;
    G.NT = N <= 128 ? (N <= 64 ? 64 : 128) : 256;
    G.tiles_m = (M + kGM - 1) / kGM;
    G.tiles_n = (N + G.NT - 1) / G.NT;
    G.a_row0 = a_row0;
    G.a_row_z = a_row_z;
    G.a_row_r = a_row_r;
    G.b_row0 = b_row0;
    G.b_row_z = b_row_z;
    G.b_row_r = b_row_r;
    G.C = C;
    G.c_sm = c_sm;
    G.c_sn = c_sn;
    G.c_sz = c_sz;
    G.a_bytes = kGM * kGBK * 2;
    G.b_bytes = (uint32_t)G.NT * kGBK * 2;
    G.status = device_status_ptr();
    if (!G.status)
        return cudaErrorInvalidDevice;
    const int64_t blocks = (int64_t)G.tiles_m * G.tiles_n * nz;
    if (blocks < 1 || blocks >= (1LL << 31))
        return cudaErrorInvalidValue;
    const CUtensorMapDataType ty = dtype == DCN1D_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                      : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    alignas(64) CUtensorMap amap, bmap;
    // the maps' column extent is the reduction length: TMA reads zeros past it
    if (!encode_2d_ld(&amap, ty, A, (uint64_t)K, (uint64_t)a_rows, (uint64_t)a_ld, 2, kGBK, kGM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d_ld(&bmap, ty, B, (uint64_t)K, (uint64_t)b_rows, (uint64_t)b_ld, 2, kGBK,
                      (uint32_t)G.NT, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const size_t smem = (size_t)kGStages * (G.a_bytes + G.b_bytes) + 8 * (2 * kGStages + 2) + 16 +
                        1024;
    const void *kern = dtype == DCN1D_F16 ? reinterpret_cast<const void *>(gemm_tc_kernel<__half>)
                                          : reinterpret_cast<const void *>(
                                                gemm_tc_kernel<__nv_bfloat16>);
    cudaError_t e = ensure_smem(kern, (int)(smem < 116 * 1024 ? 116 * 1024 : smem));
    if (e != cudaSuccess)
        return e;
    const size_t smem_launch = smem < 116 * 1024 ? 116 * 1024 : smem;   // one CTA per SM
    if (dtype == DCN1D_F16)
        gemm_tc_kernel<__half><<<(unsigned)blocks, kGThreads, smem_launch, stream>>>(G, amap, bmap);
    else
        gemm_tc_kernel<__nv_bfloat16><<<(unsigned)blocks, kGThreads, smem_launch, stream>>>(G, amap,
                                                                                            bmap);
    return cudaGetLastError();
}

// fp32 operands: row strides (elements) multiples of 4, 16-byte aligned bases.
bool gemm_x3_supported(const void *A, int64_t a_ld, const void *B, int64_t b_ld) {
    return !(reinterpret_cast<uintptr_t>(A) & 15) && !(reinterpret_cast<uintptr_t>(B) & 15) &&
           a_ld % 4 == 0 && b_ld % 4 == 0;
}

cudaError_t launch_gemm_x3(const float *A, int64_t a_rows, int64_t a_ld, int a_row0,
                           int a_row_z, int a_row_r, const float *B, int64_t b_rows, int64_t b_ld,
                           int b_row0, int b_row_z, int b_row_r, int M, int N, int K, int R,
                           int nz, int flat_rpz, float *C, int64_t c_sm, int64_t c_sn,
                           int64_t c_sz, cudaStream_t stream) {
    if (!gemm_x3_supported(A, a_ld, B, b_ld) || a_rows < 1 || b_rows < 1 ||
        a_rows >= (1LL << 31) || b_rows >= (1LL << 31))
        return cudaErrorInvalidValue;
    GemmX3Args G;
    memset(&G, 0, sizeof(G));
    G.flat = flat_rpz > 0 ? 1 : 0;
    G.rpz = flat_rpz;
    G.M = G.flat ? M * nz : M;   // flat: the rows of every z in one range
    G.N = N;
    G.K = K;
    G.R = R;
    G.NT = N <= 128 ? (N <= 64 ? 64 : 128) : 256;
    G.tiles_m = (G.M + kGM - 1) / kGM;
    G.tiles_n = (N + G.NT - 1) / G.NT;
    G.a_row0 = a_row0;
    G.a_row_z = a_row_z;
    G.a_row_r = a_row_r;
    G.b_row0 = b_row0;
    G.b_row_z = b_row_z;
    G.b_row_r = b_row_r;
    G.C = C;
    G.c_sm = c_sm;
    G.c_sn = c_sn;
    G.c_sz = c_sz;
    G.a_bytes = kGM * kXBK * 4;
    G.b_bytes = (uint32_t)G.NT * kXBK * 4;
    G.status = device_status_ptr();
    if (!G.status)
        return cudaErrorInvalidDevice;
    const int64_t blocks = (int64_t)G.tiles_m * G.tiles_n * (G.flat ? 1 : nz);
    if (blocks < 1 || blocks >= (1LL << 31))
        return cudaErrorInvalidValue;
    alignas(64) CUtensorMap amap, bmap;
    if (!encode_2d_ld(&amap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, A, (uint64_t)K, (uint64_t)a_rows,
                      (uint64_t)a_ld, 4, kXBK, kGM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d_ld(&bmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, B, (uint64_t)K, (uint64_t)b_rows,
                      (uint64_t)b_ld, 4, kXBK, (uint32_t)G.NT, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const size_t smem = (size_t)kXStages * 2 * (G.a_bytes + G.b_bytes) +
                        8 * (3 * kXStages + 2) + 16 + 1024;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(gemm_x3_kernel),
                                (int)(smem < 116 * 1024 ? 116 * 1024 : smem));
    if (e != cudaSuccess)
        return e;
    gemm_x3_kernel<<<(unsigned)blocks, kXThreads, smem < 116 * 1024 ? 116 * 1024 : smem,
                     stream>>>(G, amap, bmap);
    return cudaGetLastError();
}

bool gemm_sample_supported(const Problem &P) {
    return P.K == 3 || P.K == 4 || P.K == 5 || P.K == 7 || P.K == 9;
}

namespace {
template <class E, int KT, bool MASK>
cudaError_t launch_gs(const GemmSampleArgs &G, const CUtensorMap &amap, const CUtensorMap &bmap,
                      unsigned blocks, size_t smem, cudaStream_t stream) {
    auto kern = gemm_sample_kernel<E, KT, MASK>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), (int)smem);
    if (e != cudaSuccess)
        return e;
    kern<<<blocks, kSThreads, smem, stream>>>(G, amap, bmap);
    return cudaGetLastError();
}

template <class E, int KT>
cudaError_t launch_gs_k(const GemmSampleArgs &G, bool mask, const CUtensorMap &amap,
                        const CUtensorMap &bmap, unsigned blocks, size_t smem,
                        cudaStream_t stream) {
    return mask ? launch_gs<E, KT, true>(G, amap, bmap, blocks, smem, stream)
                : launch_gs<E, KT, false>(G, amap, bmap, blocks, smem, stream);
}

template <class E>
cudaError_t launch_gs_e(const GemmSampleArgs &G, int K, bool mask, const CUtensorMap &amap,
                        const CUtensorMap &bmap, unsigned blocks, size_t smem,
                        cudaStream_t stream) {
    switch (K) {
    case 3: return launch_gs_k<E, 3>(G, mask, amap, bmap, blocks, smem, stream);
    case 4: return launch_gs_k<E, 4>(G, mask, amap, bmap, blocks, smem, stream);
    case 5: return launch_gs_k<E, 5>(G, mask, amap, bmap, blocks, smem, stream);
    case 7: return launch_gs_k<E, 7>(G, mask, amap, bmap, blocks, smem, stream);
    case 9: return launch_gs_k<E, 9>(G, mask, amap, bmap, blocks, smem, stream);
    default: return cudaErrorInvalidValue;
    }
}
}  // namespace

// Conv group g of the backward: A = grad_out transposed ([B * L_out][C_out], this group's
// columns at goutT_g), B = W transposed ([Kg][cout_g] at wT_g); see gemm_sample_kernel.
cudaError_t launch_gemm_sample(const Problem &P, int g, const void *goutT_g, const void *wT_g,
                               void *cols16, float *gx, float *goff, float *gmask,
                               cudaStream_t stream) {
    if (!gemm_sample_supported(P))
        return cudaErrorInvalidValue;
    GemmSampleArgs G;
    memset(&G, 0, sizeof(G));
    const int Kg = P.cin_g * P.K;
    G.M = P.L_out;
    G.N = Kg;
    G.K = P.cout_g;
    G.NT = Kg <= 128 ? (Kg <= 64 ? 64 : 128) : 256;
    G.tiles_m = (G.M + kGM - 1) / kGM;
    G.tiles_n = (G.N + G.NT - 1) / G.NT;
    G.a_row_z = P.L_out;
    G.a_bytes = kGM * kGBK * 2;
    G.b_bytes = (uint32_t)G.NT * kGBK * 2;
    G.status = device_status_ptr();
    if (!G.status)
        return cudaErrorInvalidDevice;
    G.x = P.x;
    G.off = P.off;
    G.mask = P.mask;
    G.cols16 = cols16;
    G.gx = gx;
    G.goff = goff;
    G.gmask = gmask;
    G.C_in = P.C_in;
    G.L_in = P.L_in;
    G.L_out = P.L_out;
    G.stride = P.stride;
    G.padding = P.padding;
    G.dilation = P.dilation;
    G.offset_groups = P.offset_groups;
    G.cin_per_og = P.cin_per_og;
    G.cin_g = P.cin_g;
    G.g = g;
    G.unconstrained = P.unconstrained;
    const int64_t blocks = (int64_t)G.tiles_m * G.tiles_n * P.B;
    if (blocks < 1 || blocks >= (1LL << 31))
        return cudaErrorInvalidValue;
    const CUtensorMapDataType ty = P.dtype == DCN1D_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                        : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    alignas(64) CUtensorMap amap, bmap;
    if (!encode_2d_ld(&amap, ty, goutT_g, (uint64_t)P.cout_g, (uint64_t)P.B * P.L_out,
                      (uint64_t)P.C_out, 2, kGBK, kGM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d_ld(&bmap, ty, wT_g, (uint64_t)P.cout_g, (uint64_t)Kg, (uint64_t)P.cout_g, 2,
                      kGBK, (uint32_t)G.NT, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const size_t smem = (size_t)kSStages * (G.a_bytes + G.b_bytes) + 8 * (2 * kSStages + 2) + 16 +
                        1024;
    const size_t smem_launch = smem < 116 * 1024 ? 116 * 1024 : smem;   // one CTA per SM
    return P.dtype == DCN1D_F16
               ? launch_gs_e<__half>(G, P.K, P.mask != nullptr, amap, bmap, (unsigned)blocks,
                                     smem_launch, stream)
               : launch_gs_e<__nv_bfloat16>(G, P.K, P.mask != nullptr, amap, bmap,
                                            (unsigned)blocks, smem_launch, stream);
}

}  // namespace dcn1d
