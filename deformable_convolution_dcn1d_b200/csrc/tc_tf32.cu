// Fused deformable-im2col + tcgen05 tensor-core contraction for fp32 inputs,
// accurate to fp32 through three TF32 products ("3xTF32").
//
// Same GEMM as the bf16 kernel (see tc_bf16.cu): per conv group and block of N
// output channels, D[n, co] = sum_kk cols[n, kk] * W[co, kk] over kk = (ci, k).
// TF32 keeps 10 mantissa bits, so every fp32 operand v is split exactly into
// hi = v with its low 13 mantissa bits cleared (a tf32 value) and lo = v - hi,
// and the MMA accumulates hi*hi + hi*lo + lo*hi in fp32; the dropped lo*lo
// term is about 2^-22 of the product.
//
// One launch, no workspace:
//  * the bf16 kernel's roles: a TMA warp loads the W tile (128-byte swizzle) and
//    the fp32 x window of each 32-wide k-block; W itself serves as W_hi, since the
//    tf32 MMA ignores the low 13 mantissa bits of an fp32 operand.  The 8 producer
//    warps that consume a stage first write W_lo = W - W_hi of an eighth of its W
//    tile next to it (a second shared-memory tile, read by the MMA), then
//    interpolate 16 columns each in fp32 and write their hi and lo parts straight
//    into tensor memory (A operand); one thread issues 3 tcgen05.mma kind::tf32 per
//    8-wide k step; the producers drain D.
//  * Small-N, large-K problems are split along the reduction (split-K) across the
//    CTAs of a thread-block cluster, one split per CTA.  When every split's D is
//    complete, each CTA sends 16-column chunks of it through distributed shared
//    memory to the chunk's owner CTA (its stage memory, free by then), which adds the
//    splits in rank order plus the bias and stores the outputs -- deterministic,
//    and the same sums in the same order as adding per-split partial tensors.
#include <string.h>

#include "common.cuh"
#include "sampler.cuh"
#include "sm100.cuh"

namespace dcn1d {

namespace {

constexpr int kStages = 3;
constexpr int kRows = 128;         // output positions per tile = TMEM lanes
constexpr int kBK = 32;            // reduction elements per k-block (one 128-byte fp32 row)
constexpr int kSeg = 16;           // reduction elements per producer warp and k-block
constexpr int kBox = 256;          // x window box width (positions)
constexpr int kBoxStep = 248;      // second box starts here (8 positions of overlap)
constexpr int kWinMax = 503;
constexpr int kRowBytes = kBox * 4;
constexpr int kProdWarps = 16;
constexpr int kTmaWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kThreads = 18 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColD = 0;      // D: columns [0, N)
constexpr uint32_t kColA = 256;    // A stage s: hi [256 + 64 s, +32), lo [256 + 64 s + 32, +32)
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kTf32Mask = 0xFFFFE000u;

constexpr int kMaxSplits = 8;      // portable cluster size

struct TfArgs {
    Problem P;
    int N;              // MMA N = output channels per block (multiple of 32, <= 256)
    int n_cob;          // channel blocks per conv group
    int num_kb;         // k-blocks of the whole reduction
    int kb_per_split;   // k-blocks per split
    int splits;         // > 1: cluster launch, one split per CTA of a cluster
    int n_own;          // 16-column chunks of a tile each cluster CTA owns (at most)
    int flat;           // 1: tiles run over the flattened positions n = b * L_out + l
                        // 0: tiles stay inside one batch row (tiles_l per row)
    int tiles_l;
    int n_tiles;
    int num_units;      // splits * groups * n_cob * n_tiles
    int nch, nbox, margin;
    int nslots;         // batch rows a tile can touch (x window staged per row)
    uint32_t w_stage_bytes, x_stage_bytes, x_box_bytes, x_slot_bytes;
    uint32_t off_w, off_wlo, off_x, off_bias, off_bar;
    unsigned int *status;
};

// A unit of work: one split of the reduction for one tile of up to 128
// consecutive flattened output positions n = b * L_out + l in [nbase, n_end)
// and one block of N output channels of conv group g.  A flat tile may span
// several batch rows b_first ..; "slot" j is batch row b_first + j.  The split is
// the fastest-running index, so a cluster's CTAs hold the splits of one tile.
struct Unit {
    int split, g, cob, nbase, n_end, b_first, nslots, kb0, kb1;
};

__device__ __forceinline__ int floor8(int w) { return (w >= 0) ? (w / 8) * 8 : -(((-w) + 7) / 8) * 8; }

__device__ __forceinline__ Unit decode_unit(const TfArgs &A, int u) {
    Unit r;
    r.split = u % A.splits;
    int t = u / A.splits;
    const int nt = t % A.n_tiles;
    t /= A.n_tiles;
    r.cob = t % A.n_cob;
    r.g = t / A.n_cob;
    if (A.flat) {
        r.nbase = nt * kRows;
        r.n_end = min(r.nbase + kRows, A.P.B * A.P.L_out);
    } else {
        const int b = nt / A.tiles_l;
        const int lb = (nt - b * A.tiles_l) * kRows;
        r.nbase = b * A.P.L_out + lb;
        r.n_end = b * A.P.L_out + min(lb + kRows, A.P.L_out);
    }
    r.b_first = r.nbase / A.P.L_out;
    r.nslots = (r.n_end - 1) / A.P.L_out - r.b_first + 1;
    r.kb0 = r.split * A.kb_per_split;
    r.kb1 = min(A.num_kb, r.kb0 + A.kb_per_split);
    return r;
}

// First staged position of slot j's window: its first output's receptive field
// minus the margin, rounded down to 8 (TMA coordinates are 16-byte aligned).
__device__ __forceinline__ int slot_wx0(const TfArgs &A, const Unit &U, int j) {
    const int lmin = (j == 0) ? U.nbase - U.b_first * A.P.L_out : 0;
    return floor8(lmin * A.P.stride - A.P.padding - A.margin);
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// v - (v with its low 13 mantissa bits cleared), as bits: the operand's tf32 low part.
__device__ __forceinline__ uint32_t lo_bits(uint32_t v) {
    return __float_as_uint(__fsub_rn(__uint_as_float(v), __uint_as_float(v & kTf32Mask)));
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::tf32.
__device__ __forceinline__ void mma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N) {
    return (1u << 4)                       // D format: f32
           | (2u << 7)                     // A format: tf32
           | (2u << 10)                    // B format: tf32
           | ((uint32_t)(N >> 3) << 17)
           | ((uint32_t)(M >> 4) << 24);
}

template <int K>
struct TapsF {
    uint32_t addr[K];   // byte offset of the tap's neighbour pair in a stage row
    float f[K];
    float m[K];
    uint32_t slow;      // bit k: tap k outside the staged window
};

// One col value by the slow path: the position is recomputed from the offset
// in global memory, exact floor, neighbours from global memory.
template <bool MASK>
__device__ __forceinline__ float slow_value(const Problem &P, float start, int k, float off,
                                            float m, const float *row) {
    float pos = __fadd_rn(__fadd_rn(start, (float)(k * P.dilation)), off);
    if (!P.unconstrained)
        pos = fminf(fmaxf(pos, start), __fadd_rn(start, (float)(P.dilation * (P.K - 1))));
    const Tap e = tap_floor_exact(pos);
    const float x0 = (e.i0 >= 0 && e.i0 < P.L_in) ? row[e.i0] : 0.0f;
    const float x1 = (e.i0 >= -1 && e.i0 < P.L_in - 1) ? row[e.i0 + 1] : 0.0f;
    const float v = __fmaf_rn(e.f, __fsub_rn(x1, x0), x0);
    return MASK ? __fmul_rn(v, m) : v;
}

// 8 col values (elements j0 .. j0+7 of a segment whose phase is K0), split in
// tf32 hi and lo parts.
template <int K, int K0, int J0, bool MASK, bool SLOW>
__device__ __forceinline__ void produce8(uint32_t (&hi)[8], uint32_t (&lo)[8], const TapsF<K> &tp,
                                         uint32_t xrow_addr, const Problem &P, float start,
                                         const float *xg, const float *offrow,
                                         const float *maskrow) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int kidx = (K0 + J0 + i) % K;
        const int crel = (K0 + J0 + i) / K;
        float v;
        if (SLOW && ((tp.slow >> kidx) & 1u)) {
            v = slow_value<MASK>(P, start, kidx, offrow[kidx], MASK ? maskrow[kidx] : 1.0f,
                                 xg + (int64_t)crel * P.L_in);
        } else {
            const uint32_t a = xrow_addr + tp.addr[kidx] + crel * kRowBytes;
            const float x0 = lds_f32(a), x1 = lds_f32(a + 4);
            v = __fmaf_rn(tp.f[kidx], __fsub_rn(x1, x0), x0);
            if (MASK)
                v = __fmul_rn(v, tp.m[kidx]);
        }
        const uint32_t h = __float_as_uint(v) & kTf32Mask;
        hi[i] = h;
        lo[i] = __float_as_uint(__fsub_rn(v, __uint_as_float(h)));
    }
}

template <int K, int K0, bool MASK, bool SLOW>
__device__ __forceinline__ void produce_segment(uint32_t tmem_hi, uint32_t tmem_lo,
                                                const TapsF<K> &tp, uint32_t xrow_addr,
                                                const Problem &P, float start, const float *xg,
                                                const float *offrow, const float *maskrow) {
    uint32_t hi[8], lo[8];
    produce8<K, K0, 0, MASK, SLOW>(hi, lo, tp, xrow_addr, P, start, xg, offrow, maskrow);
    tmem_st8(tmem_hi, hi);
    tmem_st8(tmem_lo, lo);
    produce8<K, K0, 8, MASK, SLOW>(hi, lo, tp, xrow_addr, P, start, xg, offrow, maskrow);
    tmem_st8(tmem_hi + 8, hi);
    tmem_st8(tmem_lo + 8, lo);
}

template <int K, bool MASK, bool SLOW>
__device__ __forceinline__ void produce_dispatch(int k0, uint32_t tmem_hi, uint32_t tmem_lo,
                                                 const TapsF<K> &tp, uint32_t xrow_addr,
                                                 const Problem &P, float start, const float *xg,
                                                 const float *offrow, const float *maskrow) {
#define DCN1D_PHASE(P_)                                                                        \
    case P_:                                                                                  \
        if constexpr (P_ < K)                                                                 \
            produce_segment<K, (P_ < K ? P_ : 0), MASK, SLOW>(tmem_hi, tmem_lo, tp, xrow_addr, \
                                                              P, start, xg, offrow, maskrow); \
        break;
    switch (k0) {
        DCN1D_PHASE(0) DCN1D_PHASE(1) DCN1D_PHASE(2) DCN1D_PHASE(3) DCN1D_PHASE(4)
        DCN1D_PHASE(5) DCN1D_PHASE(6) DCN1D_PHASE(7) DCN1D_PHASE(8) DCN1D_PHASE(9)
        DCN1D_PHASE(10) DCN1D_PHASE(11) DCN1D_PHASE(12) DCN1D_PHASE(13) DCN1D_PHASE(14)
        DCN1D_PHASE(15)
        default: break;
    }
#undef DCN1D_PHASE
}

// 18 warps: at most 96 registers per thread (5 warps share a 16K-register sub-partition).
template <int K, bool MASK>
__global__ void __maxnreg__(96)
    tc_tf32_kernel(const __grid_constant__ TfArgs A, const __grid_constant__ CUtensorMap whimap,
                   const __grid_constant__ CUtensorMap xmap) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const Problem &P = A.P;
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    const uint32_t sraw = smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - sraw);
    const uint32_t w_st0 = sbase + A.off_w;
    const uint32_t wlo_st0 = sbase + A.off_wlo;
    const uint32_t x_st0 = sbase + A.off_x;
    const uint32_t bar0 = sbase + A.off_bar;
    float *bias_s = reinterpret_cast<float *>(smem + A.off_bias);
    for (int i = threadIdx.x; i < P.C_out; i += kThreads)
        bias_s[i] = P.bias ? static_cast<const float *>(P.bias)[i] : 0.0f;
    auto bar_full = [&](int s) { return bar0 + 8u * s; };
    auto bar_empty = [&](int s) { return bar0 + 8u * (kStages + s); };
    auto bar_afull = [&](int s) { return bar0 + 8u * (2 * kStages + s); };
    const uint32_t bar_dfull = bar0 + 8u * (3 * kStages);
    const uint32_t bar_dempty = bar0 + 8u * (3 * kStages + 1);
    const uint32_t bar_drain = bar0 + 8u * (3 * kStages + 2);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + A.off_bar + 8 * (3 * kStages + 3));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
            mbar_init(bar_afull(s), kProdWarps / 2);
        }
        mbar_init(bar_dfull, 1);
        mbar_init(bar_dempty, kProdWarps);
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_holder), kTmemCols);
        tc_fence_before();
    }
    if (warp == kTmaWarp && lane == 0) {
        tma_prefetch_desc(&whimap);
        tma_prefetch_desc(&xmap);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const BoundedWait wait{abort_flag, kWaitNs, A.status};

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            for (int u = blockIdx.x; u < A.num_units; u += gridDim.x) {
                const Unit U = decode_unit(A, u);
                const int corow = U.g * P.cout_g + U.cob * A.N;
                const uint32_t tx = A.w_stage_bytes + (uint32_t)U.nslots * A.x_slot_bytes;
                for (int kb = U.kb0; kb < U.kb1; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!wait(bar_empty(s), ph ^ 1u))
                        goto tma_done;
                    mbar_arrive_expect_tx(bar_full(s), tx);
                    tma_load_2d(w_st0 + s * A.w_stage_bytes, &whimap, kb * kBK, corow, bar_full(s));
                    const int c_lo = (kb * kBK) / K;
                    for (int j = 0; j < U.nslots; ++j) {   // one window per batch row of the tile
                        const int xrow = (U.b_first + j) * P.C_in + U.g * P.cin_g + c_lo;
                        const int wx0 = slot_wx0(A, U, j);
                        const uint32_t xdst = x_st0 + s * A.x_stage_bytes + j * A.x_slot_bytes;
                        tma_load_2d(xdst, &xmap, wx0, xrow, bar_full(s));
                        if (A.nbox == 2)
                            tma_load_2d(xdst + A.x_box_bytes, &xmap, wx0 + kBoxStep, xrow,
                                        bar_full(s));
                    }
                }
            }
        tma_done:
            volatile int never = 0;
            const BoundedWait drain{&never, kWaitNs, A.status};
            for (uint32_t j = (it > kStages ? it - kStages : 0); j < it; ++j)
                drain(bar_full(j % kStages), (j / kStages) & 1u);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_tf32_f32(128, A.N);
            uint32_t it = 0, tc = 0;
            for (int u = blockIdx.x; u < A.num_units; u += gridDim.x, ++tc) {
                const Unit U = decode_unit(A, u);
                if (!wait(bar_dempty, (tc & 1u) ^ 1u))
                    goto mma_done;
                tc_fence_after();
                for (int kb = U.kb0; kb < U.kb1; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!wait(bar_full(s), ph) || !wait(bar_afull(s), ph))
                        goto mma_done;
                    tc_fence_after();
                    const uint32_t whi = w_st0 + s * A.w_stage_bytes;
                    const uint32_t wlo = wlo_st0 + s * A.w_stage_bytes;
                    const uint32_t ahi = tmem + kColA + 64u * s;
                    const uint32_t alo = ahi + 32u;
#pragma unroll
                    for (int j = 0; j < kBK / 8; ++j) {
                        const uint32_t acc = (kb > U.kb0 || j > 0) ? 1u : 0u;
                        mma_tf32_ts(tmem + kColD, ahi + 8u * j, sw128_kmajor_desc(whi + 32u * j),
                                    idesc, acc);
                        mma_tf32_ts(tmem + kColD, ahi + 8u * j, sw128_kmajor_desc(wlo + 32u * j),
                                    idesc, 1u);
                        mma_tf32_ts(tmem + kColD, alo + 8u * j, sw128_kmajor_desc(whi + 32u * j),
                                    idesc, 1u);
                    }
                    mma_commit(bar_empty(s));
                }
                mma_commit(bar_dfull);
            }
        mma_done:
            mma_commit(bar_drain);
            volatile int never = 0;
            const BoundedWait drain{&never, kWaitNs, A.status};
            drain(bar_drain, 0);
        }
    } else {
        // ------------------------------------------------------------ producers + epilogue
        const int q = warp % 4;          // TMEM lane quarter
        const int h = warp / 4;          // epilogue share (0..3)
        const int par = h >> 1;          // k-blocks of this parity (relative to the unit start)
        const int half = h & 1;          // which 16 of the 32 elements of a k-block
        const int row = 32 * q + lane;
        const float M = kFloorMagic;
        const float spanf = (float)(P.dilation * (K - 1));

        auto epilogue = [&](int u, uint32_t tcnt) -> bool {
            const Unit U = decode_unit(A, u);
            const int n = U.nbase + row;
            const bool valid = n < U.n_end;
            const int b = valid ? n / P.L_out : 0;
            const int l = valid ? n - b * P.L_out : 0;
            const int co0 = U.g * P.cout_g + U.cob * A.N;
            if (!__all_sync(0xffffffffu, wait(bar_dfull, tcnt & 1u)))
                return false;
            tc_fence_after();
            float *dst = static_cast<float *>(P.out) + (((int64_t)b * P.C_out + co0) * P.L_out + l);
            for (int cc = h; cc < A.N / 16; cc += 4) {
                uint32_t v[16];
                tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + kColD + 16u * cc, v);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int co = 16 * cc + i;
                        dst[(int64_t)co * P.L_out] =
                            __fadd_rn(__uint_as_float(v[i]), bias_s[co0 + co]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_dempty);
            return true;
        };

        // Offsets (and mask) of the next (unit, offset group), loaded one group ahead
        // (past K = 7: when needed, to keep the registers).
        constexpr bool kAhead = K <= 7;
        float raw_off[K], raw_m[K];
        int pf_u = -1, pf_og = -1;
        auto prefetch = [&](int u, const Unit &U, int og) {
            pf_u = u;
            pf_og = og;
            if (u >= A.num_units)
                return;
            const int n = U.nbase + row;
            const int b = n < U.n_end ? n / P.L_out : 0;
            const int l = n < U.n_end ? n - b * P.L_out : 0;
            const int64_t obase = (((int64_t)b * P.offset_groups + og) * P.L_out + l) * K;
#pragma unroll
            for (int k = 0; k < K; ++k) {
                raw_off[k] = static_cast<const float *>(P.off)[obase + k];
                raw_m[k] = MASK ? static_cast<const float *>(P.mask)[obase + k] : 1.0f;
            }
        };
        auto og_of = [&](const Unit &U, int kb) {
            return (U.g * P.cin_g + (kb * kBK) / K) / P.cin_per_og;
        };
        if (kAhead && (int)blockIdx.x < A.num_units) {
            const Unit U0 = decode_unit(A, blockIdx.x);
            prefetch(blockIdx.x, U0, og_of(U0, U0.kb0));
        }
        int pend_u = -1;
        uint32_t pend_cnt = 0, ucount = 0, it_base = 0;
        for (int u = blockIdx.x; u < A.num_units; u += gridDim.x) {
            const Unit U = decode_unit(A, u);
            const int u_next = u + (int)gridDim.x;
            const int n = U.nbase + row;
            const bool valid = n < U.n_end;
            const int b = valid ? n / P.L_out : U.b_first;
            const int l = valid ? n - b * P.L_out : 0;
            const int slot = b - U.b_first;                 // this row's window in the stage
            const uint32_t slot_off = (uint32_t)slot * A.x_slot_bytes;
            const float start = (float)(l * P.stride - P.padding);
            const uint32_t win_bits = kFloorMagicBits + (uint32_t)slot_wx0(A, U, slot);
            const int og_last = (U.g * P.cin_g + ((U.kb1 * kBK - 1) / K)) / P.cin_per_og;
            const float *xb = static_cast<const float *>(P.x) + (int64_t)b * P.C_in * P.L_in;
            TapsF<K> tp;
            int og_cur = -1;
            int og = og_of(U, U.kb0);
            int og_next_c = (og + 1) * P.cin_per_og - U.g * P.cin_g;   // group-relative
            const int nkb = U.kb1 - U.kb0;
            const int kb_first_stage = (nkb < kStages ? nkb : kStages);
            for (int r = par; r < nkb; r += 2) {
                const int kb = U.kb0 + r;
                const uint32_t it = it_base + (uint32_t)r;
                const int s = it % kStages;
                const uint32_t ph = (it / kStages) & 1u;
                const int kk0 = kb * kBK + kSeg * half;
                const int c_first = kk0 / K;
                const int k0 = kk0 - c_first * K;
                const int c_lo = (kb * kBK) / K;
                while (c_first >= og_next_c) {
                    ++og;
                    og_next_c += P.cin_per_og;
                }
                if (og != og_cur) {
                    og_cur = og;
                    if (pf_u != u || pf_og != og)
                        prefetch(u, U, og);
                    tp.slow = 0;
#pragma unroll
                    for (int k = 0; k < K; ++k) {
                        float pos = __fadd_rn(__fadd_rn(start, (float)(k * P.dilation)), raw_off[k]);
                        if (!P.unconstrained)
                            pos = fminf(fmaxf(pos, start), __fadd_rn(start, spanf));
                        const float tt = __fadd_rd(pos, M);
                        const uint32_t rel = __float_as_uint(tt) - win_bits;   // i0 - wx0
                        tp.f[k] = __fsub_rn(pos, __fsub_rn(tt, M));
                        tp.m[k] = raw_m[k];
                        if (rel < (uint32_t)(kBox - 1)) {
                            tp.addr[k] = slot_off + rel * 4u;
                        } else if (A.nbox == 2 && rel < (uint32_t)kWinMax) {
                            tp.addr[k] = slot_off + A.x_box_bytes + (rel - kBoxStep) * 4u;
                        } else {
                            tp.addr[k] = 0;
                            tp.slow |= 1u << k;
                        }
                        if (!valid) {   // rows past the last output: finite zeros, never stored
                            tp.f[k] = 0.0f;
                            tp.m[k] = 0.0f;
                            tp.addr[k] = 0;
                            tp.slow &= ~(1u << k);
                        }
                    }
                    if constexpr (kAhead) {
                        if (og < og_last) {
                            prefetch(u, U, og + 1);
                        } else if (u_next < A.num_units) {
                            const Unit Un = decode_unit(A, u_next);
                            prefetch(u_next, Un, og_of(Un, Un.kb0));
                        }
                    }
                }
                if (!__all_sync(0xffffffffu, wait(bar_full(s), ph)))
                    goto prod_done;
                {
                    // this warp's eighth of the stage's W_lo tile (any layout: elementwise);
                    // the proxy fence orders it before the tensor core's reads, which
                    // follow this warp's arrival on the stage's A barrier
                    const uint32_t share = A.w_stage_bytes / 8u;
                    const uint32_t w0 = (uint32_t)(2 * q + half) * share;
                    const uint32_t whi_s = w_st0 + s * A.w_stage_bytes;
                    const uint32_t wlo_s = wlo_st0 + s * A.w_stage_bytes;
                    for (uint32_t o = w0 + 16u * lane; o < w0 + share; o += 512u) {
                        uint4 v = lds_v4(whi_s + o);
                        v.x = lo_bits(v.x);
                        v.y = lo_bits(v.y);
                        v.z = lo_bits(v.z);
                        v.w = lo_bits(v.w);
                        sts_v4(wlo_s + o, v);
                    }
                    fence_proxy_async_smem();
                }
                {
                    const uint32_t xrow_addr =
                        x_st0 + s * A.x_stage_bytes + (uint32_t)(c_first - c_lo) * kRowBytes;
                    const float *xg = xb + (int64_t)(U.g * P.cin_g + c_first) * P.L_in;
                    const int64_t obase = (((int64_t)b * P.offset_groups + og) * P.L_out + l) * K;
                    const float *offrow = static_cast<const float *>(P.off) + obase;
                    const float *maskrow = MASK ? static_cast<const float *>(P.mask) + obase : nullptr;
                    const uint32_t lanebase = tmem + ((uint32_t)(32 * q) << 16);
                    const uint32_t thi = lanebase + kColA + 64u * s + 16u * half;
                    if (__any_sync(0xffffffffu, tp.slow != 0))
                        produce_dispatch<K, MASK, true>(k0, thi, thi + 32u, tp, xrow_addr, P, start,
                                                        xg, offrow, maskrow);
                    else
                        produce_dispatch<K, MASK, false>(k0, thi, thi + 32u, tp, xrow_addr, P,
                                                         start, xg, offrow, maskrow);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(bar_afull(s));
                }
                if (pend_u >= 0 && r + 2 >= kb_first_stage) {
                    if (!epilogue(pend_u, pend_cnt))
                        goto prod_done;
                    pend_u = -1;
                }
            }
            if (pend_u >= 0) {
                if (!epilogue(pend_u, pend_cnt))
                    goto prod_done;
                pend_u = -1;
            }
            pend_u = u;
            pend_cnt = ucount++;
            it_base += (uint32_t)nkb;
        }
        if (pend_u >= 0 && A.splits == 1)
            epilogue(pend_u, pend_cnt);
    prod_done:;
    }

    if (A.splits > 1) {
        // ------------------------------------------------------------ split-K reduction
        // One unit per CTA.  Chunk c (16 accumulator columns) of the tile belongs to
        // cluster rank c % S and lands in its receive area at slot [this rank][c / S]
        // as [128 rows][16 columns] fp32, over the owner's stage memory; the four
        // 16-byte column groups of row r sit in the order g ^ ((r >> 1) & 3), so the
        // 16-byte accesses of eight consecutive rows cover all 32 banks.
        const int S = A.splits;
        const uint32_t rank = cluster_ctarank();
        const int nchunk = A.N / 16;
        const uint32_t slot_bytes = (uint32_t)A.n_own * 16u * 128u * 4u;
        bool have_d = false;
        if (warp < kProdWarps && (int)blockIdx.x < A.num_units) {
            have_d = __all_sync(0xffffffffu, wait(bar_dfull, 0));
            tc_fence_after();
        }
        // 1: every CTA's accumulator is complete and its stage memory idle (loads
        //    landed, MMAs done)
        cluster_barrier();
        const int q = warp % 4, h = warp / 4, row = 32 * q + lane;
        if (warp < kProdWarps && have_d) {
            for (int c = h; c < nchunk; c += 4) {
                uint32_t v[16];
                tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + kColD + 16u * c, v);
                tmem_wait_ld();
                const uint32_t owner = (uint32_t)(c % S);
                const uint32_t local = sbase + rank * slot_bytes +
                                       (uint32_t)(c / S) * (16u * 128u * 4u) + 64u * row;
                const uint32_t sw = ((uint32_t)row >> 1) & 3u;
                if (owner == rank) {   // this CTA's own chunks stay local
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        sts_v4(local + 16u * ((uint32_t)g ^ sw),
                               make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]));
                } else {
                    const uint32_t remote = cluster_map(local, owner);
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        st_cluster_v4(remote + 16u * ((uint32_t)g ^ sw), v[4 * g], v[4 * g + 1],
                                      v[4 * g + 2], v[4 * g + 3]);
                }
            }
        }
        // 2: every chunk has reached its owner
        cluster_barrier();
        if (warp < kProdWarps && have_d) {
            const Unit U = decode_unit(A, blockIdx.x);
            const int n = U.nbase + row;
            const bool valid = n < U.n_end;
            const int b = valid ? n / P.L_out : 0;
            const int l = valid ? n - b * P.L_out : 0;
            const int co0 = U.g * P.cout_g + U.cob * A.N;
            float *dst = static_cast<float *>(P.out) + (((int64_t)b * P.C_out + co0) * P.L_out + l);
            const uint32_t sw = ((uint32_t)row >> 1) & 3u;
            for (int lc = h; lc < A.n_own; lc += 4) {   // owned chunks over the 4 warps
                const int c = lc * S + (int)rank;
                if (c >= nchunk)
                    break;
                const uint32_t a = sbase + (uint32_t)lc * (16u * 128u * 4u) + 64u * row;
                float acc[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    acc[i] = 0.0f;
                for (int sp = 0; sp < S; ++sp) {   // splits in rank order
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const uint4 p = lds_v4(a + (uint32_t)sp * slot_bytes +
                                               16u * ((uint32_t)g ^ sw));
                        acc[4 * g] = __fadd_rn(acc[4 * g], __uint_as_float(p.x));
                        acc[4 * g + 1] = __fadd_rn(acc[4 * g + 1], __uint_as_float(p.y));
                        acc[4 * g + 2] = __fadd_rn(acc[4 * g + 2], __uint_as_float(p.z));
                        acc[4 * g + 3] = __fadd_rn(acc[4 * g + 3], __uint_as_float(p.w));
                    }
                }
                if (valid) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int co = 16 * c + i;
                        const float r = P.bias ? __fadd_rn(acc[i], bias_s[co0 + co]) : acc[i];
                        dst[(int64_t)co * P.L_out] = r;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

struct TfPlan {
    TfArgs A;
    size_t smem;
};

// Shared-memory layout of A for the given tile mode; false if it does not fit.
bool layout_tf(const Problem &P, TfArgs &A, size_t *smem_out) {
    const int64_t rows = P.L_out < kRows ? P.L_out : kRows;   // outputs of one batch row in a tile
    const int64_t need = (rows - 1) * P.stride + (int64_t)P.dilation * (P.K - 1) + 2 +
                         2 * A.margin + 7;
    if (need > kWinMax)
        return false;
    A.nbox = need > kBox - 1 ? 2 : 1;
    if (A.flat) {
        const int slots = (kRows - 1 + P.L_out - 1) / P.L_out + 1;
        A.nslots = slots < P.B ? slots : P.B;
    } else {
        A.nslots = 1;
    }
    A.w_stage_bytes = (uint32_t)A.N * 128u;
    A.x_box_bytes = (uint32_t)A.nch * kRowBytes;
    A.x_slot_bytes = A.x_box_bytes * A.nbox;
    A.x_stage_bytes = A.x_slot_bytes * A.nslots;
    A.off_w = 0;
    A.off_wlo = A.off_w + kStages * A.w_stage_bytes;
    A.off_x = A.off_wlo + kStages * A.w_stage_bytes;
    A.off_bias = A.off_x + kStages * A.x_stage_bytes;
    A.off_bar = A.off_bias + (uint32_t)((P.C_out * 4 + 15) / 16 * 16);
    size_t smem = A.off_bar + 8 * (3 * kStages + 3) + 16 + 1024;
    if (smem > 227 * 1024)
        return false;
    *smem_out = smem < 116 * 1024 ? 116 * 1024 : smem;   // one CTA per SM
    return true;
}

// The plan for blocks of N output channels; false if it does not fit.
bool plan_for_n(const Problem &P, int N, TfPlan *out) {
    TfArgs A;
    memset(&A, 0, sizeof(A));
    A.P = P;
    const int Kg = P.cin_g * P.K;
    A.N = N;
    if (P.cout_g % A.N != 0)
        return false;
    A.n_cob = P.cout_g / A.N;
    A.num_kb = Kg / kBK;
    A.nch = (kBK - 1) / P.K + 2;
    A.margin = P.unconstrained ? 32 : 0;
    size_t smem = 0;
    // Flat tiles fill all 128 MMA rows when L_out is not a multiple of 128;
    // row tiles need only one x window per stage.
    A.flat = (P.L_out % kRows != 0) ? 1 : 0;
    if (!layout_tf(P, A, &smem)) {
        if (!A.flat)
            return false;
        A.flat = 0;
        if (!layout_tf(P, A, &smem))
            return false;
    }
    A.tiles_l = (P.L_out + kRows - 1) / kRows;
    A.n_tiles = A.flat ? (int)(((int64_t)P.B * P.L_out + kRows - 1) / kRows) : P.B * A.tiles_l;
    const int base_units = P.groups * A.n_cob * A.n_tiles;
    const int sms = sm_count() > 0 ? sm_count() : 148;
    int splits = sms / (base_units > 0 ? base_units : 1);
    const int max_splits = A.num_kb / 8 > 0 ? A.num_kb / 8 : 1;   // at least 8 k-blocks a split
    if (splits > max_splits)
        splits = max_splits;
    if (splits > kMaxSplits)
        splits = kMaxSplits;
    if (splits < 1)
        splits = 1;
    // The splits' partial sums meet in the owners' stage memory: S slots of the owned
    // chunks' [128][16] fp32 blocks must fit below the bias.
    const int nchunk = A.N / 16;
    for (;; --splits) {
        A.kb_per_split = (A.num_kb + splits - 1) / splits;
        A.splits = (A.num_kb + A.kb_per_split - 1) / A.kb_per_split;
        A.n_own = (nchunk + A.splits - 1) / A.splits;
        if (A.splits == 1 || (size_t)A.splits * A.n_own * 16 * 128 * 4 <= A.off_bias)
            break;
    }
    A.num_units = A.splits * base_units;
    out->A = A;
    out->smem = smem;
    return true;
}

bool make_tf_plan(const Problem &P, TfPlan *out) {
    if ((int64_t)P.B * P.L_out + kRows > INT32_MAX || (int64_t)P.B * P.C_in > INT32_MAX)
        return false;   // flattened position and TMA row indices are 32-bit
    // (128-channel blocks, halving the reduction's volume where the reduction splits,
    // measured slower: the producers then pace the contraction)
    return plan_for_n(P, P.cout_g < 256 ? P.cout_g : 256, out);
}

template <int K, bool MASK>
cudaError_t launch_tf_km(const TfPlan &pl, cudaStream_t stream) {
    const Problem &P = pl.A.P;
    TfArgs A = pl.A;
    A.status = device_status_ptr();
    if (!A.status)
        return cudaErrorInvalidDevice;
    const int Kg = P.cin_g * P.K;
    alignas(64) CUtensorMap mhi, mx;
    if (!encode_2d(&mhi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, P.w, (uint64_t)Kg, (uint64_t)P.C_out, 4,
                   kBK, (uint32_t)A.N, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, P.x, (uint64_t)P.L_in,
                   (uint64_t)P.B * P.C_in, 4, kBox, (uint32_t)A.nch, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const int sms = sm_count();
    if (sms <= 0)
        return cudaErrorNoDevice;
    auto kern = tc_tf32_kernel<K, MASK>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), (int)pl.smem);
    if (e != cudaSuccess)
        return e;
    // split-K: one unit per CTA, the splits of a tile a cluster (units <= SMs by the plan)
    const int grid = A.splits > 1 ? A.num_units : (A.num_units < sms ? A.num_units : sms);
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)A.splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    timing_begin(stream);
    e = cudaLaunchKernelEx(&cfg, kern, A, mhi, mx);
    timing_end(stream);
    if (e != cudaSuccess)
        return e;
    return cudaGetLastError();
}

template <int K>
cudaError_t launch_tf_k(const TfPlan &pl, cudaStream_t stream) {
    return pl.A.P.mask ? launch_tf_km<K, true>(pl, stream) : launch_tf_km<K, false>(pl, stream);
}

}  // namespace

bool tc_tf32_supported(const Problem &P) {
    if (P.dtype != DCN1D_F32 || !fast_floor_ok(P))
        return false;
    if (P.K < 1 || P.K > 16)
        return false;
    if (P.cout_g % 32 != 0)
        return false;
    if ((P.cin_g * P.K) % kBK != 0)
        return false;
    if (P.L_in % 4 != 0)   // TMA row stride must be a multiple of 16 bytes
        return false;
    const bool og_whole_group = (P.cin_per_og % P.cin_g) == 0;
    if (!og_whole_group && (P.cin_per_og * P.K) % kSeg != 0)
        return false;
    if ((reinterpret_cast<uintptr_t>(P.x) & 15) || (reinterpret_cast<uintptr_t>(P.w) & 15))
        return false;
    if (P.C_out > 8192)
        return false;
    TfPlan pl;
    return make_tf_plan(P, &pl);
}

int tc_tf32_splits(const Problem &P) {
    TfPlan pl;
    return make_tf_plan(P, &pl) ? pl.A.splits : 0;
}

cudaError_t launch_tc_tf32(const Problem &P, cudaStream_t stream) {
    TfPlan pl;
    if (!make_tf_plan(P, &pl))
        return cudaErrorInvalidValue;
    switch (P.K) {
#define DCN1D_K(K_) \
    case K_: return launch_tf_k<K_>(pl, stream);
        DCN1D_K(1) DCN1D_K(2) DCN1D_K(3) DCN1D_K(4) DCN1D_K(5) DCN1D_K(6) DCN1D_K(7) DCN1D_K(8)
        DCN1D_K(9) DCN1D_K(10) DCN1D_K(11) DCN1D_K(12) DCN1D_K(13) DCN1D_K(14) DCN1D_K(15)
        DCN1D_K(16)
#undef DCN1D_K
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace dcn1d
