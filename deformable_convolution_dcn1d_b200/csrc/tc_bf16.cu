// Fused deformable-im2col + tcgen05 tensor-core contraction, 16-bit inputs (bf16,
// or fp16: the same kernel with the element type a template parameter) and fp32
// accumulation.
//
// Per conv group g the forward is a GEMM over the reduction index kk = (ci, k)
// of the group (k fastest, the weight's own order):
//   D[n, co] = sum_kk cols[n, kk] * W[g*Cg_out + co, kk],   n = output position l
// where cols[n, kk] = m * lerp(x[b, ci, :], pos(l, k)) is the deformable im2col
// ("conv1d" page, "Description", with the sampling of the deformable-
// convolution article, "Step 2").  The cols never exist in global memory:
//
//  * a TILE is 128 consecutive output positions of one (g, b) and one block of
//    N output channels (all Cg_out of them when Cg_out <= 256); the CTA is
//    persistent over tiles;
//  * TMA warp: per 64-wide k-block, one TMA load of the weight tile
//    W[co 0..N-1][kk block] (128-byte swizzle, K-major: the MMA's B operand)
//    and one or two TMA loads of the x window [channels of the block][up to
//    503 positions] (zero-filled outside the signal) into a stage;
//  * producer warps (16 = four per TMEM lane quarter): thread = output row;
//    it turns its row's taps into (window address, fraction pair, mask pair)
//    once per offset group; the four warps of a quarter split the work as
//    (k-block parity) x (half of the k-block), so two k-blocks are produced at
//    once and each warp computes 32 col values per k-block from the staged
//    window in bf16x2 arithmetic, written straight into TENSOR MEMORY with
//    tcgen05.st (the MMA's A operand) -- no shared-memory round trip;
//  * MMA warp: one thread issues 4 tcgen05.mma (M=128, N, K=16) per
//    k-block, A from tensor memory, B from shared memory, D (fp32) in tensor
//    memory, and commits completion to the stage's "empty" barrier;
//  * epilogue, by the same 16 warps (each drains a quarter of its lane
//    quarter's columns): tcgen05.ld the accumulator, add the bias, round to
//    bf16 and store; lanes are consecutive l, so each store is 64 contiguous
//    bytes of out[b, co, :].  A tile's epilogue runs after the producers have
//    staged the first kStages k-blocks of their next tile;
//  * the accumulator alternates between tensor-memory columns [0, N) and
//    [128, 128 + N) from tile to tile, so consecutive tiles share only
//    [128, 256).  The epilogue drains that shared slot first, parking its
//    values in shared memory and releasing the slot before storing them; the
//    next tile's MMAs start on their own slot at once and add the shared part of
//    the staged k-blocks as soon as it is released.  Channel blocks of at most
//    128 rotate over three slots and never wait for a drain;
//  * the last, partial round of tiles: when it holds at most half a grid, the
//    kernel is launched as clusters of two CTAs and the two CTAs of a cluster
//    each take half of one such tile's k-blocks; the second sends its fp32
//    partial sum through distributed shared memory into the first one's freed
//    weight stages, and the first adds it in its drain.
// Stages are chained by mbarriers; every wait is bounded (sm100.cuh).
#include <string.h>

#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "sampler.cuh"
#include "sm100.cuh"

namespace dcn1d {

namespace {

constexpr int kStages = 4;
constexpr int kRows = 128;         // output positions per tile = TMEM lanes
constexpr int kBK = 64;            // reduction elements per k-block
constexpr int kSeg = 32;           // reduction elements per producer warp and k-block
constexpr int kBox = 256;          // x window box width (positions)
constexpr int kBoxStep = 248;      // second box starts here (8 positions of overlap)
constexpr int kWinMax = 503;       // window positions usable by a tap (pair inside one box)
constexpr int kRowBytes = kBox * 2;
constexpr int kProdWarps = 16;     // producer + epilogue warps 0-15: 4 per TMEM lane quarter
constexpr int kTmaWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kThreads = 18 * 32;
constexpr uint32_t kTmemCols = 512;
// Accumulator: columns [0, N) for even tiles of a CTA, [128, 128 + N) for odd ones, so
// columns [128, 256) are the only ones two consecutive tiles share (N > 128); N <= 128
// tiles rotate over [0, 128), [128, 256), [256, 384).  A stages: [384 + 32 s, +32).
constexpr int kSlotCols = 128;
constexpr uint32_t kColA = 384;
constexpr uint64_t kWaitNs = 2000000000ull;   // 2 s

struct TcArgs {
    Problem P;
    int N;             // MMA N: output channels per block (multiple of 32, <= 256)
    int n_cob;         // channel blocks per conv group (Cg_out / N)
    int num_kb;        // k-blocks per tile
    int half_kb;       // > 0: producer groups take contiguous halves [0, half_kb) and
                       // [half_kb, num_kb); 0: they take the even and the odd k-blocks
    int tiles_l;       // tiles per (g, channel block, b)
    int num_tiles;
    int nch;           // x rows per stage
    int nbox;          // x boxes per stage (1 or 2)
    int margin;        // staged positions beyond the receptive fields (unconstrained)
    uint32_t w_stage_bytes, x_stage_bytes, x_box_bytes;
    int pair_store;    // 1: L_out even and out 4-byte aligned (32-bit epilogue stores)
    int xtma;          // 1: x windows by TMA; 0 (L_in not a multiple of 8, even): by the
                       // loader warp's 4-byte cp.async copies into the same layout
    int pair_tail;     // 1: launched as clusters of two CTAs; when the last round holds at
                       // most half a grid of tiles, the two CTAs of a cluster each take half
                       // of one such tile's reduction (positions [0, n/2) and [n/2, n))
    int park;          // 1: the drain parks the shared accumulator slot's values in shared
                       // memory (N > 128 and room for 32 KB), so it releases the slot
                       // before its stores
    uint32_t off_w, off_x, off_bias, off_pos, off_park, off_bar;   // shared-memory layout
    unsigned int *status;                       // device status word
    uint64_t wait_ns;                           // limit of every mbarrier wait
};

// The accumulator of a CTA's tile number tc: its first column, the slot only it uses
// (N > 128: 0 for even tiles, 2 for odd ones; N <= 128: tc % 3) and how many earlier
// tiles used that slot.
struct Acc {
    uint32_t col;
    int own;
    uint32_t own_uses;
};
__device__ __forceinline__ Acc acc_of(uint32_t tc, bool two) {
    Acc a;
    if (two) {
        a.col = (tc & 1u) ? (uint32_t)kSlotCols : 0u;
        a.own = (tc & 1u) ? 2 : 0;
        a.own_uses = tc / 2u;
    } else {
        a.own = (int)(tc % 3u);
        a.col = (uint32_t)kSlotCols * (uint32_t)a.own;
        a.own_uses = tc / 3u;
    }
    return a;
}

// The k-block at pipeline position i of a tile.  The two producer groups take the
// positions by the parity of their ring index, so each group owns every other stage of
// the ring (the ring depth is even), and the ring index parity alternates with the
// position.  With contiguous halves (positions 0, 1, 2, 3, ... -> k-blocks 0, n/2, 1,
// n/2 + 1, ...) a group walks its channels in order and meets each offset group once;
// otherwise the positions are the k-blocks themselves.
__device__ __forceinline__ int kb_at(const TcArgs &A, int i) {
    return A.half_kb ? ((i & 1) ? A.half_kb + (i >> 1) : (i >> 1)) : i;
}

// The i-th unit of work of this CTA: tile t, pipeline positions [p0, p1), and whether it
// is a whole tile (part 0), the first half of a split tile whose result this CTA stores
// (part 1, cluster rank 0) or the second half, sent to the first as a partial sum (part 2).
// Tiles go round-robin over the grid; the last, partial round is split in halves between
// the CTAs of a cluster when it fits in half the grid.  t < 0: no more work.
struct Work {
    int t, p0, p1, part;
};
__device__ __forceinline__ Work work_at(const TcArgs &A, int i) {
    const int grid = (int)gridDim.x, c = (int)blockIdx.x;
    const int full = A.num_tiles / grid;
    const int tail = A.num_tiles - full * grid;
    Work w{-1, 0, A.num_kb, 0};
    if (i < full) {
        w.t = i * grid + c;
    } else if (i == full && tail > 0) {
        if (A.pair_tail && 2 * tail <= grid) {
            if ((c >> 1) < tail) {
                w.t = full * grid + (c >> 1);
                const int h = A.num_kb / 2;
                if (c & 1) {
                    w.p0 = h;
                    w.part = 2;
                } else {
                    w.p1 = h;
                    w.part = 1;
                }
            }
        } else if (c < tail) {
            w.t = full * grid + c;
        }
    }
    return w;
}

struct Tile {
    int g, b, lbase, wx0;
    int co0;           // first output channel of the tile's block
};

__device__ __forceinline__ Tile decode_tile(const TcArgs &A, int t) {
    Tile r;
    // channel blocks of one (g, b, positions) are consecutive tiles: they run at the
    // same time on neighbouring CTAs and share the x window through L2
    // (one block per group is the common case: no division then)
    const int cob = A.n_cob == 1 ? 0 : t % A.n_cob;
    const int t2 = A.n_cob == 1 ? t : t / A.n_cob;
    const int lt = t2 % A.tiles_l;
    const int gb = t2 / A.tiles_l;
    r.b = gb % A.P.B;
    r.g = gb / A.P.B;
    r.co0 = r.g * A.P.cout_g + cob * A.N;
    r.lbase = lt * kRows;
    int w = r.lbase * A.P.stride - A.P.padding - A.margin;
    r.wx0 = (w >= 0) ? (w / 8) * 8 : -(((-w) + 7) / 8) * 8;
    return r;
}

// 16-bit shared load at addr + OFF, zero-extended into a 32-bit register by the
// load itself (the offset rides in the instruction, not in an extra add).
template <uint32_t OFF>
__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u16 %0, [%1+%2];" : "=r"(v) : "r"(addr), "n"(OFF));
    return v;
}

// 4-byte asynchronous global -> shared copy; `bytes` (4 or 0) are read, the rest of the
// 4 bytes zero-filled.
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(bytes)
                 : "memory");
}

// One arrival on `bar` once every cp.async this thread issued so far has landed (the
// arrival counts against the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// The 16-bit element type E of a problem (bf16 or fp16): its pair type, packing,
// unpacking, TMA data type and MMA instruction descriptor (kind::f16 takes both).
template <class E>
struct Elem;

template <>
struct Elem<__nv_bfloat16> {
    using E2 = __nv_bfloat162;
    static constexpr CUtensorMapDataType kTma = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    static __host__ __device__ constexpr uint32_t idesc(int M, int N) {
        return idesc_bf16_f32(M, N);
    }
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        E2 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
    static __device__ __forceinline__ float lo(uint32_t u) { return __uint_as_float(u << 16); }
    static __device__ __forceinline__ float hi(uint32_t u) {
        return __uint_as_float(u & 0xFFFF0000u);
    }
};

template <>
struct Elem<__half> {
    using E2 = __half2;
    static constexpr CUtensorMapDataType kTma = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    static __host__ __device__ constexpr uint32_t idesc(int M, int N) {
        return idesc_f16_f32(M, N);
    }
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        E2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
    static __device__ __forceinline__ float lo(uint32_t u) {
        return __half2float(__ushort_as_half((unsigned short)(u & 0xFFFFu)));
    }
    static __device__ __forceinline__ float hi(uint32_t u) {
        return __half2float(__ushort_as_half((unsigned short)(u >> 16)));
    }
};

template <class E>
__device__ __forceinline__ typename Elem<E>::E2 as_e2(uint32_t u) {
    return *reinterpret_cast<typename Elem<E>::E2 *>(&u);
}
template <class E>
__device__ __forceinline__ uint32_t as_u32(typename Elem<E>::E2 h) {
    return *reinterpret_cast<uint32_t *>(&h);
}

// Per-row tap state of one offset group.  Elements come in pairs (kk, kk+1),
// i.e. taps (k, (k+1) % K), so fractions and mask values are kept pre-packed
// as 16-bit pairs indexed by the first tap of the pair.
//
// Register budget (96 a thread): from K = kPosSmemMinK on, the taps' positions, which
// only the slow path reads, live in shared memory instead (`pos_s`, this thread's column
// of a [K][512] array); past K = 7 a group's offsets are loaded when they are needed
// instead of one group ahead.  Both measured faster (K = 9: no spills, K = 5 with a mask:
// fewer registers).
constexpr int kPosSmemMinK = 4;
template <int K>
constexpr bool kWideK = K >= kPosSmemMinK;
template <int K>
constexpr bool kAheadK = K <= 7;

template <int K>
struct Taps {
    uint32_t addr[K];    // byte offset of the tap's neighbour pair in a stage row
    uint32_t fpair[K];   // E x2 (f_k, f_{(k+1)%K})
    uint32_t mpair[K];   // E x2 (m_k, m_{(k+1)%K})
    float pos[kWideK<K> ? 1 : K];   // position, for taps outside the window (slow path)
    uint32_t slow;       // bit k: tap k outside the staged window
};

constexpr int kProdThreads = kProdWarps * 32;

template <int K>
__device__ __forceinline__ float tap_pos(const Taps<K> &tp, const float *pos_s, int k) {
    if constexpr (kWideK<K>)
        return pos_s[k * kProdThreads];
    else
        return tp.pos[k];
}

// The col value of one element by the slow path: exact floor, global loads.
template <class E, int K, bool MASK>
__device__ __forceinline__ float slow_element(const Taps<K> &tp, const float *pos_s, int kidx,
                                              int hi, const E *row, int L_in) {
    const Tap e = tap_floor_exact(tap_pos<K>(tp, pos_s, kidx));
    const float x0 = (e.i0 >= 0 && e.i0 < L_in) ? ld_f32(row + e.i0) : 0.0f;
    const float x1 = (e.i0 >= -1 && e.i0 < L_in - 1) ? ld_f32(row + e.i0 + 1) : 0.0f;
    const float r = __fmaf_rn(e.f, __fsub_rn(x1, x0), x0);
    if (!MASK)
        return r;
    const uint32_t mp = tp.mpair[(kidx + K - hi) % K];
    return __fmul_rn(r, hi ? Elem<E>::hi(mp) : Elem<E>::lo(mp));
}

// Col values 2I and 2I+1 of a segment whose first element has phase K0 = kk0 % K:
// taps (k0, k1) of channel rows (c0, c1) relative to the segment's first channel.
// The lerp x0 + f (x1 - x0) runs on the two elements in bf16x2 arithmetic.
template <class E, int K, int K0, bool MASK, bool SLOW, int I>
__device__ __forceinline__ void produce_pair(uint32_t (&out)[kSeg / 2], const Taps<K> &tp,
                                             const float *pos_s, const uint32_t (&base)[K],
                                             const E *xg, int64_t xg_row_stride, int L_in) {
    constexpr int k0 = (K0 + 2 * I) % K, c0 = (K0 + 2 * I) / K;
    constexpr int k1 = (K0 + 2 * I + 1) % K, c1 = (K0 + 2 * I + 1) / K;
    constexpr uint32_t o0 = c0 * kRowBytes, o1 = c1 * kRowBytes;
    const uint32_t x0 =
        __byte_perm(lds_u16<o0>(base[k0]), lds_u16<o1>(base[k1]), 0x5410);
    const uint32_t x1 =
        __byte_perm(lds_u16<o0 + 2>(base[k0]), lds_u16<o1 + 2>(base[k1]), 0x5410);
    typename Elem<E>::E2 v = __hfma2(as_e2<E>(tp.fpair[k0]),
                                     __hsub2(as_e2<E>(x1), as_e2<E>(x0)), as_e2<E>(x0));
    if (MASK)
        v = __hmul2(v, as_e2<E>(tp.mpair[k0]));
    out[I] = as_u32<E>(v);
    if (SLOW && (((tp.slow >> k0) | (tp.slow >> k1)) & 1u)) {
        float lo = __low2float(v), hi = __high2float(v);
        if ((tp.slow >> k0) & 1u)
            lo = slow_element<E, K, MASK>(tp, pos_s, k0, 0, xg + c0 * xg_row_stride, L_in);
        if ((tp.slow >> k1) & 1u)
            hi = slow_element<E, K, MASK>(tp, pos_s, k1, 1, xg + c1 * xg_row_stride, L_in);
        out[I] = Elem<E>::pack(lo, hi);
    }
}

template <class E, int K, int K0, bool MASK, bool SLOW, int... Is>
__device__ __forceinline__ void produce_pairs(uint32_t (&out)[kSeg / 2], const Taps<K> &tp,
                                              const float *pos_s, const uint32_t (&base)[K],
                                              const E *xg, int64_t xg_row_stride, int L_in,
                                              std::integer_sequence<int, Is...>) {
    (produce_pair<E, K, K0, MASK, SLOW, Is>(out, tp, pos_s, base, xg, xg_row_stride, L_in),
     ...);
}

// kSeg col values of one row for the reduction elements kk0 .. kk0+kSeg-1 of a k-block,
// packed bf16x2 (element 2i in the low half of out[i]).  Phase K0 = kk0 % K is a
// compile-time constant, so every tap index and row offset below is static.
template <class E, int K, int K0, bool MASK, bool SLOW>
__device__ __forceinline__ void produce_segment(uint32_t (&out)[kSeg / 2], const Taps<K> &tp,
                                                const float *pos_s, uint32_t xrow_addr,
                                                const E *xg, int64_t xg_row_stride, int L_in) {
    uint32_t base[K];
#pragma unroll
    for (int k = 0; k < K; ++k)
        base[k] = xrow_addr + tp.addr[k];
    produce_pairs<E, K, K0, MASK, SLOW>(out, tp, pos_s, base, xg, xg_row_stride, L_in,
                                     std::make_integer_sequence<int, kSeg / 2>{});
}

// Jump to the segment code of phase k0 (a switch, so one indirect branch).
template <class E, int K, bool MASK, bool SLOW>
__device__ __forceinline__ void produce_dispatch(int k0, uint32_t (&out)[kSeg / 2], const Taps<K> &tp,
                                                 const float *pos_s, uint32_t xrow_addr,
                                                 const E *xg, int64_t xg_row_stride, int L_in) {
    if constexpr (kSeg % K == 0) {   // segments start on a channel: phase 0 only
        produce_segment<E, K, 0, MASK, SLOW>(out, tp, pos_s, xrow_addr, xg, xg_row_stride,
                                            L_in);
    } else {
#define DCN1D_PHASE(P_)                                                                          \
    case P_:                                                                                    \
        if constexpr (P_ < K)                                                                   \
            produce_segment<E, K, (P_ < K ? P_ : 0), MASK, SLOW>(out, tp, pos_s, xrow_addr, xg,   \
                                                              xg_row_stride, L_in);             \
        break;
        switch (k0) {
            DCN1D_PHASE(0) DCN1D_PHASE(1) DCN1D_PHASE(2) DCN1D_PHASE(3) DCN1D_PHASE(4)
            DCN1D_PHASE(5) DCN1D_PHASE(6) DCN1D_PHASE(7) DCN1D_PHASE(8)
            default: break;
        }
#undef DCN1D_PHASE
    }
}

// STALL (test builds of the failure path only): the loader issues nothing, so the
// first wait of every other role runs out; the kernel must then record the timeout,
// drain and exit on its own.  Every forward launch uses STALL = false.
template <class E, int K, bool MASK, bool STALL>
// 18 warps: 5 land on some SM sub-partitions, each of which holds 16K registers,
// so a thread may use at most 16384 / (5 * 32) -> 96 registers.
__global__ void __maxnreg__(96)
    tc_bf16_kernel(const __grid_constant__ TcArgs A, const __grid_constant__ CUtensorMap wmap,
                   const __grid_constant__ CUtensorMap xmap) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const Problem &P = A.P;
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    // The 128-byte swizzle needs 1024-byte aligned stages: align the base by hand
    // (the launch reserves 1 KB of slack for this).
    const uint32_t sraw = smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - sraw);
    const uint32_t w_st0 = sbase + A.off_w;
    const uint32_t x_st0 = sbase + A.off_x;
    const uint32_t bar0 = sbase + A.off_bar;
    float *bias_s = reinterpret_cast<float *>(smem + A.off_bias);
    for (int i = threadIdx.x; i < P.C_out; i += kThreads)
        bias_s[i] = P.bias ? ld_f32(static_cast<const E *>(P.bias) + i) : 0.0f;
    auto bar_full = [&](int s) { return bar0 + 8u * s; };
    auto bar_empty = [&](int s) { return bar0 + 8u * (kStages + s); };
    auto bar_afull = [&](int s) { return bar0 + 8u * (2 * kStages + s); };
    const uint32_t bar_dfull = bar0 + 8u * (3 * kStages);
    const uint32_t bar_drain = bar0 + 8u * (3 * kStages + 1);
    // one per 128-column accumulator slot: the drain of the slot's last tile is done
    auto bar_dfree = [&](int slot) { return bar0 + 8u * (3 * kStages + 2 + slot); };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + A.off_bar + 8 * (3 * kStages + 5));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            // TMA mode: the loader's expect-tx arrival; copy mode: also one arrival per
            // loader lane when its copies have landed
            mbar_init(bar_full(s), A.xtma ? 1 : 33);
            mbar_init(bar_empty(s), 1);
            mbar_init(bar_afull(s), kProdWarps / 2);
        }
        mbar_init(bar_dfull, 1);
        mbar_init(bar_drain, 1);
        for (int j = 0; j < 3; ++j)
            mbar_init(bar_dfree(j), kProdWarps);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_holder), kTmemCols);
        tc_fence_before();
    }
    if (warp == kTmaWarp && lane == 0) {
        tma_prefetch_desc(&wmap);
        if (A.xtma)
            tma_prefetch_desc(&xmap);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // the limit is a constant except in the STALL test build
    const uint64_t wait_ns = STALL ? A.wait_ns : kWaitNs;
    const BoundedWait wait{abort_flag, wait_ns, A.status};

    if (warp == kTmaWarp && !A.xtma) {
        // ------------------------------------------------------------ loader, copy mode
        // The weight tile by TMA (lane 0); the x window [nch rows][nbox boxes] by 4-byte
        // copies from all 32 lanes (L_in even, so every copied pair starts on an even
        // element and lies inside its row or outside the signal, zero-filled).
        uint32_t it = 0;
        const int rows_total = P.B * P.C_in;
        const E *xbase = static_cast<const E *>(P.x);
        const int words = A.nbox * (kBox / 2);   // 4-byte words per staged row
        if (!STALL) {
            for (int wi = 0;; ++wi) {
                const Work Wk = work_at(A, wi);
                if (Wk.t < 0)
                    break;
                const Tile T = decode_tile(A, Wk.t);
                const int xrow0 = T.b * P.C_in + T.g * P.cin_g;
                for (int pos = Wk.p0; pos < Wk.p1; ++pos, ++it) {
                    const int kb = kb_at(A, pos);
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!__all_sync(0xffffffffu, wait(bar_empty(s), ph ^ 1u)))
                        goto copy_done;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(bar_full(s), A.w_stage_bytes);
                        tma_load_2d(w_st0 + s * A.w_stage_bytes, &wmap, kb * kBK, T.co0,
                                    bar_full(s));
                    }
                    const int c_lo = (kb * kBK) / K;
                    const uint32_t xdst = x_st0 + s * A.x_stage_bytes;
                    for (int r = 0; r < A.nch; ++r) {
                        const int xr = xrow0 + c_lo + r;
                        const bool row_ok = xr < rows_total;
                        const E *xrow = xbase + (int64_t)(row_ok ? xr : 0) * P.L_in;
                        const uint32_t drow = xdst + (uint32_t)r * kRowBytes;
                        for (int j = lane; j < words; j += 32) {
                            const int bx = j >= kBox / 2 ? 1 : 0;
                            const int w = j - bx * (kBox / 2);
                            const int p = T.wx0 + bx * kBoxStep + 2 * w;
                            const bool ok = row_ok && p >= 0 && p < P.L_in;
                            cp_async4(drow + (uint32_t)bx * A.x_box_bytes + 4u * (uint32_t)w,
                                      ok ? static_cast<const void *>(xrow + p)
                                         : static_cast<const void *>(xbase),
                                      ok ? 4u : 0u);
                        }
                    }
                    cp_async_arrive(bar_full(s));
                }
            }
        }
    copy_done:
        cp_async_wait_all();
        if (lane == 0) {   // the weight tiles still in flight (bounded)
            volatile int never = 0;
            const BoundedWait drain{&never, wait_ns, A.status};
            for (uint32_t j = (it > kStages ? it - kStages : 0); j < it; ++j)
                drain(bar_full(j % kStages), (j / kStages) & 1u);
        }
    } else if (warp == kTmaWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && !STALL) {
            uint32_t it = 0;
            for (int wi = 0;; ++wi) {
                const Work Wk = work_at(A, wi);
                if (Wk.t < 0)
                    break;
                const Tile T = decode_tile(A, Wk.t);
                const int xrow0 = T.b * P.C_in + T.g * P.cin_g;
                for (int pos = Wk.p0; pos < Wk.p1; ++pos, ++it) {
                    const int kb = kb_at(A, pos);
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!wait(bar_empty(s), ph ^ 1u))
                        goto tma_done;
                    mbar_arrive_expect_tx(bar_full(s), A.w_stage_bytes + A.x_stage_bytes);
                    tma_load_2d(w_st0 + s * A.w_stage_bytes, &wmap, kb * kBK, T.co0,
                                bar_full(s));
                    const int c_lo = (kb * kBK) / K;
                    const uint32_t xdst = x_st0 + s * A.x_stage_bytes;
                    tma_load_2d(xdst, &xmap, T.wx0, xrow0 + c_lo, bar_full(s));
                    if (A.nbox == 2)
                        tma_load_2d(xdst + A.x_box_bytes, &xmap, T.wx0 + kBoxStep, xrow0 + c_lo,
                                    bar_full(s));
                }
            }
        tma_done:
            // Let every load this thread issued land before the CTA can exit
            // (bounded; on the normal path they have all been consumed already).
            volatile int never = 0;
            const BoundedWait drain{&never, wait_ns, A.status};
            for (uint32_t j = (it > kStages ? it - kStages : 0); j < it; ++j)
                drain(bar_full(j % kStages), (j / kStages) & 1u);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const bool two = A.N > kSlotCols;
            const uint32_t idesc = Elem<E>::idesc(128, A.N);
            const uint32_t idesc_lo = Elem<E>::idesc(128, kSlotCols);
            const uint32_t idesc_hi = Elem<E>::idesc(128, two ? A.N - kSlotCols : 32);
            uint32_t it = 0, tc = 0;
            for (int wi = 0;; ++wi, ++tc) {
                const Work Wk = work_at(A, wi);
                if (Wk.t < 0)
                    break;
                const Acc acc = acc_of(tc, two);
                // the own slot's last tile (two or three back) has been drained
                if (acc.own_uses > 0 && !wait(bar_dfree(acc.own), (acc.own_uses - 1u) & 1u))
                    goto mma_done;
                tc_fence_after();
                const uint32_t d = tmem + acc.col;
                // N > 128: the shared slot [128, 256) is the previous tile's, drained first.
                // Until it is free, the staged k-blocks contract into the own part only and
                // their shared part follows (at most a ring's worth of k-blocks).
                bool sh_free = !two || tc == 0;
                int pend = 0;
                // the own part: even tiles channels [0, 128) at column 0, odd tiles
                // channels [128, N) at column 256; the shared part is the other one
                auto part = [&](bool own, int p, uint32_t s) {
                    const bool lo = own == ((tc & 1u) == 0u);   // channels [0, 128)?
                    const uint32_t wst = w_st0 + s * A.w_stage_bytes + (lo ? 0u : kSlotCols * 128u);
                    const uint32_t dp = d + (lo ? 0u : (uint32_t)kSlotCols);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        mma_bf16_ts(dp, tmem + kColA + 32u * s + 8u * kk,
                                    sw128_kmajor_desc(wst + 32u * kk), lo ? idesc_lo : idesc_hi,
                                    (p > Wk.p0 || kk > 0) ? 1u : 0u);
                };
                for (int pos = Wk.p0; pos < Wk.p1; ++pos, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!wait(bar_full(s), ph) || !wait(bar_afull(s), ph))
                        goto mma_done;
                    tc_fence_after();
                    if (sh_free) {
                        const uint32_t wst = w_st0 + s * A.w_stage_bytes;
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk) {
                            mma_bf16_ts(d, tmem + kColA + 32u * s + 8u * kk,
                                        sw128_kmajor_desc(wst + 32u * kk), idesc,
                                        (pos > Wk.p0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(bar_empty(s));
                        continue;
                    }
                    part(true, pos, s);
                    ++pend;
                    const bool must = pend == kStages || pos == Wk.p1 - 1;
                    const uint32_t sh_par = (tc - 1u) & 1u;   // the shared slot's last drain
                    if (must ? wait(bar_dfree(1), sh_par) : mbar_try_wait(bar_dfree(1), sh_par)) {
                        tc_fence_after();
                        for (int p = pos + 1 - pend; p <= pos; ++p) {
                            const uint32_t sp = (it - (uint32_t)(pos - p)) % kStages;
                            part(false, p, sp);
                            mma_commit(bar_empty(sp));
                        }
                        pend = 0;
                        sh_free = true;
                    } else if (must) {
                        goto mma_done;
                    }
                }
                mma_commit(bar_dfull);
            }
        mma_done:
            // Every MMA issued has completed once this commit arrives.
            mma_commit(bar_drain);
            volatile int never = 0;
            const BoundedWait drain{&never, wait_ns, A.status};
            drain(bar_drain, 0);
        }
    } else if (warp < kProdWarps) {
        // ------------------------------------------------------------ col producers + epilogue
        const int q = warp % 4;                // TMEM lane quarter
        const int h = warp / 4;                // epilogue share (0..3)
        const int par = h >> 1;                // k-blocks of this parity
        const int half = h & 1;                // which 32 of the 64 elements of a k-block
        const int row = 32 * q + lane;
        // Epilogue of tile t (tile count tcnt): this warp's share of the accumulator columns.
        auto epilogue = [&](int t, uint32_t tcnt) -> bool {
            const Tile T = decode_tile(A, t);
            const int l = T.lbase + row;
            const bool valid = l < P.L_out;
            const float *biasg = bias_s + T.co0;
            if (!__all_sync(0xffffffffu, wait(bar_dfull, tcnt & 1u)))
                return false;
            tc_fence_after();
            E *outp = static_cast<E *>(P.out) +
                                  ((int64_t)T.b * P.C_out + (int64_t)T.co0) * P.L_out + l;
            const bool two = A.N > kSlotCols;
            const Acc acc = acc_of(tcnt, two);
            // N > 128: the chunks in the shared slot [128, 256) first (even tiles: channels
            // 128.., odd tiles: channels 0..127), then the own slot's
            const int n16 = A.N / 16, s16 = kSlotCols / 16;
            const int sh_lo = two ? ((tcnt & 1u) ? 0 : s16) : 0;
            const int sh_hi = two ? ((tcnt & 1u) ? s16 : n16) : 0;
            // The shared slot's chunks (at most two a warp) first.  Parked: bias added,
            // rounded and written to shared memory as packed pairs ([channel pair][row]
            // words, each thread reading back its own), the slot released, then stored, so
            // the next tile's MMAs wait only for the tensor-memory loads.  Otherwise stored
            // before the release.
            uint32_t *park = reinterpret_cast<uint32_t *>(smem + A.off_park) + row;
#pragma unroll 1
            for (int j = 0; j < 2; ++j) {
                const int cc = sh_lo + h + 4 * j;
                if (cc < sh_hi) {
                    uint32_t v[16];
                    tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + acc.col + 16u * cc, v);
                    tmem_wait_ld();
                    if (A.park) {
                        uint32_t *pw = park + (8 * (cc - sh_lo)) * kRows;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            pw[i * kRows] =
                                Elem<E>::pack(__uint_as_float(v[2 * i]) + biasg[16 * cc + 2 * i],
                                              __uint_as_float(v[2 * i + 1]) +
                                                  biasg[16 * cc + 2 * i + 1]);
                    } else if (valid) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int co = 16 * cc + i;
                            outp[(int64_t)co * P.L_out] =
                                from_f32<E>(__uint_as_float(v[i]) + biasg[co]);
                        }
                    }
                }
            }
            if (two) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar_dfree(1));
            }
            if (A.park && valid) {
                unsigned short *outs = reinterpret_cast<unsigned short *>(outp);
#pragma unroll 1
                for (int j = 0; j < 2; ++j) {
                    const int cc = sh_lo + h + 4 * j;
                    if (cc < sh_hi) {
                        const uint32_t *pr = park + (8 * (cc - sh_lo)) * kRows;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const uint32_t w = pr[i * kRows];
                            outs[(int64_t)(16 * cc + 2 * i) * P.L_out] = (unsigned short)(w & 0xFFFFu);
                            outs[(int64_t)(16 * cc + 2 * i + 1) * P.L_out] =
                                (unsigned short)(w >> 16);
                        }
                    }
                }
            }
            // the own slot's chunks
            {
            const int c_begin = sh_lo == 0 ? sh_hi : 0;
            const int c_end = sh_lo == 0 ? n16 : sh_lo;
            for (int cc = c_begin + h; cc < c_end; cc += 4) {
                uint32_t v[16];
                tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + acc.col + 16u * cc, v);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int co = 16 * cc + i;
                        outp[(int64_t)co * P.L_out] =
                            from_f32<E>(__uint_as_float(v[i]) + biasg[co]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_dfree(acc.own));
            }
            return true;
        };
        int pend_t = -1;        // tile whose epilogue is still to do
        uint32_t pend_cnt = 0, tcount = 0;
        const float M = kFloorMagic;
        const float spanf = (float)(P.dilation * (K - 1));
        // Offsets (and mask) of the next (tile, offset group) this thread needs, loaded
        // one group ahead so the global-load latency hides behind the current group
        // (wide K: loaded when needed, to keep the registers).
        constexpr bool kAhead = kAheadK<K>;
        float *pos_s = kWideK<K> ? reinterpret_cast<float *>(smem + A.off_pos) + threadIdx.x
                                 : nullptr;
        float raw_off[K], raw_m[K];
        int pf_t = -1, pf_og = -1;
        auto prefetch = [&](int t, const Tile &T, int og) {
            pf_t = t;
            pf_og = og;
            if (t >= A.num_tiles)
                return;
            const int l = T.lbase + row;
            const int64_t obase =
                (((int64_t)T.b * P.offset_groups + og) * P.L_out + (l < P.L_out ? l : 0)) * K;
#pragma unroll
            for (int k = 0; k < K; ++k) {
                raw_off[k] = ld_f32(static_cast<const E *>(P.off) + obase + k);
                raw_m[k] = MASK ? ld_f32(static_cast<const E *>(P.mask) + obase + k) : 1.0f;
            }
        };
        // offset group of this warp's segment at position `pos` of a tile of group Tt.g
        auto seg_og = [&](const Tile &Tt, int pos) {
            const int c = (kb_at(A, pos) * kBK + kSeg * half) / K;
            return (Tt.g * P.cin_g + c) / P.cin_per_og;
        };
        // This warp's group takes the positions whose ring index tcount*num_kb + pos has
        // its parity, so each ring stage always has the same consumer group, even when a
        // tile has an odd number of k-blocks (a parity wait is never a phase ahead).
        // positions [p0, p1) of a work unit whose first one has ring index base
        auto first_pos = [&](uint32_t base, int p0) {
            return p0 + (int)(((uint32_t)par ^ base) & 1u);
        };
        {
            const Work W0 = work_at(A, 0);
            if (kAhead && W0.t >= 0 && first_pos(0, W0.p0) < W0.p1) {
                const Tile T0 = decode_tile(A, W0.t);
                prefetch(W0.t, T0, seg_og(T0, first_pos(0, W0.p0)));
            }
        }
        uint32_t itbase = 0;    // ring index of the current unit's first position
        for (int wi = 0;; ++wi) {
            const Work Wk = work_at(A, wi);
            if (Wk.t < 0)
                break;
            const int t = Wk.t;
            const Tile T = decode_tile(A, t);
            const uint32_t itnext = itbase + (uint32_t)(Wk.p1 - Wk.p0);
            // Rows past L_out (the last tile's) sample with row 0's offsets: their taps are
            // finite and read the window or the bounds-checked slow path, and their
            // accumulator rows (each depends on its own operand row only) are never stored.
            const int l = T.lbase + row;
            const float start = (float)(l * P.stride - P.padding);
            const float hi_bound = __fadd_rn(start, spanf);   // the receptive field's end
            const float dil_f = (float)P.dilation;
            const uint32_t win_bits = kFloorMagicBits + (uint32_t)T.wx0;
            const int pos_first = first_pos(itbase, Wk.p0);
            const int pos_last =
                pos_first < Wk.p1 ? pos_first + ((Wk.p1 - 1 - pos_first) / 2) * 2 : 0;
            const int og_last = pos_first < Wk.p1 ? seg_og(T, pos_last) : 0;   // this warp's last
            const E *xb = static_cast<const E *>(P.x) + (int64_t)T.b * P.C_in * P.L_in;
            Taps<K> tp;
            // Offset group of the first channel of this warp's first segment; it only
            // grows with the channel, so it is tracked against the next boundary.
            int og_cur = -1;
            int og = (T.g * P.cin_g) / P.cin_per_og;
            int og_next_c = (og + 1) * P.cin_per_og - T.g * P.cin_g;   // group-relative
            const int npos = Wk.p1 - Wk.p0;
            const int kb_first_stage = (npos < kStages ? npos : kStages);
            for (int pos = pos_first; pos < Wk.p1; pos += 2) {
                const int kb = kb_at(A, pos);
                const uint32_t it = itbase + (uint32_t)(pos - Wk.p0);
                const int s = it % kStages;
                const uint32_t ph = (it / kStages) & 1u;
                const int kk0 = kb * kBK + kSeg * half;
                const int c_first = kk0 / K;             // group-relative channel
                const int k0 = kk0 - c_first * K;
                const int c_lo = (kb * kBK) / K;
                while (c_first >= og_next_c) {
                    ++og;
                    og_next_c += P.cin_per_og;
                }
                if (og != og_cur) {
                    og_cur = og;
                    if (pf_t != t || pf_og != og)
                        prefetch(t, T, og);   // not predicted: load now
                    float f[K], m[K];
                    tp.slow = 0;
                    // start + k*d by repeated adds of d: exact (integers below 2^24), the
                    // same value as the product
                    float tap_base = start;
#pragma unroll
                    for (int k = 0; k < K; ++k) {
                        float pos = __fadd_rn(tap_base, raw_off[k]);
                        tap_base = __fadd_rn(tap_base, dil_f);
                        if (!P.unconstrained)
                            pos = fminf(fmaxf(pos, start), hi_bound);
                        const float tt = __fadd_rd(pos, M);
                        const uint32_t rel = __float_as_uint(tt) - win_bits;   // i0 - wx0
                        f[k] = __fsub_rn(pos, __fsub_rn(tt, M));
                        m[k] = raw_m[k];
                        if constexpr (kWideK<K>)
                            pos_s[k * kProdThreads] = pos;
                        else
                            tp.pos[k] = pos;
                        if (rel < (uint32_t)(kBox - 1)) {
                            tp.addr[k] = rel * 2u;
                        } else if (A.nbox == 2 && rel < (uint32_t)kWinMax) {
                            tp.addr[k] = A.x_box_bytes + (rel - kBoxStep) * 2u;
                        } else {
                            tp.addr[k] = 0;
                            tp.slow |= 1u << k;
                        }
                    }
#pragma unroll
                    for (int k = 0; k < K; ++k) {
                        tp.fpair[k] = Elem<E>::pack(f[k], f[(k + 1) % K]);
                        tp.mpair[k] = Elem<E>::pack(m[k], m[(k + 1) % K]);
                    }
                    // next group: the following offset group of this tile, else the
                    // first one of the next tile
                    if constexpr (kAhead) {
                        if (og < og_last)
                            prefetch(t, T, og + 1);
                        else {
                            const Work Wn = work_at(A, wi + 1);   // once per tile
                            if (Wn.t >= 0 && first_pos(itnext, Wn.p0) < Wn.p1) {
                                const Tile Tn = decode_tile(A, Wn.t);
                                prefetch(Wn.t, Tn, seg_og(Tn, first_pos(itnext, Wn.p0)));
                            }
                        }
                    }
                }
                if (!__all_sync(0xffffffffu, wait(bar_full(s), ph)))
                    goto prod_done;
                {
                    const uint32_t xrow_addr =
                        x_st0 + s * A.x_stage_bytes + (uint32_t)(c_first - c_lo) * kRowBytes;
                    const E *xg =
                        xb + (int64_t)(T.g * P.cin_g + c_first) * P.L_in;
                    uint32_t packed[kSeg / 2];
                    if (__any_sync(0xffffffffu, tp.slow != 0))
                        produce_dispatch<E, K, MASK, true>(k0, packed, tp, pos_s, xrow_addr, xg,
                                                        P.L_in,
                                                        P.L_in);
                    else
                        produce_dispatch<E, K, MASK, false>(k0, packed, tp, pos_s, xrow_addr, xg,
                                                         P.L_in,
                                                         P.L_in);
                    tmem_st16(tmem + ((uint32_t)(32 * q) << 16) + kColA + 32u * s + 16u * half,
                              packed);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(bar_afull(s));
                }
                if (pend_t >= 0 && (pos - Wk.p0) + 2 >= kb_first_stage) {
                    if (!epilogue(pend_t, pend_cnt))
                        goto prod_done;
                    pend_t = -1;
                }
            }
            if (pend_t >= 0) {   // this warp had no k-block late enough in the tile
                if (!epilogue(pend_t, pend_cnt))
                    goto prod_done;
                pend_t = -1;
            }
            if (Wk.part == 0) {   // a split unit is finished at the teardown
                pend_t = t;
                pend_cnt = tcount;
            }
            ++tcount;
            itbase = itnext;
        }
        if (pend_t >= 0)
            epilogue(pend_t, pend_cnt);
    prod_done:;
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    {
        // A split last unit.  Every thread of both CTAs of the cluster reaches this point
        // on every path, aborts included, so both cluster barriers always complete.
        const int full = A.num_tiles / (int)gridDim.x;
        const Work Wl = work_at(A, full);
        if (Wl.t >= 0 && Wl.part != 0) {
            // 1: every MMA of both CTAs has completed (each issuer waited for its drain
            // commit; each loader for its copies), so the first CTA's weight stages are
            // free to take the second CTA's partial sum, [N/4][128 rows][4] fp32
            cluster_barrier();
            tc_fence_after();
            const int q = warp % 4, h = warp / 4, row = 32 * q + lane;
            const Acc acc = acc_of((uint32_t)full, A.N > kSlotCols);
            if (Wl.part == 2 && warp < kProdWarps) {
                const uint32_t dst = cluster_map(w_st0, 0);
                for (int cc = h; cc < A.N / 16; cc += 4) {
                    uint32_t v[16];
                    tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + acc.col + 16u * cc, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        st_cluster_v4(dst + 16u * ((uint32_t)(4 * cc + g) * kRows + (uint32_t)row),
                                      v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
                }
            }
            // 2: the partial sum is in place
            cluster_barrier();
            if (Wl.part == 1 && warp < kProdWarps) {
                const Tile T = decode_tile(A, Wl.t);
                const int l = T.lbase + row;
                const float *biasg = bias_s + T.co0;
                const float4 *part = reinterpret_cast<const float4 *>(smem + A.off_w) + row;
                E *outp = static_cast<E *>(P.out) +
                          ((int64_t)T.b * P.C_out + (int64_t)T.co0) * P.L_out + l;
                for (int cc = h; cc < A.N / 16; cc += 4) {
                    uint32_t v[16];
                    tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + acc.col + 16u * cc, v);
                    tmem_wait_ld();
                    if (l < P.L_out) {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const float4 pv = part[(4 * cc + g) * kRows];
                            const float pg[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int co = 16 * cc + 4 * g + i;
                                outp[(int64_t)co * P.L_out] = from_f32<E>(
                                    (__uint_as_float(v[4 * g + i]) + pg[i]) + biasg[co]);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
        }
    }
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

struct Plan {
    TcArgs A;
    size_t smem;
};

bool make_plan(const Problem &P, Plan *out) {
    TcArgs A;
    memset(&A, 0, sizeof(A));
    A.P = P;
    A.status = nullptr;
    const int Kg = P.cin_g * P.K;
    // the widest block of output channels (a multiple of 32, at most 256) that divides
    // the conv group's; each block re-forms the columns it contracts
    A.N = 0;
    for (int n = 256; n >= 32; n -= 32)
        if (P.cout_g % n == 0) {
            A.N = n;
            break;
        }
    if (A.N == 0)
        return false;
    A.n_cob = P.cout_g / A.N;
    A.num_kb = Kg / kBK;
    // Contiguous halves pay off when offset groups change inside a conv group (each
    // warp then meets every offset group of its half once instead of every group of the
    // tile); with one offset group per conv group the k-block parities measure faster.
    A.half_kb = (A.num_kb % 2 == 0 && A.num_kb >= 4 && P.cin_per_og < P.cin_g) ? A.num_kb / 2
                                                                                 : 0;
    A.xtma = (P.L_in % 8 == 0 && (reinterpret_cast<uintptr_t>(P.x) & 15) == 0) ? 1 : 0;
    A.tiles_l = (P.L_out + kRows - 1) / kRows;
    A.num_tiles = P.groups * A.n_cob * P.B * A.tiles_l;
    A.nch = (kBK - 1) / P.K + 2;
    A.margin = P.unconstrained ? 32 : 0;
    const int64_t need = (int64_t)(kRows - 1) * P.stride + (int64_t)P.dilation * (P.K - 1) + 2 +
                         2 * A.margin + 7;
    if (need > kWinMax)
        return false;
    A.nbox = need > kBox - 1 ? 2 : 1;
    A.w_stage_bytes = (uint32_t)A.N * 128u;
    A.x_box_bytes = (uint32_t)A.nch * kRowBytes;
    A.x_stage_bytes = A.x_box_bytes * A.nbox;
    A.off_w = 0;
    A.off_x = A.off_w + kStages * A.w_stage_bytes;
    A.off_bias = A.off_x + kStages * A.x_stage_bytes;
    A.off_pos = A.off_bias + (uint32_t)((P.C_out * 4 + 15) / 16 * 16);
    // wide K: the producers' tap positions, [K][512] floats
    A.off_park = A.off_pos + (P.K >= kPosSmemMinK ? (uint32_t)(P.K * kProdThreads * 4) : 0u);
    const size_t tail = 8 * (3 * kStages + 5) + 16 + 1024;   // barriers + alignment slack
    // the drain's parked shared-slot values, [64 channel pairs][128 rows] words, where
    // they fit
    const uint32_t park_bytes = (uint32_t)(kSlotCols / 2 * kRows * 4);
    A.park = (A.N > kSlotCols && A.off_park + park_bytes + tail <= 227 * 1024) ? 1 : 0;
    A.off_bar = A.off_park + (A.park ? park_bytes : 0u);
    size_t smem = A.off_bar + tail;
    if (smem > 227 * 1024)
        return false;
    // At least half the SM's shared memory, so two CTAs (each allocating all 512
    // tensor-memory columns) never share an SM.
    if (smem < 116 * 1024)
        smem = 116 * 1024;
    out->A = A;
    out->smem = smem;
    return true;
}

// Whether clusters of two CTAs of this kernel and shared-memory size can cover all `sms`
// SMs of the current device at once (asked once per device, kernel and size; the record
// keeps the last 64 answers).
bool pair_clusters_fit(const void *kern, int smem, int sms) {
    struct Seen {
        int dev;
        const void *kern;
        int smem, sms;
        bool ok;
    };
    static std::mutex mu;
    static std::vector<Seen> memo;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return false;
    std::lock_guard<std::mutex> lock(mu);
    for (const auto &m : memo)
        if (m.dev == dev && m.kern == kern && m.smem == smem && m.sms == sms)
            return m.ok;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3((unsigned)sms);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    const bool ok = cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && 2 * n >= sms;
    cudaGetLastError();   // a refused query leaves no error behind
    if (memo.size() >= 64)
        memo.erase(memo.begin());
    memo.push_back({dev, kern, smem, sms, ok});
    return ok;
}

template <class E, int K, bool MASK, bool STALL = false>
cudaError_t launch_km(const Plan &pl, cudaStream_t stream) {
    const Problem &P = pl.A.P;
    alignas(64) CUtensorMap wmap, xmap;
    const int Kg = P.cin_g * P.K;
    if (!encode_2d(&wmap, Elem<E>::kTma, P.w, (uint64_t)Kg, (uint64_t)P.C_out,
                   2, kBK, (uint32_t)pl.A.N, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!pl.A.xtma)
        memset(&xmap, 0, sizeof(xmap));   // copy mode: not read
    else if (!encode_2d(&xmap, Elem<E>::kTma, P.x, (uint64_t)P.L_in, (uint64_t)P.B * P.C_in, 2,
                        kBox, (uint32_t)pl.A.nch, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    auto kern = tc_bf16_kernel<E, K, MASK, STALL>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), (int)pl.smem);
    if (e != cudaSuccess)
        return e;
    const int sms = sm_count();
    if (sms <= 0)
        return cudaErrorNoDevice;
    TcArgs A = pl.A;
    // The last round's tiles split in halves between the CTAs of 2-CTA clusters, when that
    // round holds at most half a grid of tiles and the whole grid fits as clusters.
    const int tail = A.num_tiles % sms;
    const bool pair = !STALL && sms % 2 == 0 && A.num_kb >= 2 && tail > 0 && 2 * tail <= sms &&
                      pair_clusters_fit(reinterpret_cast<const void *>(kern), (int)pl.smem, sms);
    A.pair_tail = pair ? 1 : 0;
    const int grid = pair ? sms : (A.num_tiles < sms ? A.num_tiles : sms);
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pair ? 2u : 1u;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pair ? 1 : 0;
    timing_begin(stream);
    e = cudaLaunchKernelEx(&cfg, kern, A, wmap, xmap);
    timing_end(stream);
    if (e != cudaSuccess)
        return e;
    return cudaGetLastError();
}

template <class E, int K>
cudaError_t launch_k(const Plan &pl, cudaStream_t stream) {
    return pl.A.P.mask ? launch_km<E, K, true>(pl, stream) : launch_km<E, K, false>(pl, stream);
}

template <class E>
cudaError_t launch_e(const Plan &pl, cudaStream_t stream) {
    switch (pl.A.P.K) {
    case 3: return launch_k<E, 3>(pl, stream);
    case 4: return launch_k<E, 4>(pl, stream);
    case 5: return launch_k<E, 5>(pl, stream);
    case 7: return launch_k<E, 7>(pl, stream);
    case 9: return launch_k<E, 9>(pl, stream);
    case 16: return launch_k<E, 16>(pl, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace


bool tc_bf16_supported(const Problem &P) {
    if ((P.dtype != DCN1D_BF16 && P.dtype != DCN1D_F16) || !fast_floor_ok(P))
        return false;
    if (!(P.K == 3 || P.K == 4 || P.K == 5 || P.K == 7 || P.K == 9 || P.K == 16))
        return false;
    if (P.cout_g % 32 != 0)
        return false;
    if ((P.cin_g * P.K) % kBK != 0)
        return false;
    // x windows: by TMA when the row pitch is a multiple of 16 bytes, else by 4-byte
    // copies, which need an even L_in
    if (P.L_in % 2 != 0)
        return false;
    // Offsets are uniform across each 32-element segment of the reduction.
    const bool og_whole_group = (P.cin_per_og % P.cin_g) == 0;
    if (!og_whole_group && (P.cin_per_og * P.K) % kSeg != 0)
        return false;
    if ((reinterpret_cast<uintptr_t>(P.x) & 3) || (reinterpret_cast<uintptr_t>(P.w) & 15))
        return false;
    if (P.C_out > 8192)   // the bias is staged in shared memory
        return false;
    Plan pl;
    return make_plan(P, &pl);
}

cudaError_t launch_tc_bf16(const Problem &P, cudaStream_t stream) {
    Plan pl;
    if (!make_plan(P, &pl))
        return cudaErrorInvalidValue;
    pl.A.status = device_status_ptr();
    if (!pl.A.status)
        return cudaErrorInvalidDevice;
    pl.A.wait_ns = kWaitNs;
    return P.dtype == DCN1D_F16 ? launch_e<__half>(pl, stream)
                                : launch_e<__nv_bfloat16>(pl, stream);
}

bool tc_bf16_stalled_supported(const Problem &P) {
    return tc_bf16_supported(P) && P.dtype == DCN1D_BF16 && P.K == 3 && !P.mask &&
           P.L_in % 8 == 0;
}

cudaError_t launch_tc_bf16_stalled(const Problem &P, uint64_t wait_ns, cudaStream_t stream) {
    Plan pl;
    if (!tc_bf16_stalled_supported(P) || !make_plan(P, &pl))
        return cudaErrorInvalidValue;
    pl.A.status = device_status_ptr();
    if (!pl.A.status)
        return cudaErrorInvalidDevice;
    pl.A.wait_ns = wait_ns;
    return launch_km<__nv_bfloat16, 3, false, true>(pl, stream);
}

}  // namespace dcn1d
