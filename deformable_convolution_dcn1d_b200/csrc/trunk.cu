// PackedDeformConv1d's offset (and mask) predictor: the depthwise-separable
// block of the "dc1d (DeformConv1d)" page ("PackedDeformConv1d"; "Modulation
// (DCNv2)" for the second, sigmoid-terminated branch off the same trunk):
//
//   t[b,c,l]         = dw_b[c] + sum_k dw_w[c,k] * x[b, c, l*s - p + k*d]   (zero outside)
//   offsets[b,g,l,k] = off_b[j] + sum_c off_w[j,c] * t[b,c,l],            j = g*K + k
//   mask[b,g,l,k]    = sigmoid(mask_b[j] + sum_c mask_w[j,c] * t[b,c,l])
//
// t never leaves the chip: it is formed in fp32 and consumed by the pointwise
// contraction in the same kernel.  Two kernels:
//
//  * trunk_tc_kernel (16-bit inputs, C_in a multiple of 64 up to 512): a tile is
//    128 output positions of one batch element.  Sixteen producer warps compute
//    the tile's t for every channel (fp32 FMAs over x read straight from global
//    memory, rounded once to the input type) into shared memory in the 128-byte
//    swizzled K-major layout the tensor core reads; then one thread issues
//    tcgen05.mma (M=128, N up to 256, K=16) against pointwise-weight tiles that
//    a TMA warp streams through a ring of stages, accumulating in tensor memory
//    (two 256-column buffers, so the next column chunk's MMAs run while the
//    producer warps drain the previous one).  The drain adds the bias, applies
//    the sigmoid on the mask head and stores in the [B, G, L_out, K] layout.
//  * trunk_simt_kernel (every dtype and shape): 64 positions x 64 head channels
//    per block, t formed per 16-channel slice in shared memory, CUDA-core FMAs.
#include <string.h>

#include "common.cuh"
#include "sm100.cuh"

namespace dcn1d {

namespace {

// ---------------------------------------------------------------- CUDA-core kernel

constexpr int kSimtL = 64, kSimtJ = 64, kSimtC = 16, kSimtThreads = 256;

// One output of a head: bias, sigmoid on the mask head, [B, G, L_out, K] address.
template <class T>
__device__ __forceinline__ void store_head(const TrunkProblem &P, int head, int j, int b, int l,
                                           float z) {
    const T *bias = static_cast<const T *>(head ? P.mask_b : P.off_b);
    if (bias)
        z += ld_f32(bias + j);
    if (head)
        z = 1.0f / (1.0f + expf(-z));
    const int g = j / P.K, k = j - g * P.K;
    T *out = static_cast<T *>(head ? P.mask_out : P.off_out);
    out[(((int64_t)b * P.offset_groups + g) * P.L_out + l) * P.K + k] = from_f32<T>(z);
}

template <class T>
__global__ void __launch_bounds__(kSimtThreads)
    trunk_simt_kernel(const __grid_constant__ TrunkProblem P) {
    __shared__ float ts[kSimtC][kSimtL + 4];
    __shared__ float ws[kSimtC][kSimtJ + 4];
    const int l0 = blockIdx.x * kSimtL;
    const int jt0 = blockIdx.y * kSimtJ;   // over both heads: [0, J) offsets, [J, 2J) mask
    const int b = blockIdx.z;
    const int heads = P.mask_out ? 2 : 1;
    const int Jt = heads * P.J;
    const int tid = threadIdx.x;
    const int tj = tid / 16, tl = tid % 16;
    const T *x = static_cast<const T *>(P.x) + (int64_t)b * P.C_in * P.L_in;
    const T *dww = static_cast<const T *>(P.dw_w);
    const T *dwb = static_cast<const T *>(P.dw_b);
    float acc[4][4] = {};
    for (int c0 = 0; c0 < P.C_in; c0 += kSimtC) {
        for (int i = tid; i < kSimtC * kSimtL; i += kSimtThreads) {
            const int cc = i / kSimtL, ll = i % kSimtL;
            const int c = c0 + cc, l = l0 + ll;
            float t = 0.0f;
            if (c < P.C_in && l < P.L_out) {
                t = dwb ? ld_f32(dwb + c) : 0.0f;
                for (int k = 0; k < P.K; ++k) {
                    const int pos = l * P.stride - P.padding + k * P.dilation;
                    if (pos >= 0 && pos < P.L_in)
                        t = fmaf(ld_f32(dww + (int64_t)c * P.K + k),
                                 ld_f32(x + (int64_t)c * P.L_in + pos), t);
                }
            }
            ts[cc][ll] = t;
        }
        for (int i = tid; i < kSimtC * kSimtJ; i += kSimtThreads) {
            const int jj = i / kSimtC, cc = i % kSimtC;
            const int jt = jt0 + jj, c = c0 + cc;
            float w = 0.0f;
            if (jt < Jt && c < P.C_in) {
                const int head = jt >= P.J, j = jt - head * P.J;
                const T *W = static_cast<const T *>(head ? P.mask_w : P.off_w);
                w = ld_f32(W + (int64_t)j * P.C_in + c);
            }
            ws[cc][jj] = w;
        }
        __syncthreads();
#pragma unroll 4
        for (int cc = 0; cc < kSimtC; ++cc) {
            float wv[4], tv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                wv[a] = ws[cc][tj + 16 * a];
                tv[a] = ts[cc][tl + 16 * a];
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc[a][e] = fmaf(wv[a], tv[e], acc[a][e]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int jt = jt0 + tj + 16 * a;
        if (jt >= Jt)
            continue;
        const int head = jt >= P.J;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int l = l0 + tl + 16 * e;
            if (l < P.L_out)
                store_head<T>(P, head, jt - head * P.J, b, l, acc[a][e]);
        }
    }
}

template <class T>
cudaError_t launch_simt(const TrunkProblem &P, cudaStream_t stream) {
    const int heads = P.mask_out ? 2 : 1;
    dim3 grid((P.L_out + kSimtL - 1) / kSimtL, (heads * P.J + kSimtJ - 1) / kSimtJ, P.B);
    timing_begin(stream);
    trunk_simt_kernel<T><<<grid, kSimtThreads, 0, stream>>>(P);
    timing_end(stream);
    return cudaGetLastError();
}


// ---------------------------------------------------------------- tensor-core kernel

constexpr int kTRows = 128;                 // output positions per tile = TMEM lanes
constexpr int kTBK = 64;                    // channels per k-block (128 bytes of 16-bit values)
constexpr uint32_t kTABytes = kTRows * 128; // one k-block of the A tile (16 KB)
constexpr int kTMaxN = 256;                 // head channels per column chunk (MMA N limit)
constexpr int kTMaxCin = 512;               // the whole A tile stays in shared memory
constexpr int kTBoxMax = 256;               // widest x window a TMA box holds (positions)
constexpr int kTProdWarps = 16, kTWTmaWarp = 16, kTMmaWarp = 17, kTXTmaWarp = 18;
constexpr int kTThreads = 19 * 32;
constexpr uint32_t kTTmemCols = 512;        // two accumulator buffers of 256 columns
constexpr uint64_t kTWaitNs = 2000000000ull;   // 2 s

template <class E>
struct TElem;

template <>
struct TElem<__nv_bfloat16> {
    static constexpr CUtensorMapDataType kTma = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    static __host__ __device__ constexpr uint32_t idesc(int M, int N) {
        return idesc_bf16_f32(M, N);
    }
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
    static __device__ __forceinline__ float widen(uint32_t bits16) {
        return __uint_as_float(bits16 << 16);
    }
};

template <>
struct TElem<__half> {
    static constexpr CUtensorMapDataType kTma = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    static __host__ __device__ constexpr uint32_t idesc(int M, int N) {
        return idesc_f16_f32(M, N);
    }
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
    static __device__ __forceinline__ float widen(uint32_t bits16) {
        return __half2float(__ushort_as_half((unsigned short)bits16));
    }
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint32_t (&v)[4]) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v[0]), "r"(v[1]),
                 "r"(v[2]), "r"(v[3])
                 : "memory");
}

__device__ __forceinline__ uint32_t ld_shared_u16(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// The logistic function through the hardware tanh: sigmoid(z) = (1 + tanh(z/2)) / 2.
// tanh.approx.f32 is accurate to about 2^-11 relative, far inside a 16-bit output's
// rounding (the tensor-core kernel writes bf16 or fp16 only).
__device__ __forceinline__ float sigmoid_tanh(float z) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
    return fmaf(0.5f, t, 0.5f);
}

// Bias, sigmoid (mask head) and store of 32 consecutive head columns of one row (the
// first n_valid of them when kFull is false): column i's (offset, bias) pair is tab[i],
// read two pairs per 16-byte load.  The table is written once before the CTA's first
// barrier, so these are ordinary loads the compiler may schedule ahead of their use.
// The full form has no per-column test.
template <class E, bool kMaskHead, bool kFull>
__device__ __forceinline__ void drain32(const uint32_t (&v)[32], const int4 *tab, E *orow,
                                        int n_valid) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        if (kFull || i < n_valid) {
            const int4 e = tab[i / 2];
            float z0 = __uint_as_float(v[i]) + __int_as_float(e.y);
            float z1 = __uint_as_float(v[i + 1]) + __int_as_float(e.w);
            if (kMaskHead) {
                z0 = sigmoid_tanh(z0);
                z1 = sigmoid_tanh(z1);
            }
            orow[e.x] = from_f32<E>(z0);
            if (kFull || i + 1 < n_valid)
                orow[e.z] = from_f32<E>(z1);
        }
    }
}

template <class E, bool kMaskHead>
__device__ __forceinline__ void drain32_any(const uint32_t (&v)[32], const int4 *tab,
                                            E *orow, int n_valid) {
    if (n_valid >= 32)
        drain32<E, kMaskHead, true>(v, tab, orow, 32);
    else
        drain32<E, kMaskHead, false>(v, tab, orow, n_valid);
}

struct TcTrunkArgs {
    TrunkProblem P;
    int nkb;                 // k-blocks: C_in / 64
    int nbox;                // MMA N = weight tile rows (multiple of 16, <= 256)
    int chunks_per_head;     // column chunks of kTMaxN per head
    int heads, chunks;       // heads (1 or 2) and chunks per tile
    int tiles_l, num_tiles;
    int wstages, xstages;    // weight and x ring depths
    int boxw;                // x window width (positions, multiple of 8)
    int tabj;                // column-table entries per head (J rounded up to even: each
                             // head's table starts on 16 bytes for the paired loads)
    uint32_t w_stage_bytes, x_stage_bytes;
    uint32_t off_a, off_w, off_x, off_dw, off_tab, off_bar;   // shared-memory layout
    unsigned int *status;    // device status word
};

// First position of the x window of a tile: l*s - p for its first row, rounded down to a
// multiple of 8 (a TMA box starts on 16 bytes); may be negative (zero fill).
__device__ __forceinline__ int window_start(const TrunkProblem &P, int lbase) {
    const int w = lbase * P.stride - P.padding;
    return w >= 0 ? (w / 8) * 8 : -(((-w) + 7) / 8) * 8;
}

// kStageX: the x window of every (tile, k-block) is staged in shared memory by TMA (a
// 19th warp issues those loads ahead of the producers); otherwise the producers read x
// from global memory.  Every ring (weights, x windows) has exactly one consumer order:
// a waiter is never more than one phase ahead of a barrier, which the parity waits need.
template <class E, bool kStageX>
__global__ void __launch_bounds__(kTThreads, 1)
    trunk_tc_kernel(const __grid_constant__ TcTrunkArgs A,
                    const __grid_constant__ CUtensorMap map_off,
                    const __grid_constant__ CUtensorMap map_mask,
                    const __grid_constant__ CUtensorMap map_x) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const TrunkProblem &P = A.P;
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    // The 128-byte swizzle wants 1024-byte aligned tiles (1 KB of slack is reserved).
    const uint32_t sraw = smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - sraw);
    const uint32_t a_s = sbase + A.off_a;
    const uint32_t w_s0 = sbase + A.off_w;
    const uint32_t x_s0 = sbase + A.off_x;
    float *dw_s = reinterpret_cast<float *>(smem + A.off_dw);   // [C_in][K] weights, [C_in] biases
    int2 *tab = reinterpret_cast<int2 *>(smem + A.off_tab);     // [heads][J] (offset, bias)
    const uint32_t bar0 = sbase + A.off_bar;
    const int SW = A.wstages, SX = A.xstages;
    auto w_full = [&](int s) { return bar0 + 8u * s; };
    auto w_empty = [&](int s) { return bar0 + 8u * (SW + s); };
    auto x_full = [&](int s) { return bar0 + 8u * (2 * SW + s); };
    auto x_empty = [&](int s) { return bar0 + 8u * (2 * SW + SX + s); };
    const uint32_t a_full = bar0 + 8u * (2 * SW + 2 * SX);
    const uint32_t a_empty = a_full + 8u;
    const uint32_t d_full0 = a_full + 16u;    // + 8 d
    const uint32_t d_empty0 = a_full + 32u;   // + 8 d
    const uint32_t drain_bar = a_full + 48u;
    uint32_t *tmem_holder =
        reinterpret_cast<uint32_t *>(smem + A.off_bar + 8 * (2 * SW + 2 * SX) + 56);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    {
        const E *dww = static_cast<const E *>(P.dw_w);
        const E *dwb = static_cast<const E *>(P.dw_b);
        for (int i = threadIdx.x; i < P.C_in * P.K; i += kTThreads)
            dw_s[i] = ld_f32(dww + i);
        for (int i = threadIdx.x; i < P.C_in; i += kTThreads)
            dw_s[P.C_in * P.K + i] = dwb ? ld_f32(dwb + i) : 0.0f;
        // Per head column j = g*K + k: its offset in the [G, L_out, K] block of one batch
        // element (relative to row l's first value) and its bias.
        const int LK = P.L_out * P.K;
        for (int i = threadIdx.x; i < A.heads * A.tabj; i += kTThreads) {
            const int head = i >= A.tabj, j = i - head * A.tabj;
            const int g = j / P.K, k = j - g * P.K;
            const E *bias = static_cast<const E *>(head ? P.mask_b : P.off_b);
            tab[i] = j < P.J ? make_int2(g * LK + k,
                                         __float_as_int(bias ? ld_f32(bias + j) : 0.0f))
                             : make_int2(0, 0);
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < SW; ++s) {
            mbar_init(w_full(s), 1);
            mbar_init(w_empty(s), 1);
        }
        for (int s = 0; s < SX; ++s) {
            mbar_init(x_full(s), 1);
            mbar_init(x_empty(s), kTProdWarps);   // every producer warp reads every stage
        }
        mbar_init(a_full, kTProdWarps);
        mbar_init(a_empty, 1);
        for (int d = 0; d < 2; ++d) {
            mbar_init(d_full0 + 8u * d, 1);
            mbar_init(d_empty0 + 8u * d, kTProdWarps);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kTMmaWarp) {
        tmem_alloc(smem_u32(tmem_holder), kTTmemCols);
        tc_fence_before();
    }
    if (warp == kTWTmaWarp && lane == 0) {
        tma_prefetch_desc(&map_off);
        if (A.heads > 1)
            tma_prefetch_desc(&map_mask);
        if (kStageX)
            tma_prefetch_desc(&map_x);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const BoundedWait wait{abort_flag, kTWaitNs, A.status};

    if (warp == kTWTmaWarp) {
        // ------------------------------------------------------------ weight tiles
        if (lane == 0) {
            uint32_t it = 0;
            for (int t = blockIdx.x; t < A.num_tiles; t += gridDim.x)
                for (int c = 0; c < A.chunks; ++c) {
                    const int head = c / A.chunks_per_head;
                    const int n0 = (c % A.chunks_per_head) * kTMaxN;
                    const CUtensorMap *map = head ? &map_mask : &map_off;
                    for (int kb = 0; kb < A.nkb; ++kb, ++it) {
                        const int s = it % SW;
                        const uint32_t ph = (it / SW) & 1u;
                        if (!wait(w_empty(s), ph ^ 1u))
                            goto wtma_done;
                        mbar_arrive_expect_tx(w_full(s), A.w_stage_bytes);
                        tma_load_2d(w_s0 + s * A.w_stage_bytes, map, kb * kTBK, n0, w_full(s));
                    }
                }
        wtma_done:
            // Let every load this thread issued land before the CTA can exit.
            volatile int never = 0;
            const BoundedWait drain{&never, kTWaitNs, A.status};
            const uint32_t S = (uint32_t)SW;
            for (uint32_t j = (it > S ? it - S : 0); j < it; ++j)
                drain(w_full(j % S), (j / S) & 1u);
        }
    } else if (warp == kTXTmaWarp) {
        // ------------------------------------------------------------ x windows
        if (kStageX && lane == 0) {
            uint32_t it = 0;
            for (int t = blockIdx.x; t < A.num_tiles; t += gridDim.x) {
                const int b = t / A.tiles_l;
                const int wx0 = window_start(P, (t % A.tiles_l) * kTRows);
                for (int kb = 0; kb < A.nkb; ++kb, ++it) {
                    const int s = it % SX;
                    const uint32_t ph = (it / SX) & 1u;
                    if (!wait(x_empty(s), ph ^ 1u))
                        goto xtma_done;
                    mbar_arrive_expect_tx(x_full(s), A.x_stage_bytes);
                    tma_load_2d(x_s0 + s * A.x_stage_bytes, &map_x, wx0, b * P.C_in + kb * kTBK,
                                x_full(s));
                }
            }
        xtma_done:
            volatile int never = 0;
            const BoundedWait drain{&never, kTWaitNs, A.status};
            const uint32_t S = (uint32_t)SX;
            for (uint32_t j = (it > S ? it - S : 0); j < it; ++j)
                drain(x_full(j % S), (j / S) & 1u);
        }
    } else if (warp == kTMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = TElem<E>::idesc(kTRows, A.nbox);
            uint32_t it = 0, cg = 0, tc = 0;
            for (int t = blockIdx.x; t < A.num_tiles; t += gridDim.x, ++tc) {
                if (!wait(a_full, tc & 1u))
                    goto mma_done;
                tc_fence_after();
                for (int c = 0; c < A.chunks; ++c, ++cg) {
                    const uint32_t d = cg & 1u;
                    if (!wait(d_empty0 + 8u * d, ((cg >> 1) & 1u) ^ 1u))
                        goto mma_done;
                    tc_fence_after();
                    for (int kb = 0; kb < A.nkb; ++kb, ++it) {
                        const int s = it % SW;
                        const uint32_t ph = (it / SW) & 1u;
                        if (!wait(w_full(s), ph))
                            goto mma_done;
                        tc_fence_after();
                        const uint32_t wst = w_s0 + s * A.w_stage_bytes;
                        const uint32_t ast = a_s + kb * kTABytes;
#pragma unroll
                        for (int kk = 0; kk < kTBK / 16; ++kk)
                            mma_f16_ss(tmem + 256u * d, sw128_kmajor_desc(ast + 32u * kk),
                                       sw128_kmajor_desc(wst + 32u * kk), idesc,
                                       (kb > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(w_empty(s));
                    }
                    mma_commit(d_full0 + 8u * d);
                }
                mma_commit(a_empty);   // the tile's A may be overwritten once this arrives
            }
        mma_done:
            // Every MMA issued has completed once this commit arrives.
            mma_commit(drain_bar);
            volatile int never = 0;
            const BoundedWait drain{&never, kTWaitNs, A.status};
            drain(drain_bar, 0);
        }
    } else {
        // ------------------------------------------------------------ depthwise + drain
        const int q = warp % 4;          // TMEM lane quarter
        const int h = warp / 4;          // k-blocks h, h+4, ... (global-load path); columns 64h..64h+63
        const int r = 32 * q + lane;     // tile row
        uint32_t cg = 0, tc = 0;
        for (int t = blockIdx.x; t < A.num_tiles; t += gridDim.x, ++tc) {
            const int b = t / A.tiles_l;
            const int lbase = (t % A.tiles_l) * kTRows;
            const int l = lbase + r;
            const bool valid = l < P.L_out;
            if (!__all_sync(0xffffffffu, wait(a_empty, (tc & 1u) ^ 1u)))
                goto prod_done;
            if constexpr (kStageX) {
                // Every warp takes 16 channels (two 16-byte chunks) of every k-block, so the
                // x stages are consumed in ring order whatever the ring's depth.
                // Window position of tap 0 of this row: l*s - p - window start (>= 0).
                const uint32_t rel0 =
                    (uint32_t)(r * P.stride + lbase * P.stride - P.padding -
                               window_start(P, lbase));
                for (int kb = 0; kb < A.nkb; ++kb) {
                    const uint32_t itx = tc * (uint32_t)A.nkb + (uint32_t)kb;
                    const int s = itx % SX;
                    if (!__all_sync(0xffffffffu, wait(x_full(s), (itx / SX) & 1u)))
                        goto prod_done;
                    const uint32_t xst = x_s0 + s * A.x_stage_bytes + rel0 * 2u;
                    const uint32_t row_addr = a_s + kb * kTABytes + r * 128;
#pragma unroll 1
                    for (int ch = 2 * h; ch < 2 * h + 2; ++ch) {   // 8 channels = 16 bytes
                        const int c0 = kb * kTBK + ch * 8;
                        float acc[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            acc[i] = dw_s[P.C_in * P.K + c0 + i];
                        const uint32_t xrow = xst + (uint32_t)(ch * 8) * A.boxw * 2u;
                        for (int k = 0; k < P.K; ++k) {
                            const uint32_t xa = xrow + (uint32_t)(k * P.dilation) * 2u;
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                acc[i] = fmaf(dw_s[(c0 + i) * P.K + k],
                                              TElem<E>::widen(ld_shared_u16(
                                                  xa + (uint32_t)i * A.boxw * 2u)),
                                              acc[i]);
                        }
                        uint32_t pk[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            pk[i] = TElem<E>::pack(acc[2 * i], acc[2 * i + 1]);
                        // 128-byte swizzle: 16-byte chunk `ch` of row r sits at chunk ch ^ (r % 8)
                        st_shared_v4(row_addr + ((uint32_t)(ch ^ (r & 7)) << 4), pk);
                    }
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(x_empty(s));
                }
            } else {
                const E *xb = static_cast<const E *>(P.x) + (int64_t)b * P.C_in * P.L_in;
                const int pos0 = l * P.stride - P.padding;
                for (int kb = h; kb < A.nkb; kb += 4) {
                    const uint32_t row_addr = a_s + kb * kTABytes + r * 128;
#pragma unroll 1
                    for (int ch = 0; ch < 8; ++ch) {
                        const int c0 = kb * kTBK + ch * 8;
                        float acc[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            acc[i] = dw_s[P.C_in * P.K + c0 + i];
                        if (valid) {
                            for (int k = 0; k < P.K; ++k) {
                                const int pos = pos0 + k * P.dilation;
                                if (pos >= 0 && pos < P.L_in) {
                                    const E *xp = xb + (int64_t)c0 * P.L_in + pos;
#pragma unroll
                                    for (int i = 0; i < 8; ++i)
                                        acc[i] = fmaf(dw_s[(c0 + i) * P.K + k],
                                                      ld_f32(xp + (int64_t)i * P.L_in), acc[i]);
                                }
                            }
                        }
                        uint32_t pk[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            pk[i] = TElem<E>::pack(acc[2 * i], acc[2 * i + 1]);
                        st_shared_v4(row_addr + ((uint32_t)(ch ^ (r & 7)) << 4), pk);
                    }
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(a_full);
            {
                // offset of row l's first value in batch element b's [G, L_out, K] block
                const int64_t rowoff =
                    ((int64_t)b * P.offset_groups * P.L_out + (valid ? l : 0)) * P.K;
                for (int c = 0; c < A.chunks; ++c, ++cg) {
                    const uint32_t d = cg & 1u;
                    if (!__all_sync(0xffffffffu, wait(d_full0 + 8u * d, (cg >> 1) & 1u)))
                        goto prod_done;
                    tc_fence_after();
                    const int head = c / A.chunks_per_head;
                    const int n0 = (c % A.chunks_per_head) * kTMaxN;
                    E *orow = static_cast<E *>(head ? P.mask_out : P.off_out) + rowoff;
                    const int2 *tab_h = tab + head * A.tabj;
                    // this warp's 64 columns of the chunk, 32 per tensor-memory load
                    for (int blk = 0; blk < 2; ++blk) {
                        const int col = 64 * h + 32 * blk;
                        if (col >= A.nbox)
                            break;
                        uint32_t v[32];
                        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + 256u * d + (uint32_t)col, v);
                        tmem_wait_ld();
                        const int j0 = n0 + col;
                        const int n_valid = P.J - j0 < 32 ? P.J - j0 : 32;
                        if (valid) {
                            // j0 is even and every head's table starts on 16 bytes
                            const int4 *t4 = reinterpret_cast<const int4 *>(tab_h + j0);
                            if (head)
                                drain32_any<E, true>(v, t4, orow, n_valid);
                            else
                                drain32_any<E, false>(v, t4, orow, n_valid);
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(d_empty0 + 8u * d);
                }
            }
        }
    prod_done:;
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kTMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTTmemCols);
    }
}

// ------------------------------------------------------------------ host side

struct TcPlan {
    TcTrunkArgs A;
    size_t smem;
    bool stage_x;
};

// Shared-memory layout: A tile, weight ring, x ring (staged only), depthwise weights,
// column table, barriers.  Prefers deeper weight rings, then x rings of 2..4 stages.
bool layout_tc(TcTrunkArgs &A, bool stage_x, size_t *smem_out) {
    const TrunkProblem &P = A.P;
    const size_t limit = 227 * 1024;
    const size_t dw_bytes = ((size_t)P.C_in * (P.K + 1) * 4 + 15) / 16 * 16;
    const size_t tab_bytes = (size_t)A.heads * A.tabj * 8 + 16;   // + one pair read past the end
    for (int sw = 4; sw >= 2; --sw) {
        const size_t fixed = (size_t)A.off_w + (size_t)sw * A.w_stage_bytes + dw_bytes +
                             tab_bytes + 64 + 1024;
        int sx = 1;
        if (stage_x) {
            if (fixed + 8 * (2 * sw + 2 * 2) >= limit)
                continue;
            const size_t rest = limit - fixed - 8 * (2 * sw + 2 * 4);
            sx = (int)(rest / A.x_stage_bytes);
            if (sx > 4)
                sx = 4;
            if (sx < 2)
                continue;
        }
        A.wstages = sw;
        A.xstages = sx;
        A.off_x = A.off_w + (uint32_t)sw * A.w_stage_bytes;
        A.off_dw = A.off_x + (stage_x ? (uint32_t)sx * A.x_stage_bytes : 0u);
        A.off_tab = A.off_dw + (uint32_t)dw_bytes;
        A.off_bar = A.off_tab + (uint32_t)tab_bytes;
        size_t smem = (size_t)A.off_bar + 8 * (2 * sw + 2 * sx) + 64 + 1024;
        if (smem > limit)
            continue;
        // More than half the SM's shared memory: two CTAs (each holding all 512
        // tensor-memory columns) never share an SM.
        if (smem < 116 * 1024)
            smem = 116 * 1024;
        *smem_out = smem;
        return true;
    }
    return false;
}

bool make_tc_plan(const TrunkProblem &P, TcPlan *out) {
    TcTrunkArgs A;
    memset(&A, 0, sizeof(A));
    A.P = P;
    if (P.C_in % kTBK != 0 || P.C_in > kTMaxCin || P.J < 1)
        return false;
    A.nkb = P.C_in / kTBK;
    A.nbox = P.J >= kTMaxN ? kTMaxN : (P.J + 15) / 16 * 16;
    A.chunks_per_head = (P.J + kTMaxN - 1) / kTMaxN;
    A.heads = P.mask_out ? 2 : 1;
    A.chunks = A.heads * A.chunks_per_head;
    A.tabj = (P.J + 1) & ~1;
    A.tiles_l = (P.L_out + kTRows - 1) / kTRows;
    A.num_tiles = P.B * A.tiles_l;
    A.w_stage_bytes = (uint32_t)A.nbox * 128u;
    // The x window of a tile: 128 rows of taps, plus up to 7 positions of alignment.
    const int64_t need = (int64_t)(kTRows - 1) * P.stride + (int64_t)P.dilation * (P.K - 1) + 1 + 7;
    A.boxw = (int)((need + 7) / 8 * 8);
    A.x_stage_bytes = (uint32_t)kTBK * (uint32_t)(A.boxw > 0 ? A.boxw : 8) * 2u;
    A.off_a = 0;
    A.off_w = A.off_a + (uint32_t)A.nkb * kTABytes;
    bool stage_x = need <= kTBoxMax && P.L_in % 8 == 0 &&
                   (reinterpret_cast<uintptr_t>(P.x) & 15) == 0;
    size_t smem = 0;
    if (!(stage_x && layout_tc(A, true, &smem))) {
        stage_x = false;
        if (!layout_tc(A, false, &smem))
            return false;
    }
    out->A = A;
    out->smem = smem;
    out->stage_x = stage_x;
    return true;
}

template <class E, bool kStageX>
cudaError_t launch_tc(TcPlan pl, cudaStream_t stream) {
    const TrunkProblem &P = pl.A.P;
    alignas(64) CUtensorMap moff, mmask, mx;
    if (!encode_2d(&moff, TElem<E>::kTma, P.off_w, (uint64_t)P.C_in, (uint64_t)P.J, 2, kTBK,
                   (uint32_t)pl.A.nbox, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (P.mask_out) {
        if (!encode_2d(&mmask, TElem<E>::kTma, P.mask_w, (uint64_t)P.C_in, (uint64_t)P.J, 2,
                       kTBK, (uint32_t)pl.A.nbox, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    } else {
        mmask = moff;   // never read
    }
    if (kStageX) {
        if (!encode_2d(&mx, TElem<E>::kTma, P.x, (uint64_t)P.L_in, (uint64_t)P.B * P.C_in, 2,
                       (uint32_t)pl.A.boxw, kTBK, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    } else {
        mx = moff;      // never read
    }
    pl.A.status = device_status_ptr();
    if (!pl.A.status)
        return cudaErrorInvalidDevice;
    auto kern = trunk_tc_kernel<E, kStageX>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), (int)pl.smem);
    if (e != cudaSuccess)
        return e;
    const int sms = sm_count();
    if (sms <= 0)
        return cudaErrorNoDevice;
    const int grid = pl.A.num_tiles < sms ? pl.A.num_tiles : sms;
    timing_begin(stream);
    kern<<<grid, kTThreads, pl.smem, stream>>>(pl.A, moff, mmask, mx);
    timing_end(stream);
    return cudaGetLastError();
}

template <class E>
cudaError_t launch_tc_e(const TcPlan &pl, cudaStream_t stream) {
    return pl.stage_x ? launch_tc<E, true>(pl, stream) : launch_tc<E, false>(pl, stream);
}

}  // namespace

bool trunk_tc_supported(const TrunkProblem &P) {
    if (P.dtype != DCN1D_BF16 && P.dtype != DCN1D_F16)
        return false;
    if ((reinterpret_cast<uintptr_t>(P.off_w) & 15) ||
        (P.mask_out && (reinterpret_cast<uintptr_t>(P.mask_w) & 15)))
        return false;   // TMA sources start on 16 bytes
    if ((int64_t)P.offset_groups * P.L_out * P.K >= ((int64_t)1 << 31))
        return false;   // column offsets are int32
    TcPlan pl;
    return make_tc_plan(P, &pl);
}

cudaError_t launch_trunk(const TrunkProblem &P, cudaStream_t stream, const char **kernel) {
    if (trunk_tc_supported(P)) {
        TcPlan pl;
        make_tc_plan(P, &pl);
        *kernel = "trunk_tcgen05";
        return P.dtype == DCN1D_F16 ? launch_tc_e<__half>(pl, stream)
                                    : launch_tc_e<__nv_bfloat16>(pl, stream);
    }
    *kernel = "trunk_simt";
    switch (P.dtype) {
    case DCN1D_F32: return launch_simt<float>(P, stream);
    case DCN1D_BF16: return launch_simt<__nv_bfloat16>(P, stream);
    case DCN1D_F16: return launch_simt<__half>(P, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace dcn1d
