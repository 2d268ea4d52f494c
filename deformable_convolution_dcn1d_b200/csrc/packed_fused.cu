// PackedDeformConv1d's whole forward in ONE kernel, for the depthwise layer of the
// "dc1d (DeformConv1d)" page's PackedDeformConv1d example (groups == offset_groups ==
// C_in == C_out): the offsets and the mask it predicts never reach global memory.
//
// Per tile of 128 output positions of one batch element (TMEM lane = position):
//   1. the x window of every channel (the tile's receptive fields, plus a margin when
//      unconstrained) is staged in shared memory by TMA, one 64-channel block per stage
//      of a ring one block deeper than a tile needs (a block's stage is refilled for the
//      next tile as soon as the chunks reading it are drained);
//   2. sixteen producer warps form the trunk's depthwise output
//        t[c, l] = dw_b[c] + sum_k dw_w[c, k] * x[c, l*s - p + k*d]
//      in fp32 from that window, round it once to the input type and write it straight
//      into tensor memory as the A operand of the pointwise heads ("PackedDeformConv1d":
//      a depthwise-separable block; "Modulation (DCNv2)": a second, sigmoid head);
//   3. one thread issues tcgen05.mma (M = 128, K = 16, A from tensor memory, B = a
//      pointwise-weight tile streamed by TMA) for one CHUNK of channels at a time: the
//      K offset columns and the K mask columns of cpc consecutive channels, accumulated
//      in fp32 into one of two tensor-memory buffers;
//   4. while the next chunk's MMAs run, the same sixteen warps drain the chunk: per
//      (position, channel) they add the head biases, apply the sigmoid, round the
//      predicted offset and mask to the input type (the tensors the layer hands on),
//      then sample the channel's row of the staged x window at each tap (the deformable
//      convolution's floor / fraction / clamp, fp32 interpolation) and write
//      out[b, c, l] = bias[c] + sum_k w[c, k] * m_k * x_interp(pos_k).
// Taps outside the staged window (unconstrained offsets past the margin) read x from
// global memory.  Every wait is bounded (sm100.cuh).
#include <string.h>

#include "common.cuh"
#include "sampler.cuh"
#include "sm100.cuh"

namespace dcn1d {

namespace {

constexpr int kFRows = 128;                // output positions per tile = TMEM lanes
constexpr int kFBK = 64;                   // channels per k-block of the head contraction
constexpr int kFProd = 16;                 // producer / drain warps
constexpr int kFWTma = 16, kFMma = 17, kFXTma = 18;
constexpr int kFThreads = 19 * 32;
constexpr uint32_t kFTmemCols = 512;
constexpr int kFMaxCin = 256;              // x windows of every channel, double-buffered
constexpr int kFBoxMax = 256;              // widest x window one TMA box holds
constexpr uint64_t kFWaitNs = 2000000000ull;   // 2 s
constexpr int kFCw = 8;                    // channels per drain warp and chunk

struct FusedArgs {
    TrunkProblem T;          // x, trunk weights, J = C_in * K (off_out / mask_out unused)
    const void *w, *bias;    // deformable depthwise weight [C, 1, K] and bias [C] (or NULL)
    void *out;               // [B, C, L_out]
    int unconstrained;
    int nkb;                 // C_in / 64
    int cpc;                 // channels per chunk (4 drain warps per lane quarter x kFCw)
    int N;                   // MMA N: cpc * K * heads
    int heads, chunks;       // 1 or 2; C_in / cpc
    int tiles_l, num_tiles;
    int boxw, margin;        // x window width (positions) and its margin per side
    int wstages;
    uint32_t colD1, colA;    // tensor-memory columns: D buffers at 0 and colD1, A at colA
    int xstages;             // x ring depth (>= nkb + 1)
    uint32_t w_stage_bytes, x_stage_bytes;
    uint32_t off_x, off_w, off_par, off_bar;   // shared-memory layout
    unsigned int *status;
};

template <class E>
struct FElem;

template <>
struct FElem<__nv_bfloat16> {
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
    // v rounded to the element type and back (the value a tensor of that type holds)
    static __device__ __forceinline__ float round(float v) {
        return __bfloat162float(__float2bfloat16_rn(v));
    }
    // both rounded with one paired conversion (the same value per element)
    static __device__ __forceinline__ float2 round2(float2 v) {
        const uint32_t u = pack(v.x, v.y);
        return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    }
};

template <>
struct FElem<__half> {
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
    static __device__ __forceinline__ float round(float v) {
        return __half2float(__float2half_rn(v));
    }
    static __device__ __forceinline__ float2 round2(float2 v) {
        return __half22float2(__floats2half2_rn(v.x, v.y));
    }
};

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// The logistic function through the hardware tanh: sigmoid(z) = (1 + tanh(z/2)) / 2,
// tanh.approx.f32 being accurate to about 2^-11 relative (inside the 16-bit rounding
// of the mask the layer hands on).
__device__ __forceinline__ float fsigmoid(float z) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
    return fmaf(0.5f, t, 0.5f);
}

// 8 consecutive 32-bit tensor-memory columns of this thread's lane.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t *v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ int floor8(int w) {
    return w >= 0 ? (w / 8) * 8 : -(((-w) + 7) / 8) * 8;
}

// Shared-memory parameter block (fp32): dw_w [C*K], dw_b [C], w [C*K], bias [C],
// off_b [J], mask_b [J].
// The layer's small parameters in shared memory (fp32).  dww [C][K] and dwb, fb [C] in
// channel order; fw, offb, maskb per channel PAIR and tap, [C/2][K][2], so the drain reads
// the values of its two channels for one tap with one 8-byte load (pair_at).
struct Par {
    const float *dww, *dwb, *fw, *fb, *offb, *maskb;
};

__host__ __device__ __forceinline__ int pair_at(int c, int k, int K) {
    return ((c >> 1) * K + k) * 2 + (c & 1);
}

__device__ __forceinline__ Par par_of(const float *base, int C, int K) {
    Par p;
    p.dww = base;
    p.dwb = p.dww + C * K;
    p.fw = p.dwb + C;
    p.fb = p.fw + C * K;
    p.offb = p.fb + C;
    p.maskb = p.offb + C * K;
    return p;
}

template <class E, int K, bool MASKHEAD, bool UNC>
__global__ void __launch_bounds__(kFThreads, 1)
    packed_fused_kernel(const __grid_constant__ FusedArgs A,
                        const __grid_constant__ CUtensorMap map_off,
                        const __grid_constant__ CUtensorMap map_mask,
                        const __grid_constant__ CUtensorMap map_x) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const TrunkProblem &T = A.T;
    const int C = T.C_in;
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint32_t sraw = smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - sraw);
    const uint32_t x_s0 = sbase + A.off_x;
    const uint32_t w_s0 = sbase + A.off_w;
    float *par_s = reinterpret_cast<float *>(smem + A.off_par);
    const uint32_t bar0 = sbase + A.off_bar;
    const int SW = A.wstages;
    auto w_full = [&](int s) { return bar0 + 8u * s; };
    auto w_empty = [&](int s) { return bar0 + 8u * (SW + s); };
    const int SX = A.xstages;
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

    {   // parameters, widened to fp32 once per CTA
        const E *dww = static_cast<const E *>(T.dw_w);
        const E *dwb = static_cast<const E *>(T.dw_b);
        const E *fw = static_cast<const E *>(A.w);
        const E *fb = static_cast<const E *>(A.bias);
        const E *ob = static_cast<const E *>(T.off_b);
        const E *mb = static_cast<const E *>(T.mask_b);
        float *w = par_s;   // the layout of par_of
        for (int i = threadIdx.x; i < C * K; i += kFThreads) {
            const int pi = pair_at(i / K, i % K, K);
            w[i] = ld_f32(dww + i);                                    // dw_w
            w[C * K + C + pi] = ld_f32(fw + i);                        // w
            w[2 * C * K + 2 * C + pi] = ob ? ld_f32(ob + i) : 0.0f;    // off_b
            w[3 * C * K + 2 * C + pi] = mb ? ld_f32(mb + i) : 0.0f;    // mask_b
        }
        for (int i = threadIdx.x; i < C; i += kFThreads) {
            w[C * K + i] = dwb ? ld_f32(dwb + i) : 0.0f;              // dw_b
            w[2 * C * K + C + i] = fb ? ld_f32(fb + i) : 0.0f;        // bias
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < SW; ++s) {
            mbar_init(w_full(s), 1);
            mbar_init(w_empty(s), 1);
        }
        for (int s = 0; s < SX; ++s) {
            mbar_init(x_full(s), 1);
            mbar_init(x_empty(s), kFProd);    // every producer warp reads every block
        }
        mbar_init(a_full, kFProd);
        mbar_init(a_empty, 1);
        for (int d = 0; d < 2; ++d) {
            mbar_init(d_full0 + 8u * d, 1);
            mbar_init(d_empty0 + 8u * d, kFProd);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kFMma) {
        tmem_alloc(smem_u32(tmem_holder), kFTmemCols);
        tc_fence_before();
    }
    if (warp == kFWTma && lane == 0) {
        tma_prefetch_desc(&map_off);
        if (MASKHEAD)
            tma_prefetch_desc(&map_mask);
    }
    if (warp == kFXTma && lane == 0)
        tma_prefetch_desc(&map_x);
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const BoundedWait wait{abort_flag, kFWaitNs, A.status};
    const int KC = A.cpc * K;          // columns of one head in a chunk

    if (warp == kFWTma) {
        // ------------------------------------------------------------ head weight tiles
        if (lane == 0) {
            uint32_t it = 0;
            for (int t = blockIdx.x; t < A.num_tiles; t += gridDim.x)
                for (int c = 0; c < A.chunks; ++c)
                    for (int kb = 0; kb < A.nkb; ++kb, ++it) {
                        const int s = it % SW;
                        const uint32_t ph = (it / SW) & 1u;
                        if (!wait(w_empty(s), ph ^ 1u))
                            goto wtma_done;
                        mbar_arrive_expect_tx(w_full(s), A.w_stage_bytes);
                        const uint32_t dst = w_s0 + s * A.w_stage_bytes;
                        tma_load_2d(dst, &map_off, kb * kFBK, c * KC, w_full(s));
                        if (MASKHEAD)
                            tma_load_2d(dst + (uint32_t)KC * 128u, &map_mask, kb * kFBK, c * KC,
                                        w_full(s));
                    }
        wtma_done:
            volatile int never = 0;
            const BoundedWait drain{&never, kFWaitNs, A.status};
            const uint32_t S = (uint32_t)SW;
            for (uint32_t j = (it > S ? it - S : 0); j < it; ++j)
                drain(w_full(j % S), (j / S) & 1u);
        }
    } else if (warp == kFXTma) {
        // ------------------------------------------------------------ x windows
        if (lane == 0) {
            uint32_t it = 0;
            for (int t = blockIdx.x; t < A.num_tiles; t += gridDim.x) {
                const int b = t / A.tiles_l;
                const int lbase = (t % A.tiles_l) * kFRows;
                const int wx0 = floor8(lbase * T.stride - T.padding - A.margin);
                for (int kb = 0; kb < A.nkb; ++kb, ++it) {
                    const int s = it % SX;
                    if (!wait(x_empty(s), ((it / SX) & 1u) ^ 1u))
                        goto xtma_done;
                    mbar_arrive_expect_tx(x_full(s), A.x_stage_bytes);
                    tma_load_2d(x_s0 + s * A.x_stage_bytes, &map_x, wx0, b * C + kb * kFBK,
                                x_full(s));
                }
            }
        xtma_done:
            volatile int never = 0;
            const BoundedWait drain{&never, kFWaitNs, A.status};
            const uint32_t S = (uint32_t)SX;
            for (uint32_t j = (it > S ? it - S : 0); j < it; ++j)
                drain(x_full(j % S), (j / S) & 1u);
        }
    } else if (warp == kFMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = FElem<E>::idesc(kFRows, A.N);
            uint32_t it = 0, cg = 0, tc = 0;
            for (int t = blockIdx.x; t < A.num_tiles; t += gridDim.x, ++tc) {
                if (!wait(a_full, tc & 1u))
                    goto mma_done;
                tc_fence_after();
                for (int c = 0; c < A.chunks; ++c, ++cg) {
                    const uint32_t d = cg & 1u;
                    const uint32_t dcol = d ? A.colD1 : 0u;
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
#pragma unroll
                        for (int kk = 0; kk < kFBK / 16; ++kk)
                            mma_bf16_ts(tmem + dcol, tmem + A.colA + 32u * kb + 8u * kk,
                                        sw128_kmajor_desc(wst + 32u * kk), idesc,
                                        (kb > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(w_empty(s));
                    }
                    mma_commit(d_full0 + 8u * d);
                }
                mma_commit(a_empty);   // the tile's A may be overwritten once this arrives
            }
        mma_done:
            mma_commit(drain_bar);
            volatile int never = 0;
            const BoundedWait drain{&never, kFWaitNs, A.status};
            drain(drain_bar, 0);
        }
    } else {
        // ------------------------------------------------------------ trunk + deformable drain
        const int q = warp % 4;          // TMEM lane quarter
        const int h = warp / 4;          // channel share within a k-block / chunk
        const int r = 32 * q + lane;     // tile row
        const Par p = par_of(par_s, C, K);
        const float spanf = (float)(T.dilation * (K - 1));
        uint32_t cg = 0, tc = 0;
        for (int t = blockIdx.x; t < A.num_tiles; t += gridDim.x, ++tc) {
            const int b = t / A.tiles_l;
            const int lbase = (t % A.tiles_l) * kFRows;
            const int l = lbase + r;
            const bool valid = l < T.L_out;
            const int wx0 = floor8(lbase * T.stride - T.padding - A.margin);
            const uint32_t it0 = tc * (uint32_t)A.nkb;       // ring index of block 0
            // stage address of channel block kb's window
            auto xblock = [&](int kb) {
                return x_s0 + ((it0 + (uint32_t)kb) % (uint32_t)SX) * A.x_stage_bytes;
            };
            const uint32_t rowb = (uint32_t)A.boxw * 2u;     // bytes per channel row
            const int start = l * T.stride - T.padding;      // first tap of row l
            const uint32_t rel0 = (uint32_t)(start - wx0);   // its window index (>= margin)
            if (!__all_sync(0xffffffffu, wait(a_empty, (tc & 1u) ^ 1u)))
                goto prod_done;
            // ---- trunk: this warp's 16 channels of every k-block into tensor memory
            for (int kb = 0; kb < A.nkb; ++kb) {
                const uint32_t itx = it0 + (uint32_t)kb;
                if (!__all_sync(0xffffffffu, wait(x_full(itx % SX), (itx / SX) & 1u)))
                    goto prod_done;
                const uint32_t xbuf = xblock(kb) - (uint32_t)(kb * kFBK) * rowb;
                uint32_t pk[8];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int c0 = kb * kFBK + 16 * h + 8 * half;
                    float acc[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        acc[i] = p.dwb[c0 + i];
#pragma unroll
                    for (int k = 0; k < K; ++k) {
                        const uint32_t xa =
                            xbuf + (uint32_t)c0 * rowb + (rel0 + (uint32_t)(k * T.dilation)) * 2u;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            acc[i] = fmaf(p.dww[(c0 + i) * K + k],
                                          FElem<E>::widen(lds_u16(xa + (uint32_t)i * rowb)),
                                          acc[i]);
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        pk[4 * half + i] = FElem<E>::pack(acc[2 * i], acc[2 * i + 1]);
                }
                tmem_st8(tmem + ((uint32_t)(32 * q) << 16) + A.colA + 32u * kb + 8u * h, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(a_full);
            // ---- per chunk: predicted offsets and mask, then the deformable convolution
            const E *xrow_g = static_cast<const E *>(T.x) + (int64_t)b * C * T.L_in;
            E *orow = static_cast<E *>(A.out) + (int64_t)b * C * T.L_out + l;
            const float startf = (float)start;
            for (int c = 0; c < A.chunks; ++c, ++cg) {
                const uint32_t d = cg & 1u;
                const int kbc = (c * A.cpc) / kFBK;     // the channel block this chunk reads
                const uint32_t xbuf = xblock(kbc) - (uint32_t)(kbc * kFBK) * rowb;
                const uint32_t dcol = d ? A.colD1 : 0u;
                if (!__all_sync(0xffffffffu, wait(d_full0 + 8u * d, (cg >> 1) & 1u)))
                    goto prod_done;
                tc_fence_after();
                // this warp's kFCw channels: kFCw*K columns of each head (a multiple of 8)
                uint32_t vo[kFCw * K], vm[MASKHEAD ? kFCw * K : 1];
                const uint32_t lanebase = tmem + ((uint32_t)(32 * q) << 16) + dcol;
                const int cofs = h * kFCw * K;
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    tmem_ld8(lanebase + (uint32_t)(cofs + 8 * j), vo + 8 * j);
                    if (MASKHEAD)
                        tmem_ld8(lanebase + (uint32_t)(KC + cofs + 8 * j), vm + 8 * j);
                }
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(d_empty0 + 8u * d);   // the buffer is free for chunk c + 2
                const int ch0 = c * A.cpc + h * kFCw;
                // two channels at a time: packed f32x2 arithmetic, the same roundings per
                // element as the scalar forms (and as the depthwise kernel's)
#pragma unroll
                for (int ip = 0; ip < kFCw / 2; ++ip) {
                    const int cA = ch0 + 2 * ip, cB = cA + 1;
                    const uint32_t xrA = xbuf + (uint32_t)cA * rowb, xrB = xrA + rowb;
                    float2 acc = *reinterpret_cast<const float2 *>(p.fb + cA);   // cA even
#pragma unroll
                    for (int k = 0; k < K; ++k) {
                        const int eA = (2 * ip) * K + k, eB = eA + K;   // register indices
                        const int pk = pair_at(cA, k, K);
                        const float2 z = __fadd2_rn(
                            make_float2(__uint_as_float(vo[eA]), __uint_as_float(vo[eB])),
                            *reinterpret_cast<const float2 *>(p.offb + pk));
                        const float2 off = FElem<E>::round2(z);
                        float2 m = make_float2(1.0f, 1.0f);
                        if (MASKHEAD) {
                            const float2 zm = __fadd2_rn(
                                make_float2(__uint_as_float(vm[MASKHEAD ? eA : 0]),
                                            __uint_as_float(vm[MASKHEAD ? eB : 0])),
                                *reinterpret_cast<const float2 *>(p.maskb + pk));
                            m = FElem<E>::round2(make_float2(fsigmoid(zm.x), fsigmoid(zm.y)));
                        }
                        const float bk = __fadd_rn(startf, (float)(k * T.dilation));
                        float2 pos = __fadd2_rn(make_float2(bk, bk), off);
                        if (!UNC) {
                            const float hi = __fadd_rn(startf, spanf);
                            pos.x = fminf(fmaxf(pos.x, startf), hi);
                            pos.y = fminf(fmaxf(pos.y, startf), hi);
                        }
                        const float2 tt = __fadd2_rd(pos, make_float2(kFloorMagic, kFloorMagic));
                        float2 f = __ffma2_rn(
                            __fadd2_rn(tt, make_float2(-kFloorMagic, -kFloorMagic)),
                            make_float2(-1.0f, -1.0f), pos);
                        const uint32_t wbits = kFloorMagicBits + (uint32_t)wx0;
                        const uint32_t relA = __float_as_uint(tt.x) - wbits;   // i0 - wx0
                        const uint32_t relB = __float_as_uint(tt.y) - wbits;
                        const uint32_t lim = (uint32_t)(A.boxw - 1);
                        float2 x0, x1;
                        if (relA < lim) {
                            x0.x = FElem<E>::widen(lds_u16(xrA + relA * 2u));
                            x1.x = FElem<E>::widen(lds_u16(xrA + relA * 2u + 2u));
                        } else {   // outside the staged window: exact floor, global loads
                            const Tap e = tap_floor_exact(pos.x);
                            const E *xg = xrow_g + (int64_t)cA * T.L_in;
                            x0.x = (e.i0 >= 0 && e.i0 < T.L_in) ? ld_f32(xg + e.i0) : 0.0f;
                            x1.x = (e.i0 >= -1 && e.i0 < T.L_in - 1) ? ld_f32(xg + e.i0 + 1)
                                                                     : 0.0f;
                            f.x = e.f;
                        }
                        if (relB < lim) {
                            x0.y = FElem<E>::widen(lds_u16(xrB + relB * 2u));
                            x1.y = FElem<E>::widen(lds_u16(xrB + relB * 2u + 2u));
                        } else {
                            const Tap e = tap_floor_exact(pos.y);
                            const E *xg = xrow_g + (int64_t)cB * T.L_in;
                            x0.y = (e.i0 >= 0 && e.i0 < T.L_in) ? ld_f32(xg + e.i0) : 0.0f;
                            x1.y = (e.i0 >= -1 && e.i0 < T.L_in - 1) ? ld_f32(xg + e.i0 + 1)
                                                                     : 0.0f;
                            f.y = e.f;
                        }
                        float2 v = __ffma2_rn(f, __ffma2_rn(x0, make_float2(-1.0f, -1.0f), x1),
                                              x0);
                        if (MASKHEAD)
                            v = __fmul2_rn(v, m);
                        acc = __ffma2_rn(*reinterpret_cast<const float2 *>(p.fw + pk), v, acc);
                    }
                    if (valid) {
                        orow[(int64_t)cA * T.L_out] = from_f32<E>(acc.x);
                        orow[(int64_t)cB * T.L_out] = from_f32<E>(acc.y);
                    }
                }
                // the chunk that finishes a channel block releases its stage
                if ((((c + 1) * A.cpc) % kFBK) == 0) {
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(x_empty((it0 + (uint32_t)kbc) % (uint32_t)SX));
                }
            }
        }
    prod_done:;
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kFMma) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kFTmemCols);
    }
}

// ------------------------------------------------------------------ host side

struct FusedPlan {
    FusedArgs A;
    size_t smem;
};

uint32_t round32(uint32_t v) { return (v + 31u) / 32u * 32u; }

bool make_fused_plan(const TrunkProblem &T, const Problem &P, FusedPlan *out) {
    FusedArgs A;
    memset(&A, 0, sizeof(A));
    A.T = T;
    const int C = T.C_in, K = T.K;
    if (C % kFBK != 0 || C > kFMaxCin)
        return false;
    A.heads = T.mask_w ? 2 : 1;
    A.nkb = C / kFBK;
    // A chunk: kFCw channels for each of the four drain warps of a lane quarter, i.e.
    // N = 4 * kFCw * K * heads head columns; the two accumulator buffers and the A operand
    // (C/2 columns) must fit in the tensor memory.
    A.cpc = 4 * kFCw;
    A.N = A.cpc * K * A.heads;
    if (K > 4 || A.N > 256 || A.N % 16 != 0 || C % A.cpc != 0)
        return false;
    if (2 * round32((uint32_t)A.N) + (uint32_t)C / 2 > kFTmemCols)
        return false;
    A.chunks = C / A.cpc;
    A.colD1 = round32((uint32_t)A.N);
    A.colA = 2 * A.colD1;
    A.unconstrained = P.unconstrained;
    A.margin = P.unconstrained ? 32 : 0;
    A.tiles_l = (T.L_out + kFRows - 1) / kFRows;
    A.num_tiles = T.B * A.tiles_l;
    const int64_t need = (int64_t)(kFRows - 1) * T.stride + (int64_t)T.dilation * (K - 1) + 2 +
                         2 * A.margin + 7;
    A.boxw = (int)((need + 7) / 8 * 8);
    if (A.boxw > kFBoxMax)
        return false;
    A.x_stage_bytes = (uint32_t)kFBK * (uint32_t)A.boxw * 2u;   // multiple of 1024
    A.xstages = A.nkb + 1;
    A.w_stage_bytes = (uint32_t)A.N * 128u;
    const size_t par_bytes = ((size_t)(4 * C * K + 2 * C) * 4 + 15) / 16 * 16;
    for (int sw = 4; sw >= 2; --sw) {
        A.wstages = sw;
        A.off_x = 0;
        A.off_w = (uint32_t)A.xstages * A.x_stage_bytes;
        A.off_par = A.off_w + (uint32_t)sw * A.w_stage_bytes;
        A.off_bar = A.off_par + (uint32_t)par_bytes;
        size_t smem = (size_t)A.off_bar + 8 * (2 * sw + 2 * A.xstages) + 64 + 1024;
        if (smem > 227 * 1024)
            continue;
        if (smem < 116 * 1024)
            smem = 116 * 1024;   // one CTA per SM (each holds all 512 TMEM columns)
        out->A = A;
        out->smem = smem;
        return true;
    }
    return false;
}

template <class E, int K, bool MASKHEAD, bool UNC>
cudaError_t launch_fused_k(FusedPlan pl, cudaStream_t stream) {
    const TrunkProblem &T = pl.A.T;
    alignas(64) CUtensorMap moff, mmask, mx;
    const uint32_t KC = (uint32_t)(pl.A.cpc * K);
    if (!encode_2d(&moff, FElem<E>::kTma, T.off_w, (uint64_t)T.C_in, (uint64_t)T.J, 2, kFBK, KC,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (MASKHEAD) {
        if (!encode_2d(&mmask, FElem<E>::kTma, T.mask_w, (uint64_t)T.C_in, (uint64_t)T.J, 2, kFBK,
                       KC, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    } else {
        mmask = moff;   // never read
    }
    if (!encode_2d(&mx, FElem<E>::kTma, T.x, (uint64_t)T.L_in, (uint64_t)T.B * T.C_in, 2,
                   (uint32_t)pl.A.boxw, kFBK, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    pl.A.status = device_status_ptr();
    if (!pl.A.status)
        return cudaErrorInvalidDevice;
    auto kern = packed_fused_kernel<E, K, MASKHEAD, UNC>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), (int)pl.smem);
    if (e != cudaSuccess)
        return e;
    const int sms = sm_count();
    if (sms <= 0)
        return cudaErrorNoDevice;
    const int grid = pl.A.num_tiles < sms ? pl.A.num_tiles : sms;
    timing_begin(stream);
    kern<<<grid, kFThreads, pl.smem, stream>>>(pl.A, moff, mmask, mx);
    timing_end(stream);
    return cudaGetLastError();
}

template <class E, int K>
cudaError_t launch_fused_e(const FusedPlan &pl, cudaStream_t stream) {
    const bool mh = pl.A.heads == 2, unc = pl.A.unconstrained != 0;
    if (mh)
        return unc ? launch_fused_k<E, K, true, true>(pl, stream)
                   : launch_fused_k<E, K, true, false>(pl, stream);
    return unc ? launch_fused_k<E, K, false, true>(pl, stream)
               : launch_fused_k<E, K, false, false>(pl, stream);
}

template <class E>
cudaError_t launch_fused_t(const FusedPlan &pl, cudaStream_t stream) {
    switch (pl.A.T.K) {
    case 1: return launch_fused_e<E, 1>(pl, stream);
    case 2: return launch_fused_e<E, 2>(pl, stream);
    case 3: return launch_fused_e<E, 3>(pl, stream);
    case 4: return launch_fused_e<E, 4>(pl, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool packed_fused_supported(const TrunkProblem &T, const Problem &P) {
    if (T.dtype != DCN1D_BF16 && T.dtype != DCN1D_F16)
        return false;
    if (!(P.groups == P.C_in && P.C_out == P.C_in && P.offset_groups == P.C_in))
        return false;   // the depthwise layer: channel c reads only x[c] and its own offsets
    if (T.K < 1 || T.K > 4 || !fast_floor_ok(P))
        return false;
    if (T.L_in % 8 != 0 || (reinterpret_cast<uintptr_t>(T.x) & 15) ||
        (reinterpret_cast<uintptr_t>(T.off_w) & 15) ||
        (T.mask_w && (reinterpret_cast<uintptr_t>(T.mask_w) & 15)))
        return false;   // TMA: 16-byte row strides and sources
    FusedPlan pl;
    return make_fused_plan(T, P, &pl);
}

cudaError_t launch_packed_fused(const TrunkProblem &T, const Problem &P, cudaStream_t stream) {
    FusedPlan pl;
    if (!make_fused_plan(T, P, &pl))
        return cudaErrorInvalidValue;
    pl.A.w = P.w;
    pl.A.bias = P.bias;
    pl.A.out = P.out;
    return T.dtype == DCN1D_F16 ? launch_fused_t<__half>(pl, stream)
                                : launch_fused_t<__nv_bfloat16>(pl, stream);
}

}  // namespace dcn1d
