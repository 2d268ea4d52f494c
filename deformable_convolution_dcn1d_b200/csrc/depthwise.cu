// Depthwise kernel (groups == C_in == C_out): out[b,c,l] = bias[c] +
// sum_k w[c,0,k] * m * lerp(x[b,c,:], pos(l,k)).  There is no contraction
// across channels, so the op is bound by HBM: x, offsets, mask and out should
// each cross the bus once, and the per-output instruction count has to stay
// below what the HBM rate leaves (about 55 thread-instructions per output on
// B200 at full bandwidth for K=3 bf16).
//
// One CTA owns one (b, c) row and a tile of TL consecutive outputs.
//  1. The x window its taps can reach (receptive fields plus a margin for
//     deformed taps) is staged in shared memory as neighbour PAIRS: word r
//     holds (x[wlo+r], x[wlo+r+1]) -- two bf16 in one 32-bit word (fp32: a
//     float2) -- read from DRAM with 16-byte loads, zero outside the signal.
//     One shared load then gives both neighbours of a tap.
//  2. A thread owns groups of 8 consecutive outputs: their 8*K offsets (and
//     mask) arrive as 16-byte vectors and the 8 results leave as one 16-byte
//     store.  The arithmetic runs on output pairs with packed f32x2
//     instructions.  Taps whose pair lies outside the window (an offset beyond
//     the margin) read global memory instead, so any offset value is handled.
// The floor is the conversion-free fast floor (exact for |pos| < 2^22; the
// kernel is selected only for L_in < 2^22).
#include "common.cuh"
#include "sampler.cuh"

namespace dcn1d {
namespace {

constexpr int kThreads = 256;
constexpr int kGroup = 8;   // consecutive outputs per thread-iteration

template <class T>
struct Traits;
template <>
struct Traits<__nv_bfloat16> {
    static constexpr int VN = 8;   // elements per 16-byte vector
    using Word = uint32_t;         // one neighbour pair in the window
};
template <>
struct Traits<float> {
    static constexpr int VN = 4;
    using Word = float2;
};

struct DwArgs {
    Problem P;
    int TL;          // outputs per tile (multiple of kGroup, or the whole row)
    int tiles;       // tiles per row
    int margin;      // extra positions staged on each side for deformed taps
    int win_elems;   // window length in pairs
};

__device__ __forceinline__ float2 pair_floats(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ float2 pair_floats(float2 w) { return w; }

// Stage VN window pairs starting at position p0 (window index r0).
__device__ __forceinline__ void stage_pairs(uint32_t *xp, int r0, const __nv_bfloat16 *row, int p0,
                                            int L, bool vec_ok) {
    uint32_t w[5];
    if (vec_ok && p0 >= 0 && p0 + 8 <= L) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(row + p0));
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int p = p0 + 2 * i;
            const uint32_t lo = (p >= 0 && p < L) ? (uint32_t)__bfloat16_as_ushort(row[p]) : 0u;
            const uint32_t hi = (p + 1 >= 0 && p + 1 < L) ? (uint32_t)__bfloat16_as_ushort(row[p + 1]) : 0u;
            w[i] = lo | (hi << 16);
        }
    }
    const int pn = p0 + 8;
    w[4] = (pn >= 0 && pn < L) ? (uint32_t)__bfloat16_as_ushort(row[pn]) : 0u;
    uint4 a, b;   // pair(i) = (x[i], x[i+1]): even i is a whole word, odd i straddles two
    a.x = w[0];
    a.y = __byte_perm(w[0], w[1], 0x5432);
    a.z = w[1];
    a.w = __byte_perm(w[1], w[2], 0x5432);
    b.x = w[2];
    b.y = __byte_perm(w[2], w[3], 0x5432);
    b.z = w[3];
    b.w = __byte_perm(w[3], w[4], 0x5432);
    reinterpret_cast<uint4 *>(xp + r0)[0] = a;
    reinterpret_cast<uint4 *>(xp + r0)[1] = b;
}
__device__ __forceinline__ void stage_pairs(float2 *xp, int r0, const float *row, int p0, int L,
                                            bool vec_ok) {
    float x[5];
    if (vec_ok && p0 >= 0 && p0 + 4 <= L) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(row + p0));
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            x[i] = (p0 + i >= 0 && p0 + i < L) ? row[p0 + i] : 0.0f;
    }
    x[4] = (p0 + 4 >= 0 && p0 + 4 < L) ? row[p0 + 4] : 0.0f;
    float4 *dst = reinterpret_cast<float4 *>(xp + r0);
    dst[0] = make_float4(x[0], x[1], x[1], x[2]);
    dst[1] = make_float4(x[2], x[3], x[3], x[4]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ void store8(__nv_bfloat16 *dst, const float *r) {
    uint4 o;
    o.x = pack_bf16x2(r[0], r[1]);
    o.y = pack_bf16x2(r[2], r[3]);
    o.z = pack_bf16x2(r[4], r[5]);
    o.w = pack_bf16x2(r[6], r[7]);
    *reinterpret_cast<uint4 *>(dst) = o;
}
__device__ __forceinline__ void store8(float *dst, const float *r) {
    reinterpret_cast<float4 *>(dst)[0] = make_float4(r[0], r[1], r[2], r[3]);
    reinterpret_cast<float4 *>(dst)[1] = make_float4(r[4], r[5], r[6], r[7]);
}

template <class T, int K, bool UNC, bool MASK>
__global__ void __launch_bounds__(kThreads) depthwise_kernel(DwArgs A) {
    using Word = typename Traits<T>::Word;
    constexpr int VN = Traits<T>::VN;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Word *xp = reinterpret_cast<Word *>(smem_raw);   // xp[r] = (X(wlo + r), X(wlo + r + 1))
    const Problem &P = A.P;

    const int tile = blockIdx.x % A.tiles;
    const int bc = blockIdx.x / A.tiles;   // b * C + c
    const int c = bc % P.C_in;
    const int b = bc / P.C_in;
    const int l0 = tile * A.TL;
    const int l1 = min(l0 + A.TL, P.L_out);
    const int span = P.dilation * (K - 1);

    const T *xrow = static_cast<const T *>(P.x) + (int64_t)bc * P.L_in;
    // Window [wlo, wlo + wn): wlo rounded down to a multiple of 8 for aligned vectors.
    int wlo = l0 * P.stride - P.padding - A.margin;
    wlo = (wlo >= 0) ? (wlo / 8) * 8 : -(((-wlo) + 7) / 8) * 8;
    const int whi_needed = (l1 - 1) * P.stride - P.padding + span + 2 + A.margin;
    const int wn = min(A.win_elems, ((whi_needed - wlo) + 7) / 8 * 8);

    // ---- 1. stage the window as neighbour pairs
    const bool xvec = ((reinterpret_cast<uintptr_t>(xrow) & 15) == 0);
    for (int v = threadIdx.x; v < wn / VN; v += kThreads)
        stage_pairs(xp, v * VN, xrow, wlo + v * VN, P.L_in, xvec);

    // ---- per-row constants
    const int og = c / P.cin_per_og;
    const int64_t orow = ((int64_t)b * P.offset_groups + og) * P.L_out;
    const T *offp = static_cast<const T *>(P.off) + orow * K;
    const T *maskp = MASK ? static_cast<const T *>(P.mask) + orow * K : nullptr;
    float wk[K], kd[K];
#pragma unroll
    for (int k = 0; k < K; ++k) {
        wk[k] = ld_f32(static_cast<const T *>(P.w) + (int64_t)c * K + k);
        kd[k] = (float)(k * P.dilation);
    }
    const float bias = P.bias ? ld_f32(static_cast<const T *>(P.bias) + c) : 0.0f;
    const float sf = (float)P.stride;
    const float spanf = (float)span;
    T *orow_out = static_cast<T *>(P.out) + (int64_t)bc * P.L_out;
    const bool vec = ((reinterpret_cast<uintptr_t>(offp) & 15) == 0) &&
                     (!MASK || (reinterpret_cast<uintptr_t>(maskp) & 15) == 0) &&
                     ((reinterpret_cast<uintptr_t>(orow_out) & 15) == 0) && ((l0 % kGroup) == 0);
    // bits(t) - kWinBits = floor(pos) - wlo for t = RD(pos + 1.5*2^23).
    const unsigned kWinBits = kFloorMagicBits + (unsigned)wlo;
    __syncthreads();

    // Both neighbours of a tap whose floor is t (see tap_floor_fast); checked.
    auto gather = [&](float t, float pos, float &x0, float &x1) {
        const unsigned r = __float_as_uint(t) - kWinBits;
        if (r < (unsigned)(wn - 1)) {
            const float2 p = pair_floats(xp[r]);
            x0 = p.x;
            x1 = p.y;
        } else {   // beyond the staged window: exact floor, global loads
            const Tap e = tap_floor_exact(pos);
            x0 = (e.i0 >= 0 && e.i0 < P.L_in) ? ld_f32(xrow + e.i0) : 0.0f;
            x1 = (e.i0 >= -1 && e.i0 < P.L_in - 1) ? ld_f32(xrow + e.i0 + 1) : 0.0f;
        }
    };
    // Unchecked: the caller knows the pair is inside the window.
    auto gather_fast = [&](float t) -> Word {
        return xp[__float_as_uint(t) - kWinBits];
    };
    // Largest |offset| that keeps every tap of an output inside the window (margin),
    // as a bf16/fp32 bit threshold on |offset| bits.
    const float off_limit = (float)(A.margin - 1);

    // ---- 2. groups of 8 consecutive outputs, arithmetic on output pairs
    const int ngroups = vec ? (l1 - l0) / kGroup : 0;
    for (int gi = threadIdx.x; gi < ngroups; gi += kThreads) {
        const int lg = l0 + gi * kGroup;
        constexpr int NW = kGroup * K * (int)sizeof(T) / 4;   // 32-bit words of offsets per group
        uint32_t ow[NW], mw[MASK ? NW : 1];
        const uint4 *ov = reinterpret_cast<const uint4 *>(offp + (int64_t)lg * K);
#pragma unroll
        for (int j = 0; j < NW / 4; ++j) {
            const uint4 v = __ldg(ov + j);
            ow[4 * j] = v.x; ow[4 * j + 1] = v.y; ow[4 * j + 2] = v.z; ow[4 * j + 3] = v.w;
        }
        if constexpr (MASK) {
            const uint4 *mv = reinterpret_cast<const uint4 *>(maskp + (int64_t)lg * K);
#pragma unroll
            for (int j = 0; j < NW / 4; ++j) {
                const uint4 v = __ldg(mv + j);
                mw[4 * j] = v.x; mw[4 * j + 1] = v.y; mw[4 * j + 2] = v.z; mw[4 * j + 3] = v.w;
            }
        }
        // element e (= i*K + k) of the group's offsets / mask as a float
        auto elem = [&](const uint32_t *w, int e) -> float {
            if constexpr (sizeof(T) == 2)
                return (e & 1) ? __uint_as_float(w[e >> 1] & 0xFFFF0000u)
                               : __uint_as_float(w[e >> 1] << 16);
            else
                return __uint_as_float(w[e]);
        };
        // In unconstrained mode the window covers every tap with |offset| <= margin-1;
        // constrained taps are clamped into the receptive field, always inside.
        bool inside = true;
        if constexpr (UNC) {
            if constexpr (sizeof(T) == 2) {
                uint32_t amax = 0;
#pragma unroll
                for (int j = 0; j < NW; ++j)
                    amax = __vmaxu2(amax, ow[j] & 0x7FFF7FFFu);
                const uint32_t lim = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rz(off_limit));
                inside = ((amax & 0xFFFFu) <= lim) && ((amax >> 16) <= lim);
            } else {
                // On the bits of |offset|: NaN and inf patterns exceed every finite
                // one, so a NaN offset sends the warp to the checked path (a float
                // max would drop the NaN).
                uint32_t amax = 0;
#pragma unroll
                for (int j = 0; j < NW; ++j)
                    amax = max(amax, ow[j] & 0x7FFFFFFFu);
                inside = amax <= __float_as_uint(off_limit);
            }
        }
        const float s0 = (float)(lg * P.stride - P.padding);
        float res[kGroup];
        if (__all_sync(0xffffffffu, inside)) {
#pragma unroll
            for (int i = 0; i < kGroup; i += 2) {
                const float2 st = make_float2(__fadd_rn(s0, (float)i * sf),
                                              __fadd_rn(s0, (float)(i + 1) * sf));
                float2 acc = make_float2(bias, bias);
#pragma unroll
                for (int k = 0; k < K; ++k) {
                    float2 pos = __fadd2_rn(__fadd2_rn(st, make_float2(kd[k], kd[k])),
                                            make_float2(elem(ow, i * K + k), elem(ow, (i + 1) * K + k)));
                    if (!UNC) {
                        pos.x = fminf(fmaxf(pos.x, st.x), __fadd_rn(st.x, spanf));
                        pos.y = fminf(fmaxf(pos.y, st.y), __fadd_rn(st.y, spanf));
                    }
                    const float2 t = __fadd2_rd(pos, make_float2(kFloorMagic, kFloorMagic));
                    const float2 f = __ffma2_rn(__fadd2_rn(t, make_float2(-kFloorMagic, -kFloorMagic)),
                                                make_float2(-1.0f, -1.0f), pos);
                    const float2 pa = pair_floats(gather_fast(t.x));
                    const float2 pb = pair_floats(gather_fast(t.y));
                    const float2 x0 = make_float2(pa.x, pb.x), x1 = make_float2(pa.y, pb.y);
                    float2 v = __ffma2_rn(f, __ffma2_rn(x0, make_float2(-1.0f, -1.0f), x1), x0);
                    if constexpr (MASK)
                        v = __fmul2_rn(v, make_float2(elem(mw, i * K + k), elem(mw, (i + 1) * K + k)));
                    acc = __ffma2_rn(make_float2(wk[k], wk[k]), v, acc);
                }
                res[i] = acc.x;
                res[i + 1] = acc.y;
            }
        } else {
#pragma unroll
            for (int i = 0; i < kGroup; ++i) {
                const float st = __fadd_rn(s0, (float)i * sf);
                float acc = bias;
#pragma unroll
                for (int k = 0; k < K; ++k) {
                    float pos = __fadd_rn(__fadd_rn(st, kd[k]), elem(ow, i * K + k));
                    if (!UNC)
                        pos = fminf(fmaxf(pos, st), __fadd_rn(st, spanf));
                    const float t = __fadd_rd(pos, kFloorMagic);
                    const float f = __fsub_rn(pos, __fsub_rn(t, kFloorMagic));
                    float x0, x1;
                    gather(t, pos, x0, x1);
                    float v = __fmaf_rn(f, __fsub_rn(x1, x0), x0);
                    if constexpr (MASK)
                        v = __fmul_rn(v, elem(mw, i * K + k));
                    acc = __fmaf_rn(wk[k], v, acc);
                }
                res[i] = acc;
            }
        }
        store8(orow_out + lg, res);
    }

    // ---- scalar path: everything when vectors are not allowed, else the ragged end
    const int lstart = l0 + ngroups * kGroup;
    for (int l = lstart + threadIdx.x; l < l1; l += kThreads) {
        const float st = (float)(l * P.stride - P.padding);
        float acc = bias;
#pragma unroll
        for (int k = 0; k < K; ++k) {
            float pos = __fadd_rn(__fadd_rn(st, kd[k]), ld_f32(offp + (int64_t)l * K + k));
            if (!UNC)
                pos = fminf(fmaxf(pos, st), __fadd_rn(st, spanf));
            const float t = __fadd_rd(pos, kFloorMagic);
            const float f = __fsub_rn(pos, __fsub_rn(t, kFloorMagic));
            float x0, x1;
            gather(t, pos, x0, x1);
            float v = __fmaf_rn(f, __fsub_rn(x1, x0), x0);
            if constexpr (MASK)
                v = __fmul_rn(v, ld_f32(maskp + (int64_t)l * K + k));
            acc = __fmaf_rn(wk[k], v, acc);
        }
        orow_out[l] = from_f32<T>(acc);
    }
}

template <class T, int K, bool UNC, bool MASK>
cudaError_t launch_kum(const Problem &P, cudaStream_t stream) {
    using Word = typename Traits<T>::Word;
    DwArgs A;
    A.P = P;
    A.margin = UNC ? 32 : 0;
    const int span = P.dilation * (K - 1);
    // Window of a tile of TL outputs: the reach of its taps plus the margin on both sides,
    // plus slack for rounding its start down to a multiple of 8.
    auto win_elems = [&](int TL) -> int64_t {
        return ((int64_t)(TL - 1) * P.stride + span + 2 + 2 * A.margin + 7 + 7) / 8 * 8 + 8;
    };
    int TL = 4096;
    while (TL > 32 && win_elems(TL) * (int64_t)sizeof(Word) > 48 * 1024)
        TL /= 2;
    if (TL >= P.L_out)
        TL = P.L_out;
    A.TL = TL;
    A.tiles = (P.L_out + TL - 1) / TL;
    A.win_elems = (int)win_elems(TL);
    const size_t smem = (size_t)A.win_elems * sizeof(Word);
    if (smem > 48 * 1024)
        return cudaErrorInvalidValue;   // the host selection rule keeps this from happening
    const int64_t blocks = (int64_t)A.tiles * P.B * P.C_in;
    depthwise_kernel<T, K, UNC, MASK><<<(unsigned)blocks, kThreads, smem, stream>>>(A);
    return cudaGetLastError();
}

template <class T, int K>
cudaError_t launch_k(const Problem &P, cudaStream_t stream) {
    const bool m = P.mask != nullptr;
    if (P.unconstrained)
        return m ? launch_kum<T, K, true, true>(P, stream) : launch_kum<T, K, true, false>(P, stream);
    return m ? launch_kum<T, K, false, true>(P, stream) : launch_kum<T, K, false, false>(P, stream);
}

template <class T>
cudaError_t launch_t(const Problem &P, cudaStream_t stream) {
    switch (P.K) {
    case 1: return launch_k<T, 1>(P, stream);
    case 2: return launch_k<T, 2>(P, stream);
    case 3: return launch_k<T, 3>(P, stream);
    case 4: return launch_k<T, 4>(P, stream);
    case 5: return launch_k<T, 5>(P, stream);
    case 7: return launch_k<T, 7>(P, stream);
    case 9: return launch_k<T, 9>(P, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool depthwise_supported(const Problem &P) {
    if (P.dtype == DCN1D_F16)   // the window packing reads bf16 bit patterns
        return false;
    if (!(P.groups == P.C_in && P.C_out == P.C_in))
        return false;
    if (!(P.K == 1 || P.K == 2 || P.K == 3 || P.K == 4 || P.K == 5 || P.K == 7 || P.K == 9))
        return false;
    if (!fast_floor_ok(P))
        return false;
    // The window of the smallest tile (32 outputs) must fit in 48 KB of shared memory.
    const int64_t win = 31LL * P.stride + (int64_t)P.dilation * (P.K - 1) + 2 + 64 + 32;
    return win * 8 <= 48 * 1024;
}

cudaError_t launch_depthwise(const Problem &P, cudaStream_t stream) {
    if (P.dtype == DCN1D_F32)
        return launch_t<float>(P, stream);
    return launch_t<__nv_bfloat16>(P, stream);
}

}  // namespace dcn1d
