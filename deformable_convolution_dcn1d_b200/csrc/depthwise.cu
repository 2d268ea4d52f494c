// Depthwise kernel (groups == C_in == C_out): out[b,c,l] = bias[c] +
// sum_k w[c,0,k] * m * lerp(x[b,c,:], pos(l,k)).  No contraction across
// channels, so the op is bound by HBM: every byte of x, offsets, mask and out
// should cross the bus once.
//
// One CTA owns one (b, c) row and a tile of TL consecutive outputs.
//  1. The x window the tile's taps can reach -- the receptive fields plus a
//     margin for deformed taps -- is staged in shared memory with 16-byte
//     loads (zero outside the signal), so the random-looking neighbour gathers
//     hit shared memory instead of DRAM.
//  2. Each thread owns groups of 8 consecutive outputs: it reads their 8*K
//     offsets (and mask) as K 16-byte vectors (bf16) straight from DRAM,
//     gathers both neighbours of every tap from the window, and writes the 8
//     outputs with one 16-byte store.  A tap whose neighbours fall outside the
//     staged window (an offset beyond the margin) reads them from global
//     memory instead, so any offset value is handled.
// Partial groups at the end of a row, and rows whose alignment does not allow
// vector access, take the same arithmetic through scalar loads.
#include "common.cuh"
#include "sampler.cuh"

namespace dcn1d {
namespace {

constexpr int kThreads = 256;
constexpr int kGroup = 8;   // outputs per thread-iteration

template <class T>
struct Vec;   // 16 bytes of T
template <>
struct Vec<float> {
    static constexpr int n = 4;
};
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int n = 8;
};

struct DwArgs {
    Problem P;
    int TL;          // outputs per tile (multiple of kGroup)
    int tiles;       // tiles per row
    int margin;      // extra positions staged on each side for deformed taps
    int win_elems;   // shared-memory window length (elements)
};

__device__ __forceinline__ void unpack16(const uint4 &v, float (&o)[8], const __nv_bfloat16 *) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        o[2 * i] = f.x;
        o[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void unpack16(const uint4 &v, float (&o)[8], const float *) {
    o[0] = __uint_as_float(v.x);
    o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z);
    o[3] = __uint_as_float(v.w);
}

template <class T, int K>
__global__ void __launch_bounds__(kThreads) depthwise_kernel(DwArgs A) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *xs = reinterpret_cast<T *>(smem_raw);
    const Problem &P = A.P;
    constexpr int VN = Vec<T>::n;   // elements per 16-byte vector

    const int tile = blockIdx.x % A.tiles;
    const int bc = blockIdx.x / A.tiles;   // b * C + c
    const int c = bc % P.C_in;
    const int b = bc / P.C_in;
    const int l0 = tile * A.TL;
    const int l1 = min(l0 + A.TL, P.L_out);
    const int span = P.dilation * (K - 1);
    const bool unc = P.unconstrained != 0;

    const T *xrow = static_cast<const T *>(P.x) + (int64_t)bc * P.L_in;
    // Window [wlo, wlo + win_elems): wlo rounded down to a multiple of VN.
    int wlo = l0 * P.stride - P.padding - A.margin;
    wlo = (wlo >= 0) ? (wlo / VN) * VN : -(((-wlo) + VN - 1) / VN) * VN;
    const int whi_needed = (l1 - 1) * P.stride - P.padding + span + 2 + A.margin;
    const int wn = min(A.win_elems, ((whi_needed - wlo) + VN - 1) / VN * VN);

    // ---- 1. stage the x window
    const bool xvec = ((reinterpret_cast<uintptr_t>(xrow) & 15) == 0);
    for (int v = threadIdx.x; v < wn / VN; v += kThreads) {
        const int p0 = wlo + v * VN;
        if (xvec && p0 >= 0 && p0 + VN <= P.L_in) {
            *reinterpret_cast<uint4 *>(xs + v * VN) =
                __ldg(reinterpret_cast<const uint4 *>(xrow + p0));
        } else {
#pragma unroll
            for (int j = 0; j < VN; ++j) {
                const int p = p0 + j;
                xs[v * VN + j] = (p >= 0 && p < P.L_in) ? xrow[p] : from_f32<T>(0.0f);
            }
        }
    }

    // Per-row constants.
    const int og = c / P.cin_per_og;
    const int64_t orow = ((int64_t)b * P.offset_groups + og) * P.L_out;   // in taps / K
    const T *offp = static_cast<const T *>(P.off) + orow * K;
    const T *maskp = P.mask ? static_cast<const T *>(P.mask) + orow * K : nullptr;
    float wk[K];
#pragma unroll
    for (int k = 0; k < K; ++k)
        wk[k] = ld_f32(static_cast<const T *>(P.w) + (int64_t)c * K + k);
    const float bias = P.bias ? ld_f32(static_cast<const T *>(P.bias) + c) : 0.0f;
    T *orow_out = static_cast<T *>(P.out) + (int64_t)bc * P.L_out;
    const bool ovec = ((reinterpret_cast<uintptr_t>(offp) & 15) == 0) &&
                      (!maskp || (reinterpret_cast<uintptr_t>(maskp) & 15) == 0) &&
                      ((reinterpret_cast<uintptr_t>(orow_out) & 15) == 0) &&
                      ((l0 % kGroup) == 0);
    __syncthreads();

    // Neighbour pair of one tap: from the window when inside it, else global.
    auto gather = [&](Tap t) -> float {
        const long long r = (long long)t.i0 - wlo;   // 64-bit: i0 may be near INT_MIN/MAX
        float x0, x1;
        if (r >= 0 && r < wn - 1) {
            x0 = to_f32(xs[r]);
            x1 = to_f32(xs[r + 1]);
        } else {
            x0 = (t.i0 >= 0 && t.i0 < P.L_in) ? ld_f32(xrow + t.i0) : 0.0f;
            x1 = (t.i0 >= -1 && t.i0 < P.L_in - 1) ? ld_f32(xrow + t.i0 + 1) : 0.0f;
        }
        return __fadd_rn(__fmul_rn(__fsub_rn(1.0f, t.f), x0), __fmul_rn(t.f, x1));
    };

    // ---- 2. groups of 8 outputs
    const int ngroups = (l1 - l0) / kGroup;
    if (ovec) {
        constexpr int NV = kGroup * K / VN;   // 16-byte vectors of offsets per group
        static_assert((kGroup * K) % VN == 0, "group of taps must be whole vectors");
        for (int gi = threadIdx.x; gi < ngroups; gi += kThreads) {
            const int lg = l0 + gi * kGroup;
            float of[kGroup * K], mk[kGroup * K];
            const uint4 *ov = reinterpret_cast<const uint4 *>(offp + (int64_t)lg * K);
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                float tmp[8];
                unpack16(__ldg(ov + j), tmp, static_cast<const T *>(nullptr));
#pragma unroll
                for (int u = 0; u < VN; ++u)
                    of[j * VN + u] = tmp[u];
            }
            if (maskp) {
                const uint4 *mv = reinterpret_cast<const uint4 *>(maskp + (int64_t)lg * K);
#pragma unroll
                for (int j = 0; j < NV; ++j) {
                    float tmp[8];
                    unpack16(__ldg(mv + j), tmp, static_cast<const T *>(nullptr));
#pragma unroll
                    for (int u = 0; u < VN; ++u)
                        mk[j * VN + u] = tmp[u];
                }
            }
            float res[kGroup];
#pragma unroll
            for (int i = 0; i < kGroup; ++i) {
                const int l = lg + i;
                const int start = l * P.stride - P.padding;
                float acc = bias;
#pragma unroll
                for (int k = 0; k < K; ++k) {
                    float v = gather(sample_tap(start, k, P.dilation, span, of[i * K + k], unc));
                    if (maskp)
                        v = __fmul_rn(v, mk[i * K + k]);
                    acc = __fmaf_rn(wk[k], v, acc);
                }
                res[i] = acc;
            }
            if constexpr (sizeof(T) == 2) {
                uint4 o;
                __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    h[i] = __floats2bfloat162_rn(res[2 * i], res[2 * i + 1]);
                *reinterpret_cast<uint4 *>(orow_out + lg) = o;
            } else {
                float4 *o4 = reinterpret_cast<float4 *>(orow_out + lg);
                o4[0] = make_float4(res[0], res[1], res[2], res[3]);
                o4[1] = make_float4(res[4], res[5], res[6], res[7]);
            }
        }
    }
    // Scalar path: everything when vectors are not allowed, else the ragged end.
    const int lstart = ovec ? l0 + ngroups * kGroup : l0;
    for (int l = lstart + threadIdx.x; l < l1; l += kThreads) {
        const int start = l * P.stride - P.padding;
        float acc = bias;
#pragma unroll
        for (int k = 0; k < K; ++k) {
            float v = gather(sample_tap(start, k, P.dilation, span, ld_f32(offp + (int64_t)l * K + k),
                                        unc));
            if (maskp)
                v = __fmul_rn(v, ld_f32(maskp + (int64_t)l * K + k));
            acc = __fmaf_rn(wk[k], v, acc);
        }
        orow_out[l] = from_f32<T>(acc);
    }
}

template <class T, int K>
cudaError_t launch_k(const Problem &P, cudaStream_t stream) {
    constexpr int VN = Vec<T>::n;
    DwArgs A;
    A.P = P;
    A.margin = P.unconstrained ? 32 : 0;
    const int span = P.dilation * (K - 1);
    // Shared-memory window of a tile of TL outputs: the reach of its taps plus the margin on
    // both sides, plus one vector of slack for rounding the start down to a vector boundary.
    auto win_elems = [&](int TL) -> int64_t {
        return ((int64_t)(TL - 1) * P.stride + span + 2 + 2 * A.margin + VN + VN - 1) / VN * VN +
               VN;
    };
    // Tile length: about 4096 outputs, fewer when the window would pass 48 KB.
    int TL = 4096;
    while (TL > kGroup && win_elems(TL) * (int64_t)sizeof(T) > 48 * 1024)
        TL /= 2;
    if (TL >= P.L_out)
        TL = ((P.L_out + kGroup - 1) / kGroup) * kGroup;
    A.TL = TL;
    A.tiles = (P.L_out + TL - 1) / TL;
    A.win_elems = (int)win_elems(TL);
    const size_t smem = (size_t)A.win_elems * sizeof(T);
    if (smem > 48 * 1024)
        return cudaErrorInvalidValue;   // host selection guarantees this does not happen
    const int64_t blocks = (int64_t)A.tiles * P.B * P.C_in;
    depthwise_kernel<T, K><<<(unsigned)blocks, kThreads, smem, stream>>>(A);
    return cudaGetLastError();
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
    if (!(P.groups == P.C_in && P.C_out == P.C_in))
        return false;
    if (!(P.K == 1 || P.K == 2 || P.K == 3 || P.K == 4 || P.K == 5 || P.K == 7 || P.K == 9))
        return false;
    // The window of the smallest tile (8 outputs) must fit in 48 KB of shared memory
    // (an upper bound of the launcher's window for any margin <= 32 and vector <= 8).
    const int es = P.dtype == DCN1D_F32 ? 4 : 2;
    const int64_t win = 7LL * P.stride + (int64_t)P.dilation * (P.K - 1) + 2 + 64 + 32;
    return win * es <= 48 * 1024;
}

cudaError_t launch_depthwise(const Problem &P, cudaStream_t stream) {
    if (P.dtype == DCN1D_F32)
        return launch_t<float>(P, stream);
    return launch_t<__nv_bfloat16>(P, stream);
}

}  // namespace dcn1d
