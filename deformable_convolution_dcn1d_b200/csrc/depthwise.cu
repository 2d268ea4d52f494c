// Depthwise kernel (groups == C_in == C_out): out[b,c,l] = bias[c] +
// sum_k w[c,0,k] * m * lerp(x[b,c,:], pos(l,k)).  There is no contraction
// across channels, so the op is bound by HBM: x, offsets, mask and out should
// each cross the bus once, and the per-output instruction count must stay
// below what the HBM rate leaves (~55 thread-instructions per output on B200
// at full bandwidth for K=3 bf16).
//
// One CTA owns one (b, c) row and a tile of TL consecutive outputs.
//  1. The x window its taps can reach (receptive fields plus a margin for
//     deformed taps) is staged in shared memory as neighbour PAIRS
//     (x[i], x[i+1]) in fp32, read from DRAM with 16-byte loads and zero
//     outside the signal, so one 8-byte shared load gives both neighbours.
//  2. Lane j of each warp owns output l0 + j (+ 32*warp, + 256*iteration):
//     lanes touch consecutive offsets (coalesced) and gather pairs at nearly
//     consecutive positions (few bank conflicts).  Taps whose pair lies outside
//     the window (an offset beyond the margin) read global memory instead, so
//     any offset value is handled.
// The floor is the conversion-free fast floor (exact for |pos| < 2^22, the
// range this kernel is selected for).
#include "common.cuh"
#include "sampler.cuh"

namespace dcn1d {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;   // outputs per thread per iteration (their loads go out together)

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
    int TL;          // outputs per tile
    int tiles;       // tiles per row
    int margin;      // extra positions staged on each side for deformed taps
    int win_elems;   // shared-memory window length (pairs)
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

template <class T, int K, bool UNC, bool MASK>
__global__ void __launch_bounds__(kThreads) depthwise_kernel(DwArgs A) {
    extern __shared__ __align__(16) float2 xp[];   // xp[r] = (X(wlo + r), X(wlo + r + 1))
    const Problem &P = A.P;
    constexpr int VN = Vec<T>::n;

    const int tile = blockIdx.x % A.tiles;
    const int bc = blockIdx.x / A.tiles;   // b * C + c
    const int c = bc % P.C_in;
    const int b = bc / P.C_in;
    const int l0 = tile * A.TL;
    const int l1 = min(l0 + A.TL, P.L_out);
    const int span = P.dilation * (K - 1);

    const T *xrow = static_cast<const T *>(P.x) + (int64_t)bc * P.L_in;
    // Window [wlo, wlo + wn): wlo rounded down to a multiple of VN for aligned vectors.
    int wlo = l0 * P.stride - P.padding - A.margin;
    wlo = (wlo >= 0) ? (wlo / VN) * VN : -(((-wlo) + VN - 1) / VN) * VN;
    const int whi_needed = (l1 - 1) * P.stride - P.padding + span + 2 + A.margin;
    const int wn = min(A.win_elems, ((whi_needed - wlo) + VN - 1) / VN * VN);

    // ---- 1. stage the window as neighbour pairs
    const bool xvec = ((reinterpret_cast<uintptr_t>(xrow) & 15) == 0);
    for (int v = threadIdx.x; v < wn / VN; v += kThreads) {
        const int p0 = wlo + v * VN;
        float raw[VN + 1];
        if (xvec && p0 >= 0 && p0 + VN <= P.L_in) {
            float tmp[8];
            unpack16(__ldg(reinterpret_cast<const uint4 *>(xrow + p0)), tmp,
                     static_cast<const T *>(nullptr));
#pragma unroll
            for (int j = 0; j < VN; ++j)
                raw[j] = tmp[j];
        } else {
#pragma unroll
            for (int j = 0; j < VN; ++j) {
                const int p = p0 + j;
                raw[j] = (p >= 0 && p < P.L_in) ? ld_f32(xrow + p) : 0.0f;
            }
        }
        const int pn = p0 + VN;
        raw[VN] = (pn >= 0 && pn < P.L_in) ? ld_f32(xrow + pn) : 0.0f;
#pragma unroll
        for (int j = 0; j < VN; ++j)
            xp[v * VN + j] = make_float2(raw[j], raw[j + 1]);
    }

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
    const float spanf = (float)span;
    T *orow_out = static_cast<T *>(P.out) + (int64_t)bc * P.L_out;
    __syncthreads();

    // ---- 2. outputs: lane-consecutive, kUnroll per thread per iteration
    const float step_f = (float)(kThreads * P.stride);   // start advance between a thread's outputs
    for (int lb = l0 + threadIdx.x; lb < l1; lb += kThreads * kUnroll) {
        float of[kUnroll][K], mk[kUnroll][K];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int l = lb + u * kThreads;
#pragma unroll
            for (int k = 0; k < K; ++k) {
                of[u][k] = (l < l1) ? ld_f32(offp + (int64_t)l * K + k) : 0.0f;
                if (MASK)
                    mk[u][k] = (l < l1) ? ld_f32(maskp + (int64_t)l * K + k) : 0.0f;
            }
        }
        float startf = (float)(lb * P.stride - P.padding);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int l = lb + u * kThreads;
            float acc = bias;
#pragma unroll
            for (int k = 0; k < K; ++k) {
                float pos = __fadd_rn(__fadd_rn(startf, kd[k]), of[u][k]);
                if (!UNC)
                    pos = fminf(fmaxf(pos, startf), __fadd_rn(startf, spanf));
                const Tap t = tap_floor_fast(pos);
                const unsigned r = (unsigned)t.i0 - (unsigned)wlo;   // wraps when outside
                float2 x01;
                if (r < (unsigned)(wn - 1)) {
                    x01 = xp[r];
                } else {
                    x01.x = (t.i0 >= 0 && t.i0 < P.L_in) ? ld_f32(xrow + t.i0) : 0.0f;
                    x01.y = (t.i0 >= -1 && t.i0 < P.L_in - 1) ? ld_f32(xrow + t.i0 + 1) : 0.0f;
                }
                float v = __fmaf_rn(t.f, __fsub_rn(x01.y, x01.x), x01.x);
                if (MASK)
                    v = __fmul_rn(v, mk[u][k]);
                acc = __fmaf_rn(wk[k], v, acc);
            }
            if (l < l1)
                orow_out[l] = from_f32<T>(acc);
            startf = __fadd_rn(startf, step_f);
        }
    }
}

template <class T, int K, bool UNC, bool MASK>
cudaError_t launch_kum(const Problem &P, cudaStream_t stream) {
    constexpr int VN = Vec<T>::n;
    DwArgs A;
    A.P = P;
    A.margin = UNC ? 32 : 0;
    const int span = P.dilation * (K - 1);
    // Window of a tile of TL outputs: the reach of its taps plus the margin on both sides,
    // plus slack for rounding its start down to a vector boundary.
    auto win_elems = [&](int TL) -> int64_t {
        return ((int64_t)(TL - 1) * P.stride + span + 2 + 2 * A.margin + VN + VN - 1) / VN * VN +
               VN;
    };
    int TL = 4096;
    while (TL > 32 && win_elems(TL) * (int64_t)sizeof(float2) > 48 * 1024)
        TL /= 2;
    if (TL >= P.L_out)
        TL = P.L_out;
    A.TL = TL;
    A.tiles = (P.L_out + TL - 1) / TL;
    A.win_elems = (int)win_elems(TL);
    const size_t smem = (size_t)A.win_elems * sizeof(float2);
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
    if (!(P.groups == P.C_in && P.C_out == P.C_in))
        return false;
    if (!(P.K == 1 || P.K == 2 || P.K == 3 || P.K == 4 || P.K == 5 || P.K == 7 || P.K == 9))
        return false;
    if (!fast_floor_ok(P))
        return false;
    // The window of the smallest tile (32 outputs) must fit in 48 KB of shared memory.
    const int64_t win = 31LL * P.stride + (int64_t)P.dilation * (P.K - 1) + 2 + 64 + 32;
    return win * (int64_t)sizeof(float2) <= 48 * 1024;
}

cudaError_t launch_depthwise(const Problem &P, cudaStream_t stream) {
    if (P.dtype == DCN1D_F32)
        return launch_t<float>(P, stream);
    return launch_t<__nv_bfloat16>(P, stream);
}

}  // namespace dcn1d
