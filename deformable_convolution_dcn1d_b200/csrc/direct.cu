// Generic direct kernel: one thread per output element.
//
// Correct for every valid shape and both dtypes; the specialised kernels
// (depthwise, tensor-core) take the shapes they cover and this one takes the
// rest.  Each thread walks its output's reduction over (ci, k) of its conv
// group in the weight's own order, samples x through the shared sampler and
// accumulates in fp32.  Consecutive threads own consecutive l, so the offset,
// mask and output accesses of a warp are coalesced.
#include "common.cuh"
#include "sampler.cuh"

namespace dcn1d {
namespace {

template <class T>
__global__ void __launch_bounds__(256) direct_kernel(Problem P, int64_t total) {
    int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    const T *x = static_cast<const T *>(P.x);
    const T *off = static_cast<const T *>(P.off);
    const T *mask = static_cast<const T *>(P.mask);
    const T *w = static_cast<const T *>(P.w);
    const T *bias = static_cast<const T *>(P.bias);
    T *out = static_cast<T *>(P.out);

    const int l = (int)(idx % P.L_out);
    const int64_t t = idx / P.L_out;
    const int co = (int)(t % P.C_out);
    const int b = (int)(t / P.C_out);
    const int g = co / P.cout_g;
    const int start = l * P.stride - P.padding;
    const int span = P.dilation * (P.K - 1);
    const bool unc = P.unconstrained != 0;

    float acc = bias ? ld_f32(bias + co) : 0.0f;
    for (int c = 0; c < P.cin_g; ++c) {
        const int ci = g * P.cin_g + c;
        const int og = ci / P.cin_per_og;
        const T *row = x + ((int64_t)b * P.C_in + ci) * P.L_in;
        const int64_t obase = (((int64_t)b * P.offset_groups + og) * P.L_out + l) * P.K;
        const T *wrow = w + ((int64_t)co * P.cin_g + c) * P.K;
        for (int k = 0; k < P.K; ++k) {
            Tap tp = sample_tap(start, k, P.dilation, span, ld_f32(off + obase + k), unc);
            float v = lerp_row(row, P.L_in, tp);
            if (mask)
                v = __fmul_rn(v, ld_f32(mask + obase + k));
            acc = __fmaf_rn(ld_f32(wrow + k), v, acc);
        }
    }
    out[idx] = from_f32<T>(acc);
}

}  // namespace

cudaError_t launch_direct(const Problem &P, cudaStream_t stream) {
    const int64_t total = (int64_t)P.B * P.C_out * P.L_out;
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    if (P.dtype == DCN1D_F32)
        direct_kernel<float><<<(unsigned)blocks, threads, 0, stream>>>(P, total);
    else if (P.dtype == DCN1D_F16)
        direct_kernel<__half><<<(unsigned)blocks, threads, 0, stream>>>(P, total);
    else
        direct_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, stream>>>(P, total);
    return cudaGetLastError();
}

}  // namespace dcn1d
