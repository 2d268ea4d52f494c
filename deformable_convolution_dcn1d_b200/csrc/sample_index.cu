// The sampling step alone: (i0, f) of every tap of an offsets tensor, from
// the same device functions the forward kernels use.  Used to test the integer
// decisions bit for bit.
#include "common.cuh"
#include "sampler.cuh"

namespace dcn1d {
namespace {

template <class T>
__global__ void __launch_bounds__(256) sample_index_kernel(const T *off, int64_t total, int L_out,
                                                           int K, int stride, int padding,
                                                           int dilation, int unconstrained,
                                                           int32_t *i0, float *frac) {
    int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= total)
        return;
    const int k = (int)(t % K);
    const int l = (int)((t / K) % L_out);
    // The fast floor the forward kernels use wherever it is exact; the conversion
    // floor elsewhere, so every tap matches the definition bit for bit.
    const float pos = tap_position(l * stride - padding, k, dilation, dilation * (K - 1),
                                   ld_f32(off + t), unconstrained != 0);
    Tap tp = (fabsf(pos) < (float)kFastPosLimit) ? tap_floor_fast(pos) : tap_floor_exact(pos);
    i0[t] = tp.i0;
    frac[t] = tp.f;
}

}  // namespace

cudaError_t launch_sample_index(const void *off, int dtype, int B, int G, int L_out, int K,
                                int L_in, int stride, int padding, int dilation,
                                int unconstrained, int32_t *i0, float *frac,
                                cudaStream_t stream) {
    (void)L_in;
    const int64_t total = (int64_t)B * G * L_out * K;
    const int threads = 256;
    const unsigned blocks = (unsigned)((total + threads - 1) / threads);
    if (dtype == DCN1D_F32)
        sample_index_kernel<float><<<blocks, threads, 0, stream>>>(
            static_cast<const float *>(off), total, L_out, K, stride, padding, dilation,
            unconstrained, i0, frac);
    else if (dtype == DCN1D_F16)
        sample_index_kernel<__half><<<blocks, threads, 0, stream>>>(
            static_cast<const __half *>(off), total, L_out, K, stride, padding, dilation,
            unconstrained, i0, frac);
    else
        sample_index_kernel<__nv_bfloat16><<<blocks, threads, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(off), total, L_out, K, stride, padding, dilation,
            unconstrained, i0, frac);
    return cudaGetLastError();
}

}  // namespace dcn1d
