// Internal definitions shared by the kernels and the C-ABI host code.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dcn1d.h"

namespace dcn1d {

// A validated forward problem.  All sizes fit in int32 (checked on the host).
struct Problem {
    int B, C_in, L_in, C_out, K, L_out;
    int stride, padding, dilation, groups, offset_groups;   // padding: zeros before the signal
    int padding_right;                                      // zeros after it
    int unconstrained;
    int dtype;                 // dcn1d_dtype
    int cin_g, cout_g;         // channels per conv group (input, output)
    int cin_per_og;            // input channels per offset group
    const void *x, *off, *mask, *w, *bias;
    void *out;
};

__device__ __forceinline__ float ld_f32(const float *p) { return __ldg(p); }
__device__ __forceinline__ float ld_f32(const __nv_bfloat16 *p) { return __bfloat162float(__ldg(p)); }
__device__ __forceinline__ float ld_f32(const __half *p) { return __half2float(__ldg(p)); }
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(__half v) { return __half2float(v); }

template <class T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}
template <> __device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }

// The kernels that use the conversion-free floor (sampler.cuh) need the signal
// and its staged windows well inside (-2^22, 2^22): then any tap whose floor
// lands inside a window or the signal had |pos| < 2^22, where that floor is
// exact, and the bit patterns it yields for larger |pos| cannot alias a
// window index.
inline bool fast_floor_ok(const Problem &P) {
    return (int64_t)P.L_in + (int64_t)P.padding + P.padding_right < (1 << 21);
}

// Benchmark timing hook (dcn1d_set_timing_events): launchers call these right
// before and right after the launch of their main kernel; they record the
// events set for this host thread, if any, on `stream`.
void timing_begin(cudaStream_t stream);
void timing_end(cudaStream_t stream);

// Kernel launchers (each returns cudaGetLastError() of its launch).
cudaError_t launch_direct(const Problem &P, cudaStream_t stream);
bool depthwise_supported(const Problem &P);
cudaError_t launch_depthwise(const Problem &P, cudaStream_t stream);
// The device status word (bounded-wait failures) of the current device, as a
// device address to hand to kernels (NULL on failure), and its read-and-reset.
unsigned int *device_status_ptr();
cudaError_t read_and_clear_device_status(unsigned int *word);
bool tc_tf32_supported(const Problem &P);
// One launch, no workspace; split-K problems run as clusters of tc_tf32_splits(P) CTAs.
int tc_tf32_splits(const Problem &P);
cudaError_t launch_tc_tf32(const Problem &P, cudaStream_t stream);
bool tc_bf16_supported(const Problem &P);
cudaError_t launch_tc_bf16(const Problem &P, cudaStream_t stream);
// Test of the failure path: the tensor-core kernel with its loader switched off at
// compile time and every wait limited to wait_ns (bf16, K = 3, no mask only).
bool tc_bf16_stalled_supported(const Problem &P);
cudaError_t launch_tc_bf16_stalled(const Problem &P, uint64_t wait_ns, cudaStream_t stream);
// Backward (backward.cu): the upstream gradient and the wanted gradients (each
// output NULL when not wanted), all in the problem's dtype and its inputs' shapes.
// The tensor-core GEMM of the backward pass (gemm_tc.cu): C[z][m*c_sm + n*c_sn] (fp32) =
// sum over r < R and k < K of A[row_a(z, r) + m][k] * B[row_b(z, r) + n][k], A and B
// 16-bit K-major row-major arrays with `*_ld` elements per row and `*_rows` rows.
bool gemm_tc_supported(int dtype, const void *A, int64_t a_rows, int64_t a_ld, const void *B,
                       int64_t b_rows, int64_t b_ld);
cudaError_t launch_gemm_tc(int dtype, const void *A, int64_t a_rows, int64_t a_ld, int a_row0,
                           int a_row_z, int a_row_r, const void *B, int64_t b_rows, int64_t b_ld,
                           int b_row0, int b_row_z, int b_row_r, int M, int N, int K, int R,
                           int nz, float *C, int64_t c_sm, int64_t c_sn, int64_t c_sz,
                           cudaStream_t stream);
struct BackwardGrads {
    const void *gout;                    // [B, C_out, L_out]
    void *x, *off, *mask, *w, *bias;     // outputs
};
size_t backward_workspace(const Problem &P, const BackwardGrads &G);
bool backward_uses_tensor_cores(const Problem &P, const BackwardGrads &G);
// The backward's column-gradient GEMM with the sampling gradient fused into its drain
// (gemm_tc.cu; 16-bit, K in {3, 4, 5, 7, 9}): for conv group g, grad_x / grad_offsets /
// grad_mask accumulate into the fp32 buffers given (each may be NULL) and the sampled
// columns go to cols16 (or not, if NULL); goutT_g and wT_g as for the plain GEMM.
bool gemm_sample_supported(const Problem &P);
// The same GEMM on fp32 operands by three TF32 products (gemm_tc.cu): row strides multiples
// of 4 elements, 16-byte aligned bases.  flat_rpz > 0: the M rows of every z form one range
// (row m is row m of A; its output goes to C[(m / flat_rpz) * c_sz + (m % flat_rpz) * c_sm
// + n * c_sn]) and the per-z A offsets are not used.
bool gemm_x3_supported(const void *A, int64_t a_ld, const void *B, int64_t b_ld);
cudaError_t launch_gemm_x3(const float *A, int64_t a_rows, int64_t a_ld, int a_row0,
                           int a_row_z, int a_row_r, const float *B, int64_t b_rows, int64_t b_ld,
                           int b_row0, int b_row_z, int b_row_r, int M, int N, int K, int R,
                           int nz, int flat_rpz, float *C, int64_t c_sm, int64_t c_sn,
                           int64_t c_sz, cudaStream_t stream);
cudaError_t launch_gemm_sample(const Problem &P, int g, const void *goutT_g, const void *wT_g,
                               void *cols16, float *gx, float *goff, float *gmask,
                               cudaStream_t stream);
cudaError_t launch_backward(const Problem &P, const BackwardGrads &G, void *workspace,
                            cudaStream_t stream, int *launches);
// PackedDeformConv1d's offset (and mask) predictor (trunk.cu): a depthwise convolution
// of x with the layer's K, stride, padding and dilation, then pointwise projections
// ("heads") to offset_groups*K channels: the offsets, and the mask through a sigmoid.
struct TrunkProblem {
    int B, C_in, L_in, K, L_out;
    int stride, padding, dilation, offset_groups;
    int J;                     // offset_groups * K channels per head
    int dtype;                 // dcn1d_dtype of every tensor
    const void *x, *dw_w, *dw_b, *off_w, *off_b, *mask_w, *mask_b;   // biases may be NULL
    void *off_out, *mask_out;  // [B, offset_groups, L_out, K]; mask_out NULL: no mask head
};
bool trunk_tc_supported(const TrunkProblem &T);
// PackedDeformConv1d's whole forward as one kernel (packed_fused.cu) for the depthwise
// layer (groups == offset_groups == C_in == C_out, 16-bit): the trunk T feeds the
// deformable forward P (whose offset and mask pointers are not used) on chip.
bool packed_fused_supported(const TrunkProblem &T, const Problem &P);
cudaError_t launch_packed_fused(const TrunkProblem &T, const Problem &P, cudaStream_t stream);
// Launches the trunk; *kernel receives the name of the kernel chosen.
cudaError_t launch_trunk(const TrunkProblem &T, cudaStream_t stream, const char **kernel);
cudaError_t launch_sample_index(const void *off, int dtype, int B, int G, int L_out, int K,
                                int L_in, int stride, int padding, int dilation,
                                int unconstrained, int32_t *i0, float *frac,
                                cudaStream_t stream);

}  // namespace dcn1d
