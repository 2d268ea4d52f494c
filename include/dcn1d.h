/*
 * dcn1d.h -- C ABI of the B200 (sm_100a) forward and backward passes of 1D
 * deformable convolution (DeformConv1d), with optional DCNv2 modulation mask.
 *
 * What the forward computes (sources: the "conv1d" operator page, sections
 * "Description", "Shape" and "Axis convention"; the dc1d page "dc1d
 * (DeformConv1d)", sections "Usage / DeformConv1d" and "Modulation (DCNv2)";
 * the article "A Detailed Explanation of the Calculation Workflow for Dilated
 * Convolution and Deformable Convolution", section "Deformable Convolution"
 * and its "Step 2: Deformable Sampling"):
 *
 *   out[b,co,l] = bias[co] + sum_{ci in group(co)} sum_{k<K}
 *                   weight[co, ci - c0(co), k] * m[b,g,l,k]
 *                   * lerp(x[b,ci,:], l*stride - padding + k*dilation + offsets[b,g,l,k])
 *
 *   g = ci / (C_in / offset_groups) is the offset group of channel ci (all
 *   channels of a group share offsets and mask); lerp mixes the two integer
 *   neighbours i0 = floor(pos) and i0+1 with weights (1-f) and f, f = pos - i0,
 *   and x reads zero outside [0, L_in-1].  Unless `unconstrained` is set, the
 *   position is first clamped to the tap's receptive field
 *   [l*stride - padding, l*stride - padding + dilation*(K-1)].  The position is
 *   formed in IEEE float32 with round-to-nearest: pos = (float)base + offset;
 *   i0 = floor(pos); f = pos - (float)i0.  Precondition: offsets are finite and
 *   |pos| < 2^24 (a NaN or huge offset never causes an out-of-bounds access,
 *   but its result is unspecified).  m = 1 when the mask is NULL; a mask of
 *   all ones gives bit-for-bit the same output as a NULL mask.
 *
 * Memory: every tensor is a dense, contiguous, row-major array in device
 * memory of the current CUDA device, described by a dcn1d_tensor.  The caller
 * owns and allocates every buffer, `out` included; the library never allocates,
 * frees or synchronises.  Work is enqueued on `stream` (a cudaStream_t; NULL is
 * the legacy default stream) and runs asynchronously: a returned DCN1D_OK means
 * the launch was accepted, and device-side failures surface at the caller's
 * next synchronisation.  Thread safety: calls may be made from several host
 * threads; outputs must not alias inputs.
 *
 * Errors are status codes (never an abort or a device trap).  Every argument
 * is validated on the host before anything is launched; on a non-OK status
 * nothing was enqueued.
 */
#ifndef DCN1D_H
#define DCN1D_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dcn1d_status {
    DCN1D_OK = 0,
    DCN1D_ERR_NULL = 1,        /* a required pointer (descriptor or data) is NULL          */
    DCN1D_ERR_DTYPE = 2,       /* unknown dtype, or floating tensors of mixed dtypes       */
    DCN1D_ERR_SHAPE = 3,       /* wrong ndim, or shapes that disagree with each other      */
    DCN1D_ERR_ARG = 4,         /* stride/padding/dilation/groups out of range, L_out < 1   */
    DCN1D_ERR_UNSUPPORTED = 5, /* sizes past the 32-bit index or 2^24 position limits      */
    DCN1D_ERR_LAUNCH = 6,      /* the CUDA launch itself failed (cudaGetLastError)         */
    DCN1D_ERR_TIMEOUT = 7,     /* a kernel gave up a bounded wait (see dcn1d_device_status) */
    DCN1D_ERR_CUDA = 8         /* another CUDA runtime call failed                         */
} dcn1d_status;

typedef enum dcn1d_dtype {
    DCN1D_F32 = 0,             /* IEEE float32                                             */
    DCN1D_BF16 = 1,            /* bfloat16                                                 */
    DCN1D_F16 = 2              /* IEEE float16 (binary16)                                  */
} dcn1d_dtype;

/* A dense, contiguous, row-major device array of `ndim` (<= 4) dimensions. */
typedef struct dcn1d_tensor {
    void *data;                /* device pointer; 16-byte alignment enables the fast paths */
    int32_t dtype;             /* a dcn1d_dtype                                            */
    int32_t ndim;
    int64_t shape[4];          /* shape[i] for i < ndim; the rest is ignored               */
} dcn1d_tensor;

/*
 * Output length of the convolution ("conv1d" page, "Shape"):
 *   L_out = floor((L_in + 2*padding - dilation*(kernel_size - 1) - 1) / stride + 1).
 * Returns -1 if L_in < 1, kernel_size < 1, stride < 1, padding < 0, dilation < 1,
 * any argument exceeds 2^31, or the length would be < 1.  Host only; needs no
 * device.
 */
int64_t dcn1d_out_length(int64_t L_in, int64_t kernel_size, int64_t stride, int64_t padding,
                         int64_t dilation);

/*
 * Padding given per side: `padding_left` zeros before the signal and
 * `padding_right` after it (the symmetric functions pass the same value for
 * both).  The dc1d page passes padding="valid" (0) and padding="same"; "same"
 * is read as nn.Conv1d reads it, whose output-length closed form the page
 * uses: stride 1, d(K-1)/2 zeros on the left and the rest on the right, so
 * L_out = L_in (asymmetric when dilation*(kernel_size-1) is odd).  Only the
 * left side moves the receptive fields, l*stride - padding_left + k*dilation;
 * both sides enter the length:
 *   L_out = floor((L_in + padding_left + padding_right - dilation*(K-1) - 1)/stride) + 1.
 * Returns -1 as dcn1d_out_length does.
 */
int64_t dcn1d_out_length_lr(int64_t L_in, int64_t kernel_size, int64_t stride,
                            int64_t padding_left, int64_t padding_right, int64_t dilation);

/* dcn1d_forward_ws with padding per side (see dcn1d_out_length_lr); otherwise identical. */
int dcn1d_forward_lr(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                     const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                     const dcn1d_tensor *bias, int64_t stride, int64_t padding_left,
                     int64_t padding_right, int64_t dilation, int64_t groups,
                     int64_t offset_groups, int unconstrained, dcn1d_tensor *out,
                     void *workspace, size_t workspace_bytes, void *stream);

/* dcn1d_forward_kernel_name with padding per side. */
const char *dcn1d_forward_lr_kernel_name(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                                         const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                                         const dcn1d_tensor *bias, int64_t stride,
                                         int64_t padding_left, int64_t padding_right,
                                         int64_t dilation, int64_t groups, int64_t offset_groups,
                                         int unconstrained, const dcn1d_tensor *out);

/* dcn1d_forward_workspace_size with padding per side. */
int64_t dcn1d_forward_lr_workspace_size(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                                        const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                                        const dcn1d_tensor *bias, int64_t stride,
                                        int64_t padding_left, int64_t padding_right,
                                        int64_t dilation, int64_t groups, int64_t offset_groups,
                                        int unconstrained, const dcn1d_tensor *out);

/*
 * The deformable convolution forward (formula at the top of this file).
 *
 *   x        [B, C_in, L_in]                       required
 *   offsets  [B, offset_groups, L_out, K]          required; L_out must equal
 *                                                  dcn1d_out_length(L_in, K, ...)
 *   mask     [B, offset_groups, L_out, K] or NULL  applied as given (no sigmoid)
 *   weight   [C_out, C_in / groups, K]             required
 *   bias     [C_out] or NULL
 *   out      [B, C_out, L_out]                     required, written entirely
 *
 * All floating tensors share one dtype (F32, BF16 or F16), and `out` is
 * written in that same dtype ("conv1d" page: the computation stays in the
 * input dtype).  Positions and fractions are fp32 throughout.  F32: fp32
 * interpolation and an fp32-accurate contraction (three TF32 products).
 * BF16/F16: fp32 accumulation; the tensor-core path interpolates in 16-bit
 * pairs (the fraction and x1 - x0 rounded to the dtype, then one fused
 * multiply-add), the depthwise and generic paths in fp32.  groups must divide C_in and C_out; offset_groups must divide
 * C_in; stride >= 1, padding >= 0, dilation >= 1 ("conv1d" page, "Arguments").
 * `unconstrained` != 0 lets taps sample anywhere (dc1d page, "Usage").
 *
 * Needs no scratch memory: every path, the fp32 tensor-core one included,
 * runs as one kernel launch without it.
 *
 * Returns DCN1D_OK, or DCN1D_ERR_NULL / _DTYPE / _SHAPE / _ARG / _UNSUPPORTED on
 * invalid arguments (nothing launched), DCN1D_ERR_LAUNCH if a launch failed.
 */
int dcn1d_forward(const dcn1d_tensor *x, const dcn1d_tensor *offsets, const dcn1d_tensor *mask,
                  const dcn1d_tensor *weight, const dcn1d_tensor *bias, int64_t stride,
                  int64_t padding, int64_t dilation, int64_t groups, int64_t offset_groups,
                  int unconstrained, dcn1d_tensor *out, void *stream);

/*
 * Scratch memory (bytes) the fastest path for these arguments needs: 0 for
 * every valid argument set (the fp32 tensor-core path forms the weight's low
 * tf32 part in shared memory and adds its split-K partial sums on chip); a
 * negative value is minus the status code of invalid arguments.  Host only.
 * The workspace forms of the entry points keep their signatures, so callers
 * that size a workspace by this query keep working.
 */
int64_t dcn1d_forward_workspace_size(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                                     const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                                     const dcn1d_tensor *bias, int64_t stride, int64_t padding,
                                     int64_t dilation, int64_t groups, int64_t offset_groups,
                                     int unconstrained, const dcn1d_tensor *out);

/*
 * dcn1d_forward with caller-provided scratch: `workspace` is a device buffer
 * of `workspace_bytes` bytes, 256-byte aligned, owned by the caller and used
 * only during the work enqueued on `stream` (calls that overlap on the GPU
 * must use different workspaces).  No present path reads it
 * (dcn1d_forward_workspace_size is 0), so the call behaves exactly like
 * dcn1d_forward.  A non-zero size with a NULL pointer is DCN1D_ERR_NULL.
 * Other arguments and errors as for dcn1d_forward.
 */
int dcn1d_forward_ws(const dcn1d_tensor *x, const dcn1d_tensor *offsets, const dcn1d_tensor *mask,
                     const dcn1d_tensor *weight, const dcn1d_tensor *bias, int64_t stride,
                     int64_t padding, int64_t dilation, int64_t groups, int64_t offset_groups,
                     int unconstrained, dcn1d_tensor *out, void *workspace,
                     size_t workspace_bytes, void *stream);

/*
 * dcn1d_forward for callers that cannot allocate device memory: code running
 * where cudaMalloc is not allowed or not wanted (a real-time loop, a runtime
 * that owns every allocation, a host that reserved all device memory up
 * front).  The pages describe no counterpart of this entry point; it exists
 * only for such callers.
 *
 * Same arguments, kernels and results as dcn1d_forward_ws given enough
 * scratch, but the scratch is a fixed array of 48 MiB inside the library
 * (static device memory: every GPU that loads the library may hold it until
 * the process exits).  The caller still passes all inputs and `out`; this call
 * itself allocates and frees nothing.
 *
 * Set-up: the first call on each device looks up the array's device address
 * (with that device current) and caches it; make that first call before any
 * stream capture.  The cached address belongs to the device's current driver
 * context: after a device reset (cudaDeviceReset) the next call sees a new
 * context and looks the address up again (that call is then a set-up call too).
 *
 * Scratch limit: arguments whose fastest path needs more than 48 MiB
 * (dcn1d_forward_workspace_size) are rejected with DCN1D_ERR_UNSUPPORTED and
 * nothing is launched.  Arguments that need no scratch run as dcn1d_forward --
 * at present every valid argument set, since no forward path needs scratch.
 *
 * Sharing: every call on a device uses the same array and it keeps the last
 * call's contents; each call writes every scratch byte it reads, so nothing
 * needs clearing, but calls whose work overlaps on the GPU (different streams,
 * or host threads) race on the array and must be serialised by the caller.
 *
 * Returns the codes of dcn1d_forward, DCN1D_ERR_UNSUPPORTED past the scratch
 * limit, or DCN1D_ERR_CUDA if the address lookup failed.
 */
int dcn1d_forward_noalloc(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                          const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                          const dcn1d_tensor *bias, int64_t stride, int64_t padding,
                          int64_t dilation, int64_t groups, int64_t offset_groups,
                          int unconstrained, dcn1d_tensor *out, void *stream);

/*
 * Backward pass: the gradients of sum(grad_out * forward(...)) with respect to
 * x, offsets, mask, weight and bias.  The pages train the layer through
 * autograd on the forward as written (the dc1d page, opening paragraph; its
 * demo notebook checks the offset gradient against a finite difference), so
 * these are that derivative: with v = (1-f) x[i0] + f x[i0+1] and
 * dv = sum_co weight[co, c, k] * grad_out[b, co, l] over the conv group,
 *   grad_weight[co,c,k] = sum_{b,l} grad_out[b,co,l] * m * v
 *   grad_x[b,ci,i0] += m (1-f) dv,  grad_x[b,ci,i0+1] += m f dv  (in range only)
 *   grad_mask[b,g,l,k]  = sum_{ci in offset group g} v * dv
 *   grad_offsets[b,g,l,k] = sum_{ci in g} m (x[i0+1] - x[i0]) dv, and 0 where
 *                           the constrained clamp moved the position (a
 *                           position exactly on a bound passes the gradient)
 *   grad_bias[co]       = sum_{b,l} grad_out[b,co,l]
 * floor() contributes nothing (inside a unit cell the slope is x[i0+1]-x[i0]).
 *
 * Arguments: the forward's inputs (bias is not needed), grad_out [B, C_out,
 * L_out] in their dtype, and the gradients wanted, each NULL when not wanted
 * and otherwise shaped like its input in the same dtype (grad_mask needs a
 * mask: DCN1D_ERR_ARG otherwise).  Every wanted gradient is overwritten.
 * Arithmetic is fp32; for 16-bit dtypes the two contractions run on the tensor
 * cores with 16-bit operands (grad_out, W, and the sampled columns rounded to
 * the dtype) and fp32 accumulation, when L_out, C_out and C_out/groups are
 * multiples of 8 (dcn1d_backward_kernel_name says which).  grad_x,
 * grad_offsets and grad_mask are sums of atomic fp32 additions, so their low
 * bits may differ between calls; grad_weight and grad_bias are summed in a
 * fixed order.
 *
 * Scratch: `workspace` (256-byte aligned, owned by the caller, used only by the
 * work enqueued on `stream`) of at least dcn1d_backward_workspace_size() bytes:
 * column buffers of B * C_in * K * L_out values (fp32 gradient columns when any
 * of grad_x / grad_offsets / grad_mask is wanted; the sampled columns, fp32 or
 * 16-bit on the tensor-core path, when grad_weight is wanted), on the
 * tensor-core path grad_out and W transposed, fp32 slices of grad_weight, and
 * fp32 accumulators of grad_x, grad_offsets and grad_mask.  Too small or misaligned:
 * DCN1D_ERR_ARG; NULL with a non-zero need: DCN1D_ERR_NULL.
 * Other errors as for dcn1d_forward; B * groups above 65535 is
 * DCN1D_ERR_UNSUPPORTED.
 */
int64_t dcn1d_backward_workspace_size(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                                      const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                                      const dcn1d_tensor *grad_out, int64_t stride,
                                      int64_t padding, int64_t dilation, int64_t groups,
                                      int64_t offset_groups, int unconstrained,
                                      const dcn1d_tensor *grad_x, const dcn1d_tensor *grad_offsets,
                                      const dcn1d_tensor *grad_mask,
                                      const dcn1d_tensor *grad_weight,
                                      const dcn1d_tensor *grad_bias);

int dcn1d_backward(const dcn1d_tensor *x, const dcn1d_tensor *offsets, const dcn1d_tensor *mask,
                   const dcn1d_tensor *weight, const dcn1d_tensor *grad_out, int64_t stride,
                   int64_t padding, int64_t dilation, int64_t groups, int64_t offset_groups,
                   int unconstrained, dcn1d_tensor *grad_x, dcn1d_tensor *grad_offsets,
                   dcn1d_tensor *grad_mask, dcn1d_tensor *grad_weight, dcn1d_tensor *grad_bias,
                   void *workspace, size_t workspace_bytes, void *stream);

/* dcn1d_backward and its workspace size with padding per side (see dcn1d_out_length_lr). */
/* Which contraction kernels dcn1d_backward_lr runs for these arguments
 * ("tcgen05_gemm": 16-bit operands on the tensor cores, or "cuda_core_gemm"), or
 * NULL if the arguments are invalid.  Host only. */
const char *dcn1d_backward_kernel_name(
    const dcn1d_tensor *x, const dcn1d_tensor *offsets, const dcn1d_tensor *mask,
    const dcn1d_tensor *weight, const dcn1d_tensor *grad_out, int64_t stride,
    int64_t padding_left, int64_t padding_right, int64_t dilation, int64_t groups,
    int64_t offset_groups, int unconstrained, const dcn1d_tensor *grad_x,
    const dcn1d_tensor *grad_offsets, const dcn1d_tensor *grad_mask,
    const dcn1d_tensor *grad_weight, const dcn1d_tensor *grad_bias);

int64_t dcn1d_backward_lr_workspace_size(
    const dcn1d_tensor *x, const dcn1d_tensor *offsets, const dcn1d_tensor *mask,
    const dcn1d_tensor *weight, const dcn1d_tensor *grad_out, int64_t stride,
    int64_t padding_left, int64_t padding_right, int64_t dilation, int64_t groups,
    int64_t offset_groups, int unconstrained, const dcn1d_tensor *grad_x,
    const dcn1d_tensor *grad_offsets, const dcn1d_tensor *grad_mask,
    const dcn1d_tensor *grad_weight, const dcn1d_tensor *grad_bias);

int dcn1d_backward_lr(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                      const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                      const dcn1d_tensor *grad_out, int64_t stride, int64_t padding_left,
                      int64_t padding_right, int64_t dilation, int64_t groups,
                      int64_t offset_groups, int unconstrained, dcn1d_tensor *grad_x,
                      dcn1d_tensor *grad_offsets, dcn1d_tensor *grad_mask,
                      dcn1d_tensor *grad_weight, dcn1d_tensor *grad_bias, void *workspace,
                      size_t workspace_bytes, void *stream);

/*
 * PackedDeformConv1d's offset (and mask) predictor ("dc1d (DeformConv1d)" page,
 * "PackedDeformConv1d": a depthwise-separable convolution block computes the
 * offsets inside the layer; "Modulation (DCNv2)": modulated=True adds a second
 * pointwise branch off the same depthwise trunk, ending in a sigmoid, for the
 * mask).  With J = offset_groups * K and j = g*K + k:
 *
 *   t[b,c,l]         = dw_bias[c] + sum_k dw_weight[c,0,k] * x[b, c, l*stride - padding_left + k*dilation]
 *   offsets[b,g,l,k] = off_bias[j] + sum_c off_weight[j,c] * t[b,c,l]
 *   mask[b,g,l,k]    = sigmoid(mask_bias[j] + sum_c mask_weight[j,c] * t[b,c,l])
 *
 * (x reads zero outside [0, L_in)).  The depthwise convolution takes the
 * layer's kernel size, stride, padding and dilation, so it yields one offset
 * vector per output position; nothing sits between the depthwise and the
 * pointwise convolutions.
 *
 *   x            [B, C_in, L_in]                      required
 *   dw_weight    [C_in, 1, K]                         required
 *   dw_bias      [C_in] or NULL
 *   off_weight   [J, C_in] or [J, C_in, 1]            required
 *   off_bias     [J] or NULL
 *   mask_weight  like off_weight, or NULL (no mask head)
 *   mask_bias    [J] or NULL (NULL when mask_weight is NULL)
 *   offsets_out  [B, offset_groups, L_out, K]          required, written entirely
 *   mask_out     like offsets_out; required with mask_weight, else NULL
 *
 * All tensors share one dtype; t stays on chip in fp32 and the outputs are
 * rounded to that dtype.  offset_groups must divide C_in.  Device memory
 * owned by the caller; runs on `stream`, asynchronously, and allocates
 * nothing.  Returns DCN1D_OK, or the validation codes of dcn1d_forward
 * (nothing launched), DCN1D_ERR_LAUNCH if the launch failed.
 */
int dcn1d_packed_trunk(const dcn1d_tensor *x, const dcn1d_tensor *dw_weight,
                       const dcn1d_tensor *dw_bias, const dcn1d_tensor *off_weight,
                       const dcn1d_tensor *off_bias, const dcn1d_tensor *mask_weight,
                       const dcn1d_tensor *mask_bias, int64_t stride, int64_t padding_left,
                       int64_t padding_right, int64_t dilation, int64_t offset_groups,
                       dcn1d_tensor *offsets_out, dcn1d_tensor *mask_out, void *stream);

/* Which trunk kernel dcn1d_packed_trunk launches ("trunk_tcgen05" or "trunk_simt"),
 * or NULL if the arguments are invalid.  Host only. */
const char *dcn1d_packed_trunk_kernel_name(
    const dcn1d_tensor *x, const dcn1d_tensor *dw_weight, const dcn1d_tensor *dw_bias,
    const dcn1d_tensor *off_weight, const dcn1d_tensor *off_bias,
    const dcn1d_tensor *mask_weight, const dcn1d_tensor *mask_bias, int64_t stride,
    int64_t padding_left, int64_t padding_right, int64_t dilation, int64_t offset_groups,
    const dcn1d_tensor *offsets_out, const dcn1d_tensor *mask_out);

/*
 * The whole PackedDeformConv1d forward: dcn1d_packed_trunk, then the deformable
 * convolution (dcn1d_forward_lr) of x with the predicted offsets and, when
 * mask_weight is given, the predicted mask.  weight [C_out, C_in/groups, K]
 * (K = dw_weight's), bias [C_out] or NULL, out [B, C_out, L_out].
 * offsets_out / mask_out may be NULL: the predicted tensors then live in
 * `workspace` (caller-owned device memory, 256-byte aligned, used only by the
 * work this call enqueues).  dcn1d_packed_forward_workspace_size() gives the
 * bytes for those tensors plus the forward's own scratch; a workspace smaller
 * than the predicted tensors is DCN1D_ERR_ARG (NULL: DCN1D_ERR_NULL), and
 * between that and the full size the forward runs a kernel without scratch.
 * Enqueues the trunk kernel and the forward's kernels on `stream`.
 *
 * One kernel instead, with no workspace at all, for the depthwise layer of the
 * dc1d page's PackedDeformConv1d example: when offsets_out and mask_out are
 * both NULL, groups == offset_groups == C_in == C_out, the dtype is BF16 or
 * F16, K <= 4 (K <= 3 with a mask head when C_in is 256), C_in a multiple of
 * 64 up to 256, L_in a multiple of 8 and x and the head weights 16-byte
 * aligned.  The trunk's output, the predicted offsets and the mask then stay
 * on chip: each tile's offsets and mask (rounded to the dtype, as the tensors
 * the two-launch path hands on) feed the deformable convolution inside the
 * kernel.  dcn1d_packed_forward_kernel_name() says which form runs.
 */
int dcn1d_packed_forward(const dcn1d_tensor *x, const dcn1d_tensor *dw_weight,
                         const dcn1d_tensor *dw_bias, const dcn1d_tensor *off_weight,
                         const dcn1d_tensor *off_bias, const dcn1d_tensor *mask_weight,
                         const dcn1d_tensor *mask_bias, const dcn1d_tensor *weight,
                         const dcn1d_tensor *bias, int64_t stride, int64_t padding_left,
                         int64_t padding_right, int64_t dilation, int64_t groups,
                         int64_t offset_groups, int unconstrained, dcn1d_tensor *offsets_out,
                         dcn1d_tensor *mask_out, dcn1d_tensor *out, void *workspace,
                         size_t workspace_bytes, void *stream);

/* Workspace bytes dcn1d_packed_forward wants for these arguments (see there), or
 * minus the status code of invalid arguments.  Host only. */
int64_t dcn1d_packed_forward_workspace_size(
    const dcn1d_tensor *x, const dcn1d_tensor *dw_weight, const dcn1d_tensor *dw_bias,
    const dcn1d_tensor *off_weight, const dcn1d_tensor *off_bias,
    const dcn1d_tensor *mask_weight, const dcn1d_tensor *mask_bias, const dcn1d_tensor *weight,
    const dcn1d_tensor *bias, int64_t stride, int64_t padding_left, int64_t padding_right,
    int64_t dilation, int64_t groups, int64_t offset_groups, int unconstrained,
    const dcn1d_tensor *offsets_out, const dcn1d_tensor *mask_out, const dcn1d_tensor *out);

/* Which form dcn1d_packed_forward takes for these arguments: "packed_fused_tcgen05"
 * (one kernel, no workspace) or "<trunk kernel>+<forward kernel>" (two launches,
 * e.g. "trunk_tcgen05+depthwise"); NULL if the arguments are invalid.  Host only. */
const char *dcn1d_packed_forward_kernel_name(
    const dcn1d_tensor *x, const dcn1d_tensor *dw_weight, const dcn1d_tensor *dw_bias,
    const dcn1d_tensor *off_weight, const dcn1d_tensor *off_bias,
    const dcn1d_tensor *mask_weight, const dcn1d_tensor *mask_bias, const dcn1d_tensor *weight,
    const dcn1d_tensor *bias, int64_t stride, int64_t padding_left, int64_t padding_right,
    int64_t dilation, int64_t groups, int64_t offset_groups, int unconstrained,
    const dcn1d_tensor *offsets_out, const dcn1d_tensor *mask_out, const dcn1d_tensor *out);

/* A static, human-readable name of a status code ("DCN1D_OK", ...). Never NULL. */
const char *dcn1d_status_string(int status);

/*
 * The sampling step alone, for testing the integer decisions bit for bit: for
 * every tap of `offsets` ([B, G, L_out, K], F32 or BF16, device memory) write
 * the integer neighbour i0 = floor(pos) to `i0` and the fraction f = pos - i0
 * to `frac` (each a device array of B*G*L_out*K elements, same order as
 * offsets), using the same device function as the forward kernels.  L_out
 * must equal dcn1d_out_length(L_in, K, stride, padding, dilation).
 * Errors as for dcn1d_forward.
 */
int dcn1d_sample_index(const dcn1d_tensor *offsets, int64_t L_in, int64_t stride,
                       int64_t padding, int64_t dilation, int unconstrained, int32_t *i0,
                       float *frac, void *stream);

/*
 * Which kernel dcn1d_forward launches for these arguments, as a static string
 * ("direct", "depthwise", "tcgen05_bf16", "tcgen05_3xtf32"), or NULL if the
 * arguments are invalid.  Host only; launches nothing.  For tests and
 * benchmarks.
 */
const char *dcn1d_forward_kernel_name(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                                      const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                                      const dcn1d_tensor *bias, int64_t stride, int64_t padding,
                                      int64_t dilation, int64_t groups, int64_t offset_groups,
                                      int unconstrained, const dcn1d_tensor *out);

/*
 * For benchmarks: the next dcn1d_forward / dcn1d_forward_ws call on this host
 * thread records `begin` (a cudaEvent_t) on its stream right before launching
 * its kernel and `end` right after it, then forgets both.  Every forward is one
 * kernel launch, so the pair brackets all of its device work.  NULL events record
 * nothing.
 */
void dcn1d_set_timing_events(void *begin, void *end);

/*
 * Device-side status of the kernels enqueued so far on the current device.
 * Kernels that wait on on-chip barriers bound every wait (about 2 s); a kernel
 * that gives up records it in a device status word and exits, leaving its
 * output incomplete.  This call synchronises `stream`, reads and clears that
 * word, and returns DCN1D_ERR_TIMEOUT if any kernel gave up since the last
 * call, DCN1D_ERR_CUDA if the synchronisation or the read failed, else
 * DCN1D_OK.  It is the only entry point that synchronises.
 */
int dcn1d_device_status(void *stream);

/*
 * Number of kernels the last accepted dcn1d_forward / dcn1d_forward_ws call on
 * this host thread enqueued (0 if none).  For counting launches in benchmarks.
 */
int dcn1d_last_launch_count(void);

/*
 * TEST HOOK of the failure path of dcn1d_device_status (no counterpart on the
 * pages; not part of the forward).  Runs the bf16 tensor-core kernel of
 * dcn1d_forward on these arguments (bf16, kernel size 3, no mask, no bias,
 * shapes that kernel takes) in a build whose loader never issues a load, with
 * every on-chip wait limited to `wait_limit_ns` (1 us .. 100 ms).  No stage
 * ever fills, so the waits run out: the kernel records the timeout in the
 * device status word, lets nothing it issued stay in flight, frees its tensor
 * memory and exits; `out` is left unwritten.  The next dcn1d_device_status on
 * this device returns DCN1D_ERR_TIMEOUT.  No GPU fault, trap or hang is
 * involved.  Returns DCN1D_ERR_UNSUPPORTED for other shapes or dtypes,
 * DCN1D_ERR_ARG for a limit outside the range, else the codes of
 * dcn1d_forward.
 */
int dcn1d_test_forward_stalled(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                               const dcn1d_tensor *weight, int64_t stride, int64_t padding,
                               int64_t dilation, int64_t groups, int64_t offset_groups,
                               int unconstrained, dcn1d_tensor *out, int64_t wait_limit_ns,
                               void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DCN1D_H */
