// The C ABI (include/dcn1d.h): argument validation, kernel selection and
// launch on the caller's stream.  Allocates nothing and never synchronises.
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "sm100.cuh"

namespace dcn1d {
namespace {

thread_local int g_last_launches = 0;
thread_local cudaEvent_t g_time_begin = nullptr, g_time_end = nullptr;

constexpr int64_t kMaxElems = (int64_t)1 << 31;   // every tensor indexed with int32 rows
constexpr int64_t kMaxPos = (int64_t)1 << 24;     // positions exact in float32

int64_t numel(const dcn1d_tensor *t) {
    int64_t n = 1;
    for (int i = 0; i < t->ndim; ++i)
        n *= t->shape[i];
    return n;
}

// Descriptor present, known dtype, right rank, non-negative extents, data
// present unless the tensor is empty.
int check_desc(const dcn1d_tensor *t, int ndim) {
    if (!t)
        return DCN1D_ERR_NULL;
    if (t->dtype != DCN1D_F32 && t->dtype != DCN1D_BF16 && t->dtype != DCN1D_F16)
        return DCN1D_ERR_DTYPE;
    if (t->ndim != ndim)
        return DCN1D_ERR_SHAPE;
    for (int i = 0; i < ndim; ++i)
        if (t->shape[i] < 0)
            return DCN1D_ERR_SHAPE;
    if (!t->data && numel(t) > 0)
        return DCN1D_ERR_NULL;
    return DCN1D_OK;
}

bool shape_is(const dcn1d_tensor *t, int64_t a, int64_t b, int64_t c, int64_t d = -1) {
    if (t->shape[0] != a || t->shape[1] != b || t->shape[2] != c)
        return false;
    return d < 0 || t->shape[3] == d;
}

enum Kernel { kDirect = 0, kDepthwise = 1, kTcBf16 = 2, kTcTf32 = 3 };

const char *kernel_names[] = {"direct", "depthwise", "tcgen05_bf16", "tcgen05_3xtf32"};

// The fastest kernel for P.  No forward kernel needs workspace; the workspace forms of
// the entry points accept (and ignore) one, so that callers sized for a path that might
// need scratch keep working.
Kernel select_kernel(const Problem &P, size_t /*ws_bytes*/) {
    if (depthwise_supported(P))
        return kDepthwise;
    if (tc_bf16_supported(P))
        return kTcBf16;
    if (tc_tf32_supported(P))
        return kTcTf32;
    return kDirect;
}

size_t workspace_bytes(const Problem & /*P*/) { return 0; }

// Full validation; fills P and the chosen kernel on success.
int validate(const dcn1d_tensor *x, const dcn1d_tensor *off, const dcn1d_tensor *mask,
             const dcn1d_tensor *w, const dcn1d_tensor *bias, int64_t stride, int64_t padding,
             int64_t padding_right,
             int64_t dilation, int64_t groups, int64_t offset_groups, int unconstrained,
             const dcn1d_tensor *out, Problem *P) {
    int st;
    if (!x || !off || !w || !out)
        return DCN1D_ERR_NULL;
    if ((st = check_desc(x, 3)) || (st = check_desc(off, 4)) || (st = check_desc(w, 3)) ||
        (st = check_desc(out, 3)))
        return st;
    if (mask && (st = check_desc(mask, 4)))
        return st;
    if (bias && (st = check_desc(bias, 1)))
        return st;
    const int dt = x->dtype;
    if (off->dtype != dt || w->dtype != dt || out->dtype != dt || (mask && mask->dtype != dt) ||
        (bias && bias->dtype != dt))
        return DCN1D_ERR_DTYPE;

    if (stride < 1 || padding < 0 || padding_right < 0 || dilation < 1 || groups < 1 ||
        offset_groups < 1)
        return DCN1D_ERR_ARG;
    const int64_t B = x->shape[0], C_in = x->shape[1], L_in = x->shape[2];
    const int64_t C_out = w->shape[0], K = w->shape[2];
    if (C_in < 1 || L_in < 1 || C_out < 1 || K < 1)
        return DCN1D_ERR_SHAPE;
    if (C_in % groups || C_out % groups || C_in % offset_groups)
        return DCN1D_ERR_ARG;
    if (w->shape[1] * groups != C_in)
        return DCN1D_ERR_SHAPE;
    if (stride >= kMaxPos || padding >= kMaxPos || padding_right >= kMaxPos ||
        dilation >= kMaxPos || K >= kMaxPos || L_in >= kMaxPos)
        return DCN1D_ERR_UNSUPPORTED;
    const int64_t L_out = dcn1d_out_length_lr(L_in, K, stride, padding, padding_right, dilation);
    if (L_out < 1)
        return DCN1D_ERR_ARG;
    if (!shape_is(off, B, offset_groups, L_out, K))
        return DCN1D_ERR_SHAPE;
    if (mask && !shape_is(mask, B, offset_groups, L_out, K))
        return DCN1D_ERR_SHAPE;
    if (bias && bias->shape[0] != C_out)
        return DCN1D_ERR_SHAPE;
    if (!shape_is(out, B, C_out, L_out))
        return DCN1D_ERR_SHAPE;
    // Largest position any tap forms before its offset: (L_out-1)*s - p + d*(K-1) >= 0 and
    // smallest -p; both must be exact in float32.
    if ((L_out - 1) * stride + dilation * (K - 1) >= kMaxPos)
        return DCN1D_ERR_UNSUPPORTED;
    if (numel(x) >= kMaxElems || numel(off) >= kMaxElems || numel(w) >= kMaxElems ||
        numel(out) >= kMaxElems)
        return DCN1D_ERR_UNSUPPORTED;

    P->B = (int)B;
    P->C_in = (int)C_in;
    P->L_in = (int)L_in;
    P->C_out = (int)C_out;
    P->K = (int)K;
    P->L_out = (int)L_out;
    P->stride = (int)stride;
    P->padding = (int)padding;
    P->padding_right = (int)padding_right;
    P->dilation = (int)dilation;
    P->groups = (int)groups;
    P->offset_groups = (int)offset_groups;
    P->unconstrained = unconstrained ? 1 : 0;
    P->dtype = dt;
    P->cin_g = (int)(C_in / groups);
    P->cout_g = (int)(C_out / groups);
    P->cin_per_og = (int)(C_in / offset_groups);
    P->x = x->data;
    P->off = off->data;
    P->mask = mask ? mask->data : nullptr;
    P->w = w->data;
    P->bias = bias ? bias->data : nullptr;
    P->out = out->data;
    return DCN1D_OK;
}

// Validation of a backward call: the forward's checks with grad_out in the place
// of out, then every wanted gradient against its input's dtype and shape.
int validate_backward(const dcn1d_tensor *x, const dcn1d_tensor *off, const dcn1d_tensor *mask,
                      const dcn1d_tensor *w, const dcn1d_tensor *gout, int64_t stride,
                      int64_t padding,
                      int64_t padding_right, int64_t dilation, int64_t groups, int64_t offset_groups,
                      int unconstrained, const dcn1d_tensor *gx, const dcn1d_tensor *goff,
                      const dcn1d_tensor *gmask, const dcn1d_tensor *gw, const dcn1d_tensor *gbias,
                      Problem *P, BackwardGrads *G) {
    int st = validate(x, off, mask, w, nullptr, stride, padding, padding_right, dilation, groups,
                      offset_groups, unconstrained, gout, P);
    if (st != DCN1D_OK)
        return st;
    auto like = [&](const dcn1d_tensor *g, const dcn1d_tensor *in, int nd) -> int {
        if (!g)
            return DCN1D_OK;
        if (!in)
            return DCN1D_ERR_ARG;   // a mask gradient without a mask
        const int s2 = check_desc(g, nd);
        if (s2 != DCN1D_OK)
            return s2;
        if (g->dtype != x->dtype)
            return DCN1D_ERR_DTYPE;
        for (int i = 0; i < nd; ++i)
            if (g->shape[i] != in->shape[i])
                return DCN1D_ERR_SHAPE;
        return DCN1D_OK;
    };
    if ((st = like(gx, x, 3)) || (st = like(goff, off, 4)) || (st = like(gmask, mask, 4)) ||
        (st = like(gw, w, 3)))
        return st;
    if (gbias) {
        if ((st = check_desc(gbias, 1)) != DCN1D_OK)
            return st;
        if (gbias->dtype != x->dtype)
            return DCN1D_ERR_DTYPE;
        if (gbias->shape[0] != P->C_out)
            return DCN1D_ERR_SHAPE;
    }
    if ((int64_t)P->B * P->groups > 65535)   // one GEMM grid slice per (batch, group)
        return DCN1D_ERR_UNSUPPORTED;
    G->gout = gout->data;
    G->x = gx ? gx->data : nullptr;
    G->off = goff ? goff->data : nullptr;
    G->mask = gmask ? gmask->data : nullptr;
    G->w = gw ? gw->data : nullptr;
    G->bias = gbias ? gbias->data : nullptr;
    return DCN1D_OK;
}

// Launches the forward of a validated problem with the fastest kernel that
// `ws_bytes` of workspace allows; *launches receives the kernel launches made.
cudaError_t run_forward(const Problem &P, void *workspace, size_t ws_bytes, cudaStream_t s,
                        int *launches) {
    cudaError_t err = cudaSuccess;
    *launches = 1;
    switch (select_kernel(P, ws_bytes)) {
    case kDirect:
        timing_begin(s);
        err = launch_direct(P, s);
        timing_end(s);
        break;
    case kDepthwise:
        timing_begin(s);
        err = launch_depthwise(P, s);
        timing_end(s);
        break;
    case kTcBf16:
        err = launch_tc_bf16(P, s);
        break;
    case kTcTf32:
        err = launch_tc_tf32(P, s);
        break;
    }
    return err;
}

// A pointwise weight: [J, C_in] or conv1d's [J, C_in, 1].
bool pointwise_shape(const dcn1d_tensor *w, int64_t J, int64_t C_in) {
    if (w->ndim == 2)
        return w->shape[0] == J && w->shape[1] == C_in;
    return w->ndim == 3 && w->shape[0] == J && w->shape[1] == C_in && w->shape[2] == 1;
}

// Validation of PackedDeformConv1d's trunk: x [B, C_in, L_in], dw_w [C_in, 1, K],
// dw_b [C_in], off_w / mask_w [J, C_in(, 1)], off_b / mask_b [J] with J = offset_groups*K,
// outputs [B, offset_groups, L_out, K].  A NULL output descriptor is allowed only when
// `outputs_optional` (the packed forward keeps such a tensor in its workspace); its
// data pointer is then left NULL in T.
int validate_trunk(const dcn1d_tensor *x, const dcn1d_tensor *dw_w, const dcn1d_tensor *dw_b,
                   const dcn1d_tensor *off_w, const dcn1d_tensor *off_b,
                   const dcn1d_tensor *mask_w, const dcn1d_tensor *mask_b, int64_t stride,
                   int64_t padding, int64_t padding_right, int64_t dilation,
                   int64_t offset_groups, const dcn1d_tensor *off_out,
                   const dcn1d_tensor *mask_out, bool outputs_optional, TrunkProblem *T) {
    int st;
    if (!x || !dw_w || !off_w)
        return DCN1D_ERR_NULL;
    if (!outputs_optional && (!off_out || (mask_w && !mask_out)))
        return DCN1D_ERR_NULL;
    if (mask_out && !mask_w)
        return DCN1D_ERR_ARG;   // a mask output without a mask head
    if (mask_b && !mask_w)
        return DCN1D_ERR_ARG;
    if ((st = check_desc(x, 3)) || (st = check_desc(dw_w, 3)))
        return st;
    if ((st = check_desc(off_w, off_w->ndim == 2 ? 2 : 3)))
        return st;
    if (mask_w && (st = check_desc(mask_w, mask_w->ndim == 2 ? 2 : 3)))
        return st;
    if ((dw_b && (st = check_desc(dw_b, 1))) || (off_b && (st = check_desc(off_b, 1))) ||
        (mask_b && (st = check_desc(mask_b, 1))))
        return st;
    if ((off_out && (st = check_desc(off_out, 4))) || (mask_out && (st = check_desc(mask_out, 4))))
        return st;
    const int dt = x->dtype;
    const dcn1d_tensor *all[] = {dw_w, dw_b, off_w, off_b, mask_w, mask_b, off_out, mask_out};
    for (const dcn1d_tensor *t : all)
        if (t && t->dtype != dt)
            return DCN1D_ERR_DTYPE;
    if (stride < 1 || padding < 0 || padding_right < 0 || dilation < 1 || offset_groups < 1)
        return DCN1D_ERR_ARG;
    const int64_t B = x->shape[0], C_in = x->shape[1], L_in = x->shape[2];
    const int64_t K = dw_w->shape[2];
    if (C_in < 1 || L_in < 1 || K < 1)
        return DCN1D_ERR_SHAPE;
    if (C_in % offset_groups)
        return DCN1D_ERR_ARG;
    if (dw_w->shape[0] != C_in || dw_w->shape[1] != 1)
        return DCN1D_ERR_SHAPE;
    if (stride >= kMaxPos || padding >= kMaxPos || padding_right >= kMaxPos ||
        dilation >= kMaxPos || K >= kMaxPos || L_in >= kMaxPos || offset_groups >= kMaxPos)
        return DCN1D_ERR_UNSUPPORTED;
    const int64_t J = offset_groups * K;
    if (!pointwise_shape(off_w, J, C_in) || (mask_w && !pointwise_shape(mask_w, J, C_in)))
        return DCN1D_ERR_SHAPE;
    if ((dw_b && dw_b->shape[0] != C_in) || (off_b && off_b->shape[0] != J) ||
        (mask_b && mask_b->shape[0] != J))
        return DCN1D_ERR_SHAPE;
    const int64_t L_out = dcn1d_out_length_lr(L_in, K, stride, padding, padding_right, dilation);
    if (L_out < 1)
        return DCN1D_ERR_ARG;
    if ((off_out && !shape_is(off_out, B, offset_groups, L_out, K)) ||
        (mask_out && !shape_is(mask_out, B, offset_groups, L_out, K)))
        return DCN1D_ERR_SHAPE;
    if ((L_out - 1) * stride + dilation * (K - 1) >= kMaxPos)
        return DCN1D_ERR_UNSUPPORTED;
    if (numel(x) >= kMaxElems || B * J * L_out >= kMaxElems || J * C_in >= kMaxElems ||
        B > 65535)
        return DCN1D_ERR_UNSUPPORTED;
    T->B = (int)B;
    T->C_in = (int)C_in;
    T->L_in = (int)L_in;
    T->K = (int)K;
    T->L_out = (int)L_out;
    T->stride = (int)stride;
    T->padding = (int)padding;
    T->dilation = (int)dilation;
    T->offset_groups = (int)offset_groups;
    T->J = (int)J;
    T->dtype = dt;
    T->x = x->data;
    T->dw_w = dw_w->data;
    T->dw_b = dw_b ? dw_b->data : nullptr;
    T->off_w = off_w->data;
    T->off_b = off_b ? off_b->data : nullptr;
    T->mask_w = mask_w ? mask_w->data : nullptr;
    T->mask_b = mask_b ? mask_b->data : nullptr;
    T->off_out = off_out ? off_out->data : nullptr;
    T->mask_out = mask_out ? mask_out->data : nullptr;
    return DCN1D_OK;
}

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

// Workspace of the packed forward: the predicted tensors the caller did not supply,
// then the forward's own scratch.
struct PackedLayout {
    size_t off_bytes, mask_bytes, fwd_offset, total;
    bool fused;   // one kernel: the predicted tensors stay on chip, no workspace
};

// Validation and layout shared by the packed forward and its workspace query.
// `ws_base` NULL (a size query) places the predicted tensors at a placeholder
// address; the descriptors are then used for shape checks only.
int packed_prepare(const dcn1d_tensor *x, const dcn1d_tensor *dw_w, const dcn1d_tensor *dw_b,
                   const dcn1d_tensor *off_w, const dcn1d_tensor *off_b,
                   const dcn1d_tensor *mask_w, const dcn1d_tensor *mask_b,
                   const dcn1d_tensor *weight, const dcn1d_tensor *bias, int64_t stride,
                   int64_t padding, int64_t padding_right, int64_t dilation, int64_t groups,
                   int64_t offset_groups, int unconstrained, const dcn1d_tensor *off_out,
                   const dcn1d_tensor *mask_out, const dcn1d_tensor *out, char *ws_base,
                   TrunkProblem *T, dcn1d_tensor *off_d, dcn1d_tensor *mask_d, Problem *P,
                   PackedLayout *lay) {
    int st = validate_trunk(x, dw_w, dw_b, off_w, off_b, mask_w, mask_b, stride, padding,
                            padding_right, dilation, offset_groups, off_out, mask_out, true, T);
    if (st != DCN1D_OK)
        return st;
    if (!weight)
        return DCN1D_ERR_NULL;
    if ((st = check_desc(weight, 3)) != DCN1D_OK)
        return st;
    if (weight->shape[2] != T->K)
        return DCN1D_ERR_SHAPE;
    const size_t es = x->dtype == DCN1D_F32 ? 4 : 2;
    const size_t n = (size_t)T->B * T->J * T->L_out;
    lay->off_bytes = off_out ? 0 : round256(n * es);
    lay->mask_bytes = (mask_w && !mask_out) ? round256(n * es) : 0;
    lay->fwd_offset = lay->off_bytes + lay->mask_bytes;
    char *base = ws_base ? ws_base : reinterpret_cast<char *>((uintptr_t)256);
    auto predicted = [&](char *data) {
        dcn1d_tensor d;
        memset(&d, 0, sizeof(d));
        d.data = data;
        d.dtype = x->dtype;
        d.ndim = 4;
        d.shape[0] = T->B;
        d.shape[1] = T->offset_groups;
        d.shape[2] = T->L_out;
        d.shape[3] = T->K;
        return d;
    };
    *off_d = off_out ? *off_out : predicted(base);
    if (mask_w)
        *mask_d = mask_out ? *mask_out : predicted(base + lay->off_bytes);
    st = validate(x, off_d, mask_w ? mask_d : nullptr, weight, bias, stride, padding,
                  padding_right, dilation, groups, offset_groups, unconstrained, out, P);
    if (st != DCN1D_OK)
        return st;
    // The caller asked for neither predicted tensor and the layer is the depthwise one the
    // fused kernel takes: nothing goes through global memory between the two stages.
    lay->fused = !off_out && !mask_out && packed_fused_supported(*T, *P);
    if (lay->fused) {
        lay->off_bytes = lay->mask_bytes = lay->fwd_offset = lay->total = 0;
        return DCN1D_OK;
    }
    lay->total = lay->fwd_offset + round256(workspace_bytes(*P));
    return DCN1D_OK;
}

}  // namespace

void timing_begin(cudaStream_t stream) {
    if (g_time_begin)
        cudaEventRecord(g_time_begin, stream);
}

void timing_end(cudaStream_t stream) {
    if (g_time_end)
        cudaEventRecord(g_time_end, stream);
    g_time_begin = g_time_end = nullptr;   // one forward only
}

// One status word per device (a __device__ variable exists once per device).
__device__ unsigned int g_device_status = 0;

// Cached per device and context (a device reset starts a new context, in which the
// variable may live elsewhere).
unsigned int *device_status_ptr() {
    static std::mutex mu;
    static unsigned int *ptrs[64] = {};
    static void *ctx_of[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    void *ctx = current_context();
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev] || ctx_of[dev] != ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess)
            return nullptr;
        ptrs[dev] = static_cast<unsigned int *>(p);
        ctx_of[dev] = ctx;
    }
    return ptrs[dev];
}

cudaError_t read_and_clear_device_status(unsigned int *word) {
    cudaError_t e = cudaMemcpyFromSymbol(word, g_device_status, sizeof(unsigned int));
    if (e != cudaSuccess)
        return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_device_status, &zero, sizeof(unsigned int));
}

}  // namespace dcn1d

using namespace dcn1d;

extern "C" {

int64_t dcn1d_out_length_lr(int64_t L_in, int64_t K, int64_t stride, int64_t padding_left,
                            int64_t padding_right, int64_t dilation) {
    if (L_in < 1 || K < 1 || stride < 1 || padding_left < 0 || padding_right < 0 ||
        dilation < 1)
        return -1;
    // Arguments past 2^31 are refused so the products below cannot overflow.
    const int64_t lim = (int64_t)1 << 31;
    if (L_in > lim || K > lim || stride > lim || padding_left > lim || padding_right > lim ||
        dilation > lim)
        return -1;
    const int64_t num = L_in + padding_left + padding_right - dilation * (K - 1) - 1;
    if (num < 0)
        return -1;
    return num / stride + 1;
}

int64_t dcn1d_out_length(int64_t L_in, int64_t K, int64_t stride, int64_t padding,
                         int64_t dilation) {
    return dcn1d_out_length_lr(L_in, K, stride, padding, padding, dilation);
}

const char *dcn1d_status_string(int status) {
    switch (status) {
    case DCN1D_OK: return "DCN1D_OK";
    case DCN1D_ERR_NULL: return "DCN1D_ERR_NULL";
    case DCN1D_ERR_DTYPE: return "DCN1D_ERR_DTYPE";
    case DCN1D_ERR_SHAPE: return "DCN1D_ERR_SHAPE";
    case DCN1D_ERR_ARG: return "DCN1D_ERR_ARG";
    case DCN1D_ERR_UNSUPPORTED: return "DCN1D_ERR_UNSUPPORTED";
    case DCN1D_ERR_LAUNCH: return "DCN1D_ERR_LAUNCH";
    case DCN1D_ERR_TIMEOUT: return "DCN1D_ERR_TIMEOUT";
    case DCN1D_ERR_CUDA: return "DCN1D_ERR_CUDA";
    default: return "DCN1D_UNKNOWN_STATUS";
    }
}

int dcn1d_forward_lr(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                     const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                     const dcn1d_tensor *bias, int64_t stride, int64_t padding_left,
                     int64_t padding_right, int64_t dilation, int64_t groups,
                     int64_t offset_groups, int unconstrained, dcn1d_tensor *out,
                     void *workspace, size_t workspace_bytes, void *stream) {
    g_last_launches = 0;
    Problem P;
    int st = validate(x, offsets, mask, weight, bias, stride, padding_left, padding_right,
                      dilation, groups, offset_groups, unconstrained, out, &P);
    if (st != DCN1D_OK)
        return st;
    if (workspace_bytes > 0 && !workspace)
        return DCN1D_ERR_NULL;
    if (P.B == 0)
        return DCN1D_OK;   // empty batch: nothing to compute
    int launches = 0;
    if (run_forward(P, workspace, workspace ? workspace_bytes : 0,
                    static_cast<cudaStream_t>(stream), &launches) != cudaSuccess)
        return DCN1D_ERR_LAUNCH;
    g_last_launches = launches;
    return DCN1D_OK;
}

int dcn1d_forward_ws(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                     const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                     const dcn1d_tensor *bias, int64_t stride, int64_t padding, int64_t dilation,
                     int64_t groups, int64_t offset_groups, int unconstrained, dcn1d_tensor *out,
                     void *workspace, size_t workspace_bytes, void *stream) {
    return dcn1d_forward_lr(x, offsets, mask, weight, bias, stride, padding, padding, dilation,
                            groups, offset_groups, unconstrained, out, workspace, workspace_bytes,
                            stream);
}

int dcn1d_forward(const dcn1d_tensor *x, const dcn1d_tensor *offsets, const dcn1d_tensor *mask,
                  const dcn1d_tensor *weight, const dcn1d_tensor *bias, int64_t stride,
                  int64_t padding, int64_t dilation, int64_t groups, int64_t offset_groups,
                  int unconstrained, dcn1d_tensor *out, void *stream) {
    return dcn1d_forward_ws(x, offsets, mask, weight, bias, stride, padding, dilation, groups,
                            offset_groups, unconstrained, out, nullptr, 0, stream);
}

int dcn1d_test_forward_stalled(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                               const dcn1d_tensor *weight, int64_t stride, int64_t padding,
                               int64_t dilation, int64_t groups, int64_t offset_groups,
                               int unconstrained, dcn1d_tensor *out, int64_t wait_limit_ns,
                               void *stream) {
    g_last_launches = 0;
    Problem P;
    int st = validate(x, offsets, nullptr, weight, nullptr, stride, padding, padding, dilation,
                      groups, offset_groups, unconstrained, out, &P);
    if (st != DCN1D_OK)
        return st;
    if (wait_limit_ns < 1000 || wait_limit_ns > 100000000)   // 1 us .. 100 ms
        return DCN1D_ERR_ARG;
    if (P.B == 0 || !tc_bf16_stalled_supported(P))
        return DCN1D_ERR_UNSUPPORTED;
    if (launch_tc_bf16_stalled(P, (uint64_t)wait_limit_ns, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return DCN1D_ERR_LAUNCH;
    g_last_launches = 1;
    return DCN1D_OK;
}

int64_t dcn1d_forward_lr_workspace_size(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                                        const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                                        const dcn1d_tensor *bias, int64_t stride,
                                        int64_t padding_left, int64_t padding_right,
                                        int64_t dilation, int64_t groups, int64_t offset_groups,
                                        int unconstrained, const dcn1d_tensor *out) {
    Problem P;
    const int st = validate(x, offsets, mask, weight, bias, stride, padding_left, padding_right,
                            dilation, groups, offset_groups, unconstrained, out, &P);
    if (st != DCN1D_OK)
        return -st;
    return (int64_t)workspace_bytes(P);
}

int64_t dcn1d_forward_workspace_size(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                                     const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                                     const dcn1d_tensor *bias, int64_t stride, int64_t padding,
                                     int64_t dilation, int64_t groups, int64_t offset_groups,
                                     int unconstrained, const dcn1d_tensor *out) {
    return dcn1d_forward_lr_workspace_size(x, offsets, mask, weight, bias, stride, padding,
                                           padding, dilation, groups, offset_groups,
                                           unconstrained, out);
}

const char *dcn1d_backward_kernel_name(
    const dcn1d_tensor *x, const dcn1d_tensor *offsets, const dcn1d_tensor *mask,
    const dcn1d_tensor *weight, const dcn1d_tensor *grad_out, int64_t stride,
    int64_t padding_left, int64_t padding_right, int64_t dilation, int64_t groups,
    int64_t offset_groups, int unconstrained, const dcn1d_tensor *grad_x,
    const dcn1d_tensor *grad_offsets, const dcn1d_tensor *grad_mask,
    const dcn1d_tensor *grad_weight, const dcn1d_tensor *grad_bias) {
    Problem P;
    BackwardGrads G;
    if (validate_backward(x, offsets, mask, weight, grad_out, stride, padding_left, padding_right,
                          dilation, groups, offset_groups, unconstrained, grad_x, grad_offsets,
                          grad_mask, grad_weight, grad_bias, &P, &G) != DCN1D_OK)
        return nullptr;
    return backward_uses_tensor_cores(P, G) ? "tcgen05_gemm" : "cuda_core_gemm";
}

int64_t dcn1d_backward_lr_workspace_size(
    const dcn1d_tensor *x, const dcn1d_tensor *offsets, const dcn1d_tensor *mask,
    const dcn1d_tensor *weight, const dcn1d_tensor *grad_out, int64_t stride,
    int64_t padding_left, int64_t padding_right, int64_t dilation, int64_t groups,
    int64_t offset_groups, int unconstrained, const dcn1d_tensor *grad_x,
    const dcn1d_tensor *grad_offsets, const dcn1d_tensor *grad_mask,
    const dcn1d_tensor *grad_weight, const dcn1d_tensor *grad_bias) {
    Problem P;
    BackwardGrads G;
    const int st = validate_backward(x, offsets, mask, weight, grad_out, stride, padding_left,
                                     padding_right, dilation, groups, offset_groups,
                                     unconstrained, grad_x, grad_offsets, grad_mask, grad_weight,
                                     grad_bias, &P, &G);
    if (st != DCN1D_OK)
        return -(int64_t)st;
    return (int64_t)backward_workspace(P, G);
}

int64_t dcn1d_backward_workspace_size(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                                      const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                                      const dcn1d_tensor *grad_out, int64_t stride,
                                      int64_t padding, int64_t dilation, int64_t groups,
                                      int64_t offset_groups, int unconstrained,
                                      const dcn1d_tensor *grad_x, const dcn1d_tensor *grad_offsets,
                                      const dcn1d_tensor *grad_mask,
                                      const dcn1d_tensor *grad_weight,
                                      const dcn1d_tensor *grad_bias) {
    return dcn1d_backward_lr_workspace_size(x, offsets, mask, weight, grad_out, stride, padding,
                                            padding, dilation, groups, offset_groups,
                                            unconstrained, grad_x, grad_offsets, grad_mask,
                                            grad_weight, grad_bias);
}

int dcn1d_backward_lr(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                      const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                      const dcn1d_tensor *grad_out, int64_t stride, int64_t padding_left,
                      int64_t padding_right, int64_t dilation, int64_t groups,
                      int64_t offset_groups, int unconstrained, dcn1d_tensor *grad_x,
                      dcn1d_tensor *grad_offsets, dcn1d_tensor *grad_mask,
                      dcn1d_tensor *grad_weight, dcn1d_tensor *grad_bias, void *workspace,
                      size_t workspace_bytes, void *stream) {
    g_last_launches = 0;
    Problem P;
    BackwardGrads G;
    const int st = validate_backward(x, offsets, mask, weight, grad_out, stride, padding_left,
                                     padding_right, dilation, groups, offset_groups,
                                     unconstrained, grad_x, grad_offsets, grad_mask, grad_weight,
                                     grad_bias, &P, &G);
    if (st != DCN1D_OK)
        return st;
    const size_t need = backward_workspace(P, G);
    if (need > 0 && !workspace)
        return DCN1D_ERR_NULL;
    if (need > workspace_bytes || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return DCN1D_ERR_ARG;
    int launches = 0;
    if (launch_backward(P, G, workspace, static_cast<cudaStream_t>(stream), &launches) !=
        cudaSuccess)
        return DCN1D_ERR_LAUNCH;
    g_last_launches = launches;
    return DCN1D_OK;
}

int dcn1d_backward(const dcn1d_tensor *x, const dcn1d_tensor *offsets, const dcn1d_tensor *mask,
                   const dcn1d_tensor *weight, const dcn1d_tensor *grad_out, int64_t stride,
                   int64_t padding, int64_t dilation, int64_t groups, int64_t offset_groups,
                   int unconstrained, dcn1d_tensor *grad_x, dcn1d_tensor *grad_offsets,
                   dcn1d_tensor *grad_mask, dcn1d_tensor *grad_weight, dcn1d_tensor *grad_bias,
                   void *workspace, size_t workspace_bytes, void *stream) {
    return dcn1d_backward_lr(x, offsets, mask, weight, grad_out, stride, padding, padding,
                             dilation, groups, offset_groups, unconstrained, grad_x,
                             grad_offsets, grad_mask, grad_weight, grad_bias, workspace,
                             workspace_bytes, stream);
}

const char *dcn1d_forward_lr_kernel_name(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                                         const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                                         const dcn1d_tensor *bias, int64_t stride,
                                         int64_t padding_left, int64_t padding_right,
                                         int64_t dilation, int64_t groups, int64_t offset_groups,
                                         int unconstrained, const dcn1d_tensor *out) {
    Problem P;
    if (validate(x, offsets, mask, weight, bias, stride, padding_left, padding_right, dilation,
                 groups, offset_groups, unconstrained, out, &P) != DCN1D_OK)
        return nullptr;
    const Kernel k = select_kernel(P, SIZE_MAX);
    if (k == kTcBf16 && P.dtype == DCN1D_F16)
        return "tcgen05_f16";   // the same 16-bit tensor-core kernel with fp16 operands
    return kernel_names[k];
}

const char *dcn1d_forward_kernel_name(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                                      const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                                      const dcn1d_tensor *bias, int64_t stride, int64_t padding,
                                      int64_t dilation, int64_t groups, int64_t offset_groups,
                                      int unconstrained, const dcn1d_tensor *out) {
    return dcn1d_forward_lr_kernel_name(x, offsets, mask, weight, bias, stride, padding, padding,
                                        dilation, groups, offset_groups, unconstrained, out);
}

int dcn1d_last_launch_count(void) { return g_last_launches; }

void dcn1d_set_timing_events(void *begin, void *end) {
    g_time_begin = static_cast<cudaEvent_t>(begin);
    g_time_end = static_cast<cudaEvent_t>(end);
}

int dcn1d_device_status(void *stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return DCN1D_ERR_CUDA;
    unsigned int word = 0;
    if (read_and_clear_device_status(&word) != cudaSuccess)
        return DCN1D_ERR_CUDA;
    return word ? DCN1D_ERR_TIMEOUT : DCN1D_OK;
}

int dcn1d_sample_index(const dcn1d_tensor *offsets, int64_t L_in, int64_t stride,
                       int64_t padding, int64_t dilation, int unconstrained, int32_t *i0,
                       float *frac, void *stream) {
    int st = check_desc(offsets, 4);
    if (st != DCN1D_OK)
        return st;
    const int64_t B = offsets->shape[0], G = offsets->shape[1], L_out = offsets->shape[2],
                  K = offsets->shape[3];
    const int64_t n = numel(offsets);
    if (n > 0 && (!i0 || !frac))
        return DCN1D_ERR_NULL;
    if (stride < 1 || padding < 0 || dilation < 1 || L_in < 1 || K < 1)
        return DCN1D_ERR_ARG;
    if (stride >= kMaxPos || padding >= kMaxPos || dilation >= kMaxPos || K >= kMaxPos ||
        L_in >= kMaxPos)
        return DCN1D_ERR_UNSUPPORTED;
    const int64_t want = dcn1d_out_length(L_in, K, stride, padding, dilation);
    if (want < 1)
        return DCN1D_ERR_ARG;
    if (L_out != want)
        return DCN1D_ERR_SHAPE;
    if ((L_out - 1) * stride + dilation * (K - 1) >= kMaxPos || n >= kMaxElems)
        return DCN1D_ERR_UNSUPPORTED;
    if (n == 0)
        return DCN1D_OK;
    cudaError_t err = launch_sample_index(offsets->data, offsets->dtype, (int)B, (int)G,
                                          (int)L_out, (int)K, (int)L_in, (int)stride,
                                          (int)padding, (int)dilation, unconstrained,
                                          i0, frac, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? DCN1D_OK : DCN1D_ERR_LAUNCH;
}

int dcn1d_packed_trunk(const dcn1d_tensor *x, const dcn1d_tensor *dw_weight,
                       const dcn1d_tensor *dw_bias, const dcn1d_tensor *off_weight,
                       const dcn1d_tensor *off_bias, const dcn1d_tensor *mask_weight,
                       const dcn1d_tensor *mask_bias, int64_t stride, int64_t padding_left,
                       int64_t padding_right, int64_t dilation, int64_t offset_groups,
                       dcn1d_tensor *offsets_out, dcn1d_tensor *mask_out, void *stream) {
    g_last_launches = 0;
    TrunkProblem T;
    int st = validate_trunk(x, dw_weight, dw_bias, off_weight, off_bias, mask_weight, mask_bias,
                            stride, padding_left, padding_right, dilation, offset_groups,
                            offsets_out, mask_out, false, &T);
    if (st != DCN1D_OK)
        return st;
    if (T.B == 0)
        return DCN1D_OK;
    const char *name = nullptr;
    if (launch_trunk(T, static_cast<cudaStream_t>(stream), &name) != cudaSuccess)
        return DCN1D_ERR_LAUNCH;
    g_last_launches = 1;
    return DCN1D_OK;
}

const char *dcn1d_packed_trunk_kernel_name(
    const dcn1d_tensor *x, const dcn1d_tensor *dw_weight, const dcn1d_tensor *dw_bias,
    const dcn1d_tensor *off_weight, const dcn1d_tensor *off_bias,
    const dcn1d_tensor *mask_weight, const dcn1d_tensor *mask_bias, int64_t stride,
    int64_t padding_left, int64_t padding_right, int64_t dilation, int64_t offset_groups,
    const dcn1d_tensor *offsets_out, const dcn1d_tensor *mask_out) {
    TrunkProblem T;
    if (validate_trunk(x, dw_weight, dw_bias, off_weight, off_bias, mask_weight, mask_bias,
                       stride, padding_left, padding_right, dilation, offset_groups, offsets_out,
                       mask_out, false, &T) != DCN1D_OK)
        return nullptr;
    return trunk_tc_supported(T) ? "trunk_tcgen05" : "trunk_simt";
}

const char *dcn1d_packed_forward_kernel_name(
    const dcn1d_tensor *x, const dcn1d_tensor *dw_weight, const dcn1d_tensor *dw_bias,
    const dcn1d_tensor *off_weight, const dcn1d_tensor *off_bias,
    const dcn1d_tensor *mask_weight, const dcn1d_tensor *mask_bias, const dcn1d_tensor *weight,
    const dcn1d_tensor *bias, int64_t stride, int64_t padding_left, int64_t padding_right,
    int64_t dilation, int64_t groups, int64_t offset_groups, int unconstrained,
    const dcn1d_tensor *offsets_out, const dcn1d_tensor *mask_out, const dcn1d_tensor *out) {
    TrunkProblem T;
    Problem P;
    dcn1d_tensor od, md;
    PackedLayout lay;
    if (packed_prepare(x, dw_weight, dw_bias, off_weight, off_bias, mask_weight, mask_bias,
                       weight, bias, stride, padding_left, padding_right, dilation, groups,
                       offset_groups, unconstrained, offsets_out, mask_out, out, nullptr, &T, &od,
                       &md, &P, &lay) != DCN1D_OK)
        return nullptr;
    if (lay.fused)
        return "packed_fused_tcgen05";
    // two launches: the trunk, then the forward on the predicted tensors
    static const char *names[2][4] = {
        {"trunk_simt+direct", "trunk_simt+depthwise", "trunk_simt+tcgen05_bf16",
         "trunk_simt+tcgen05_3xtf32"},
        {"trunk_tcgen05+direct", "trunk_tcgen05+depthwise", "trunk_tcgen05+tcgen05_bf16",
         "trunk_tcgen05+tcgen05_3xtf32"}};
    return names[trunk_tc_supported(T) ? 1 : 0][select_kernel(P, SIZE_MAX)];
}

int64_t dcn1d_packed_forward_workspace_size(
    const dcn1d_tensor *x, const dcn1d_tensor *dw_weight, const dcn1d_tensor *dw_bias,
    const dcn1d_tensor *off_weight, const dcn1d_tensor *off_bias,
    const dcn1d_tensor *mask_weight, const dcn1d_tensor *mask_bias, const dcn1d_tensor *weight,
    const dcn1d_tensor *bias, int64_t stride, int64_t padding_left, int64_t padding_right,
    int64_t dilation, int64_t groups, int64_t offset_groups, int unconstrained,
    const dcn1d_tensor *offsets_out, const dcn1d_tensor *mask_out, const dcn1d_tensor *out) {
    TrunkProblem T;
    Problem P;
    dcn1d_tensor od, md;
    PackedLayout lay;
    const int st = packed_prepare(x, dw_weight, dw_bias, off_weight, off_bias, mask_weight,
                                  mask_bias, weight, bias, stride, padding_left, padding_right,
                                  dilation, groups, offset_groups, unconstrained, offsets_out,
                                  mask_out, out, nullptr, &T, &od, &md, &P, &lay);
    if (st != DCN1D_OK)
        return -(int64_t)st;
    return (int64_t)lay.total;
}

int dcn1d_packed_forward(const dcn1d_tensor *x, const dcn1d_tensor *dw_weight,
                         const dcn1d_tensor *dw_bias, const dcn1d_tensor *off_weight,
                         const dcn1d_tensor *off_bias, const dcn1d_tensor *mask_weight,
                         const dcn1d_tensor *mask_bias, const dcn1d_tensor *weight,
                         const dcn1d_tensor *bias, int64_t stride, int64_t padding_left,
                         int64_t padding_right, int64_t dilation, int64_t groups,
                         int64_t offset_groups, int unconstrained, dcn1d_tensor *offsets_out,
                         dcn1d_tensor *mask_out, dcn1d_tensor *out, void *workspace,
                         size_t workspace_bytes, void *stream) {
    g_last_launches = 0;
    if (workspace_bytes > 0 && !workspace)
        return DCN1D_ERR_NULL;
    TrunkProblem T;
    Problem P;
    dcn1d_tensor od, md;
    PackedLayout lay;
    char *ws = static_cast<char *>(workspace);
    int st = packed_prepare(x, dw_weight, dw_bias, off_weight, off_bias, mask_weight, mask_bias,
                            weight, bias, stride, padding_left, padding_right, dilation, groups,
                            offset_groups, unconstrained, offsets_out, mask_out, out,
                            ws ? ws : nullptr, &T, &od, &md, &P, &lay);
    if (st != DCN1D_OK)
        return st;
    if (lay.fwd_offset > 0 && (!ws || workspace_bytes < lay.fwd_offset))
        return ws ? DCN1D_ERR_ARG : DCN1D_ERR_NULL;   // no room for the predicted tensors
    if (T.B == 0)
        return DCN1D_OK;
    if (lay.fused) {
        if (launch_packed_fused(T, P, static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return DCN1D_ERR_LAUNCH;
        g_last_launches = 1;
        return DCN1D_OK;
    }
    T.off_out = od.data;
    T.mask_out = mask_weight ? md.data : nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const char *name = nullptr;
    if (launch_trunk(T, s, &name) != cudaSuccess)
        return DCN1D_ERR_LAUNCH;
    int launches = 0;
    const size_t rest = workspace_bytes - lay.fwd_offset;
    if (run_forward(P, rest > 0 ? ws + lay.fwd_offset : nullptr, rest, s, &launches) !=
        cudaSuccess)
        return DCN1D_ERR_LAUNCH;
    g_last_launches = 1 + launches;
    return DCN1D_OK;
}

}  // extern "C"
